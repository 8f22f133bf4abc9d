"""The forward kernel's barrier protocol, run as a discrete-event model with the hardware's
parity-wait semantics under random schedules (tests/fwd_protocol_model.py): dense and
block-sparse issue orders, K/V rings of 2 and 4 stages, several units per CTA.  The model
found the block-sparse empty-query-tile race that the kernel now avoids (an empty tile's
o_done committed without waiting for o_free); the earlier logic is kept as a switch so
that the model's power to see it is itself checked."""
import random

import pytest

from tests import fwd_protocol_model as model


def _random_masks(rng, units, nt, causal, density):
    return model.random_masks(rng, units, nt, causal, density)


@pytest.mark.parametrize("stages,split_p", [(2, False), (4, False), (4, True)])
def test_dense_issue_order_is_safe(stages, split_p):
    """Dense order (head dim 128: 2 stages; 64: 4 stages; 8-bit: 4 stages with P published
    in halves)."""
    rng = random.Random(stages + 10 * split_p)
    for case in range(200):
        nkv = []
        for _ in range(rng.randrange(1, 5)):
            a = rng.randrange(1, 9)
            nkv.append((a, a + rng.randrange(0, 2)))  # causal pairs: tile 1 sees one more
        for sched in range(4):
            assert model.run("dense", None, None, nkv, seed=100 * case + sched,
                             stages=stages, split_p=split_p) == "ok"


@pytest.mark.parametrize("stages", [2, 4])
def test_block_sparse_issue_order_is_safe(stages):
    rng = random.Random(10 + stages)
    for case in range(600):
        m0 = _random_masks(rng, rng.randrange(1, 5), rng.randrange(1, 12),
                           rng.random() < 0.5, rng.choice([0.0, 0.2, 0.5, 0.9, 1.0]))
        for sched in range(4):
            assert model.run("sparse", m0, None, None, seed=100 * case + sched,
                             stages=stages) == "ok"


def test_model_sees_the_empty_tile_race():
    """Unit 0: both slots have work; unit 1: the query tile has no active key tile.  If an
    empty slot's o_done were committed without waiting for o_free, the second unit's commits
    could land before warpgroup 0 polls the first, which some schedule must expose."""
    m0 = [[0, 1], []]
    failures = 0
    for seed in range(40):
        try:
            model.run("sparse", m0, None, None, seed=seed, empty_tile_waits_o_free=False)
        except (model.Deadlock, model.Hazard):
            failures += 1
        assert model.run("sparse", m0, None, None, seed=seed) == "ok"
    assert failures > 0


def test_model_sees_a_missing_merge_handshake():
    """Block-sparse: without warpgroup 1's wait for merge_free, it can publish the next
    unit's row maximum and sum over values warpgroup 0 has not read yet."""
    import importlib.util
    import os
    import tempfile
    src = open(model.__file__).read()
    a = '''                if u > 0:
                    yield ("wait", "merge_free", u - 1)
'''
    assert src.count(a) == 1
    d = tempfile.mkdtemp()
    path = os.path.join(d, "mutant.py")
    with open(path, "w") as f:
        f.write(src.replace(a, ""))
    spec = importlib.util.spec_from_file_location("mutant", path)
    mutant = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mutant)
    caught = 0
    for seed in range(60):
        try:
            mutant.run("sparse", [[0], [], [], [1, 2]], None, None, seed=seed)
        except (mutant.Hazard, mutant.Deadlock):
            caught += 1
    assert caught > 0
