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
    m0, m1 = [], []
    for _ in range(units):
        p = rng.randrange(max(1, (nt + 1) // 2))
        lists = []
        for t in (0, 1):
            qt = 2 * p + t
            vis = range(nt) if not causal else range(min(nt, qt + 1))
            lists.append(sorted(j for j in vis if qt < nt and rng.random() < density))
        m0.append(lists[0])
        m1.append(lists[1])
    return m0, m1


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
        m0, m1 = _random_masks(rng, rng.randrange(1, 5), rng.randrange(1, 12),
                               rng.random() < 0.5, rng.choice([0.0, 0.2, 0.5, 0.9, 1.0]))
        for sched in range(4):
            assert model.run("sparse", m0, m1, None, seed=100 * case + sched,
                             stages=stages) == "ok"


def test_model_sees_the_empty_tile_race():
    """Unit 0: both query tiles have work; unit 1: both are empty.  With the earlier logic
    the second unit's o_done commits can land before the softmax warpgroups poll the
    first, which some schedule must expose."""
    m0, m1 = [[0], []], [[0, 1], []]
    failures = 0
    for seed in range(40):
        try:
            model.run("sparse", m0, m1, None, seed=seed, empty_tile_waits_o_free=False)
        except (model.Deadlock, model.Hazard):
            failures += 1
        assert model.run("sparse", m0, m1, None, seed=seed) == "ok"
    assert failures > 0
