"""The deterministic dQ kernel's barrier protocol (two S buffers, issue order dP(j+1), dQ(j),
S(j+2), K ring of 3 and V ring of 2), run as a discrete-event model under random schedules
(tests/bwdq_protocol_model.py) for one to twenty key tiles; and two mutated protocols the model
must reject.  (A two-stage K ring is safe but serialises S(j+2) behind dQ(j).)"""
import importlib.util
import os
import tempfile

from tests import bwdq_protocol_model as model


def test_dq_kernel_protocol_is_safe():
    for nkv in list(range(1, 12)) + [16, 20]:
        for seed in range(40):
            assert model.run(nkv, seed) == "ok", (nkv, seed)


def _mutant(a, b):
    src = open(model.__file__).read()
    assert src.count(a) == 1, a
    d = tempfile.mkdtemp()
    path = os.path.join(d, "mutant.py")
    with open(path, "w") as f:
        f.write(src.replace(a, b))
    spec = importlib.util.spec_from_file_location("mutant", path)
    mutant = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mutant)
    return mutant


def _caught(mutant, nkv=6, seeds=40):
    n = 0
    for seed in range(seeds):
        try:
            mutant.run(nkv, seed)
        except (mutant.Hazard, mutant.Deadlock):
            n += 1
    return n


def test_model_sees_s_issued_before_dq():
    """S(j+2) ahead of dQ(j) would overwrite dS_j before dQ reads it."""
    mutant = _mutant('''            st["issued"]["dQ"] += 1
            st["k_pending"][j] = st["k_pending"].get(j, 0) + 1
            pipe.append(("dQ", j))
            pipe.append(("C", f"k_empty{j % kstages}"))
            if j + 2 < nkv:
                yield from issue_s(j + 2)''', '''            if j + 2 < nkv:
                yield from issue_s(j + 2)
            st["issued"]["dQ"] += 1
            st["k_pending"][j] = st["k_pending"].get(j, 0) + 1
            pipe.append(("dQ", j))
            pipe.append(("C", f"k_empty{j % kstages}"))''')
    assert _caught(mutant) == 40


def test_model_sees_an_early_k_release():
    """Committing the K stage's release ahead of dQ(j) would let K_{j+3} land over K_j while
    dQ(j) still has to read it."""
    mutant = _mutant('''            pipe.append(("dQ", j))
            pipe.append(("C", f"k_empty{j % kstages}"))''', '''            pipe.append(("C", f"k_empty{j % kstages}"))
            pipe.append(("dQ", j))''')
    assert _caught(mutant, nkv=8, seeds=200) > 0
