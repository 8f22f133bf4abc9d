"""The backward key-tile kernel's barrier protocol, run as a discrete-event model with the
hardware's parity-wait semantics under random schedules (tests/bwd_protocol_model.py), with
and without the dQ product (the deterministic path drops it), for query-tile counts from
one (the last key tile under the causal mask) to twenty."""
import pytest

from tests import bwd_protocol_model as model


@pytest.mark.parametrize("with_dq", [True, False])
def test_backward_protocol_is_safe(with_dq):
    for nq in list(range(1, 10)) + [16, 20]:
        for seed in range(40):
            assert model.run(nq, seed, with_dq) == "ok"


def test_model_sees_a_reordered_product():
    """Issuing S^T(n+1) before dV(n) would overwrite P^T(n) before it is read: the model
    must report it under every schedule."""
    import importlib.util
    import os
    import tempfile
    src = open(model.__file__).read()
    a = '''            issue("dV", n)
            commit(f"do_empty{n % 2}")
            if n + 1 < nq:
                yield from issue_s(n + 1)'''
    b = '''            if n + 1 < nq:
                yield from issue_s(n + 1)
            issue("dV", n)
            commit(f"do_empty{n % 2}")'''
    assert src.count(a) == 1
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.py")
        with open(path, "w") as f:
            f.write(src.replace(a, b))
        spec = importlib.util.spec_from_file_location("mutant", path)
        mutant = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mutant)
        for seed in range(10):
            with pytest.raises(mutant.Hazard):
                mutant.run(4, seed)
