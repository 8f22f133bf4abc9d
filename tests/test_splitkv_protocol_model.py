"""The split-KV decoding kernel's barrier protocol as a discrete-event model with parity
waits and random schedules (tests/splitkv_protocol_model.py): ring depths 3 (head dim 128)
and 4 (64), slices of 0 to 16 key tiles, the softmax's conditional wait for the previous PV
before a rescale of O."""
import importlib.util
import os
import tempfile

import pytest

from tests import splitkv_protocol_model as model


@pytest.mark.parametrize("stages", [3, 4])
def test_splitkv_protocol_is_safe(stages):
    for nkv in [0, 1, 2, 3, 4, 5, 7, 9, 16]:
        for seed in range(60):
            assert model.run(nkv, seed, stages) == "ok"


def _mutant(a, b):
    src = open(model.__file__).read()
    assert src.count(a) == 1
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.py")
        with open(path, "w") as f:
            f.write(src.replace(a, b))
        spec = importlib.util.spec_from_file_location("mutant", path)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    return mod


def test_model_sees_a_skipped_pv_wait():
    """Rescaling O without waiting for the previous PV must be reported."""
    m = _mutant('''                yield ("wait", "pv_done", n - 1)
''', "")
    caught = 0
    for seed in range(40):
        try:
            m.run(6, seed, need_prob=1.0)
        except m.Hazard:
            caught += 1
    assert caught > 0
