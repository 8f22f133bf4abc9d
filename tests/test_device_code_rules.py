"""Static checks of the CUDA sources for the library's failure rules: no device code traps,
asserts or spins without a bound.  Every wait on an mbarrier goes through the bounded
`mbar_wait` (a time limit read from %globaltimer, after which the CTA records a status and
tears down), which is the only open-ended loop in the device code."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_88_b200", "csrc")


def _sources():
    files = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                   + glob.glob(os.path.join(CSRC, "*.h")))
    assert files
    for f in files:
        txt = open(f).read()
        # Comments removed: the rules are about code.
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        txt = re.sub(r"//[^\n]*", "", txt)
        yield os.path.basename(f), txt


def test_no_trap_or_device_assert():
    for name, txt in _sources():
        assert "__trap" not in txt, name
        assert not re.search(r"\btrap\s*;", txt), name
        assert not re.search(r"(?<![\w.])assert\s*\(", txt), name


def test_raw_barrier_polls_only_inside_the_bounded_wait():
    for name, txt in _sources():
        uses = [m.start() for m in re.finditer(r"\bmbar_try_wait\s*\(", txt)]
        if name != "ptx.cuh":
            assert not uses, f"{name} polls an mbarrier outside mbar_wait"
            continue
        # Definition plus the two polls inside mbar_wait.
        body = txt[txt.index("bool mbar_wait("):]
        body = body[:body.index("\n}\n")]
        assert len(uses) == 3 and body.count("mbar_try_wait(") == 2
        assert "globaltimer_ns() - t0 > timeout_ns" in body and "FA_ERR_TIMEOUT" in body


def test_no_open_ended_loops_outside_the_bounded_wait():
    for name, txt in _sources():
        loops = re.findall(r"for\s*\([^;()]*;\s*;[^)]*\)|while\s*\(\s*(?:true|1)\s*\)", txt)
        allowed = 1 if name == "ptx.cuh" else 0  # mbar_wait's poll loop
        assert len(loops) == allowed, (name, loops)
