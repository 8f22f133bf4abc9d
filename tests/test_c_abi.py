"""The boundary as a C program sees it: tests/c_abi_check.c includes the public headers as
C99 (no C++), links libfa.so and checks the host-side promises of include/fa.h without a
GPU.  Compiled with gcc and run here."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libdir():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa
    return os.path.dirname(fa.LIB_PATH)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c99_program_links_and_sees_the_documented_behaviour(libdir, tmp_path):
    exe = str(tmp_path / "c_abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
           "-o", exe, "-L", libdir, "-l:libfa.so", f"-Wl,-rpath,{libdir}", "-lm"]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    # Hide any GPU: every call in the program must be refused before the library needs one.
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    run = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "all checks passed" in run.stdout
