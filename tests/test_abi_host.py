"""Host-side checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments with the documented status before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(autouse=True)
def _host_only(no_visible_gpu):
    """Every call below passes fake device addresses (see no_visible_gpu)."""


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    return mod


def declared_functions():
    names = []
    for h in ("fa.h", "fa_debug.h"):
        txt = open(os.path.join(ROOT, "include", h)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(fa_[a-z0-9_]+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(fa):
    names = declared_functions()
    assert len(names) >= 9
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(fa.EXPORTED) == names


def test_status_strings_and_version(fa):
    assert fa.version() == 100
    assert fa.status_string(0) == "ok"
    assert "timed out" in fa.status_string(fa.FA_ERR_TIMEOUT)
    assert fa.status_string(12345) == "unknown status"


def test_workspace_size_formula(fa):
    def up(x):
        return (x + 255) // 256 * 256
    for B, H, N, d in [(1, 16, 4096, 128), (2, 3, 1000, 64), (1, 1, 1, 64)]:
        rows = B * H * N
        padded = B * H * ((N + 127) // 128 * 128)
        # status word slot + dQ accumulator + D + base-2 logsumexp
        assert fa.fa_bwd_workspace_bytes(B, H, N, d) == 256 + up(rows * d * 4) + 2 * up(padded * 4)
    assert fa.fa_bwd_workspace_bytes(0, 1, 1, 64) == 0
    assert fa.fa_bwd_workspace_bytes(1, 1, -5, 64) == 0


A16 = 1 << 20  # a fake, 16-byte aligned "device address": never dereferenced


@pytest.mark.parametrize("args,code", [
    (dict(q=0), 1),
    (dict(B=0), 1),
    (dict(N=-1), 1),
    (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1),
    (dict(scale=0.0), 1),
    (dict(scale=-0.125), 1),
    (dict(d=96), 2),
    (dict(d=256), 2),
    (dict(q=A16 + 8), 3),
    (dict(o=A16 + 2), 3),
])
def test_fwd_rejects_bad_arguments_without_launching(fa, args, code):
    a = dict(q=A16, k=A16, v=A16, o=A16, lse=A16, B=1, H=1, N=128, d=64, causal=0, scale=0.125)
    a.update(args)
    rc = fa.fa_fwd(a["q"] or None, a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                   a["d"], a["causal"], a["scale"], stream=0)
    assert rc == code


def test_bwd_rejects_bad_arguments_without_launching(fa):
    base = [A16] * 9
    ok_ws = fa.fa_bwd_workspace_bytes(1, 2, 256, 128)
    call = lambda ptrs, ws, wsb, d=128, N=256: fa.fa_bwd(*ptrs, 1, 2, N, d, 1, 0.1, ws, wsb, stream=0)
    assert call([None] + base[1:], A16, ok_ws) == fa.FA_ERR_INVALID_ARG
    assert call(base, A16, ok_ws, d=80) == fa.FA_ERR_UNSUPPORTED
    assert call(base, None, ok_ws) == fa.FA_ERR_WORKSPACE
    assert call(base, A16, ok_ws - 1) == fa.FA_ERR_WORKSPACE
    assert call(base[:4] + [A16 + 4] + base[5:], A16, ok_ws) == fa.FA_ERR_MISALIGNED
    assert call(base, A16 + 16, ok_ws) == fa.FA_ERR_MISALIGNED


def test_f32_rejects_bad_arguments_without_launching(fa):
    p = [A16] * 5
    assert fa.fa_fwd_f32(*p, 1, 1, 16, 130, 0, 0.1, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_f32(*p, 1, 1, 16, 6, 0, 0.1, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_f32(*p, 1, 1, 0, 64, 0, 0.1, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_f32(A16 + 4, *p[1:], 1, 1, 16, 64, 0, 0.1, stream=0) == fa.FA_ERR_MISALIGNED


def test_fp8_entry_points_reject_bad_arguments_without_launching(fa):
    p = [A16] * 6
    assert fa.fa_fwd_fp8(*p, 1, 2, 256, 64, 0, 0.1, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_fp8(None, *p[1:], 1, 2, 256, 128, 0, 0.1, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8(*p, 1, 2, 256, 128, 0, -1.0, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8(A16 + 8, *p[1:], 1, 2, 256, 128, 0, 0.1, stream=0) == fa.FA_ERR_MISALIGNED
    ws = fa.fa_fp8_quantize_workspace_bytes(2, 3)
    assert ws == 256  # 3 * 2 * 3 words, rounded up
    q = lambda **kw: fa.fa_fp8_quantize(
        kw.get("q", A16), A16, A16, kw.get("signs", None), A16, A16, A16, A16, 2, 3, 100,
        kw.get("d", 128), kw.get("ws", A16), kw.get("wsb", ws), stream=0)
    assert q(d=96) == fa.FA_ERR_UNSUPPORTED
    assert q(q=None) == fa.FA_ERR_INVALID_ARG
    assert q(ws=None) == fa.FA_ERR_WORKSPACE
    assert q(wsb=ws - 1) == fa.FA_ERR_WORKSPACE
    assert q(q=A16 + 2) == fa.FA_ERR_MISALIGNED
    assert q(signs=A16 + 2) == fa.FA_ERR_MISALIGNED


def test_block_sparse_workspace_is_the_packed_mask(fa):
    # 128 bytes of bits per 128-row query tile, rounded up to 256 bytes.
    assert fa.fa_fwd_block_sparse_workspace_bytes(2, 4, 4096, 128) == 32 * 128
    assert fa.fa_fwd_block_sparse_workspace_bytes(1, 1, 1000, 64) == 8 * 128
    assert fa.fa_fwd_block_sparse_workspace_bytes(1, 1, 100, 64) == 256
    base = [A16] * 5
    call = lambda ws, wsb, N=1000: fa.fa_fwd_block_sparse(*base, 1, 2, N, 128, 0, 0.1, A16, ws,
                                                          wsb, stream=0)
    assert call(None, 4096) == fa.FA_ERR_WORKSPACE
    assert call(A16, 1023) == fa.FA_ERR_WORKSPACE
    assert call(A16 + 8, 1024) == fa.FA_ERR_MISALIGNED
    assert call(A16, 1 << 20, N=131073) == fa.FA_ERR_UNSUPPORTED


def test_primitive_self_tests_reject_bad_arguments(fa):
    assert fa.fa_debug_tma_tile(A16, A16, 1, 300, 2, 96, 0, 0, 0, 0, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_debug_tma_tile(A16, A16, 1, 300, 2, 64, 0, 0, 300, 0, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_tma_tile(A16, A16, 1, 300, 2, 64, 0, 0, 0, 1, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_tma_tile(A16 + 8, A16, 1, 300, 2, 64, 0, 0, 0, 0, stream=0) == fa.FA_ERR_MISALIGNED
    assert fa.fa_debug_tmem_roundtrip(A16, A16, 48, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_debug_tmem_roundtrip(None, A16, 64, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_fwd_schedule(1, 1, 128, 0, 0, A16, 4, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_fwd_schedule(1, 1, 128, 0, 4, A16 + 2, 4, stream=0) == fa.FA_ERR_MISALIGNED


def test_debug_entry_points_reject_bad_arguments(fa):
    assert fa.fa_debug_umma_tile(A16, A16, A16, 96, 64, 0, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_debug_umma_tile(A16, A16, A16, 64, 64, 3, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_debug_wait_timeout(10, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_debug_wait_timeout(10_000, A16 + 2, stream=0) == fa.FA_ERR_MISALIGNED
    assert fa.fa_read_device_status(A16 + 2, stream=0) == fa.FA_ERR_MISALIGNED
