"""fa_bwd_noalloc: the backward pass for callers that may not allocate device memory
(e.g. a plugin whose host framework owns all device memory and forbids direct cudaMalloc,
or a loop that cannot afford cudaMalloc's implicit device-wide synchronisation).  Its
workspace is a fixed array inside the library; these tests check that it reproduces
fa_bwd (which takes a caller-allocated workspace) on consecutive calls, and that problems
too large for the built-in array are refused before anything runs.

Kept in a file that pytest collects last, so a failure here does not hide the others."""
import math

import pytest
import torch

import synthetic
from tests._helpers import GRAD_REL_L2, cuda, rel_l2, to_np


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    return mod


def test_oversized_problem_is_refused_before_launch(fa, no_visible_gpu):
    a16 = 1 << 20  # never dereferenced: the call must fail on the size check
    ptrs = [a16] * 9
    # B*H*N*d*4 bytes of dQ accumulator alone exceed the 64 MiB built-in workspace
    assert fa.fa_bwd_workspace_bytes(1, 16, 8192, 128) > fa.NOALLOC_WORKSPACE_BYTES
    assert fa.fa_bwd_noalloc(*ptrs, 1, 16, 8192, 128, 1, 0.088, stream=0) == fa.FA_ERR_WORKSPACE
    assert fa.fa_bwd_noalloc(None, *ptrs[1:], 1, 1, 128, 128, 1, 0.088, stream=0) == fa.FA_ERR_INVALID_ARG


def _both(fa, B, N, H, d, causal, seed):
    t = synthetic.draw(B, N, H, d, seed, "bf16", with_grad=True)
    q, k, v, dO = cuda(t, ("q", "k", "v", "dO"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    ref = fa.attention_backward(q, k, v, o, lse, dO, causal=causal, scale=scale)
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    rc = fa.fa_bwd_noalloc(q, k, v, o, lse, dO, *got, B, H, N, d, causal, scale)
    assert rc == fa.FA_OK, fa.status_string(rc)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == fa.FA_OK
    return ref, got


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_consecutive_calls(fa):
    # Two calls in a row on different problems, then the first one again: each must match
    # fa_bwd, so nothing a previous call left in the shared array leaks into the next.
    for (B, N, H, d, causal, seed) in [(2, 1000, 3, 128, True, 31), (1, 777, 4, 64, False, 32),
                                       (2, 1000, 3, 128, True, 31)]:
        ref, got = _both(fa, B, N, H, d, causal, seed)
        for name, r, g in zip(("dq", "dk", "dv"), ref, got):
            assert torch.isfinite(g.float()).all(), name
            assert rel_l2(to_np(g), to_np(r)) <= GRAD_REL_L2, name
        # dK and dV are accumulated in a fixed order: identical bits
        assert torch.equal(ref[1], got[1]) and torch.equal(ref[2], got[2])


@pytest.mark.gpu
def test_noalloc_largest_admitted_problem(fa):
    # A problem near the limit (48 MiB of workspace) still runs and matches fa_bwd.
    B, N, H, d = 1, 4096, 24, 128
    assert fa.fa_bwd_workspace_bytes(B, H, N, d) <= fa.NOALLOC_WORKSPACE_BYTES
    ref, got = _both(fa, B, N, H, d, True, 33)
    for name, r, g in zip(("dq", "dk", "dv"), ref, got):
        assert rel_l2(to_np(g), to_np(r)) <= GRAD_REL_L2, name
