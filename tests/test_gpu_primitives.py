"""Single-primitive self-tests on the GPU (fa_debug.h), each against a CPU reference:
a TMA box load through the attention kernels' tensor-map encoding, a tensor-memory
store / load round trip, and the forward kernel's persistent schedule against a Python
model of it.  Plus the memory claim of the source pages: the forward and backward need
O(N d) device memory, never the N x N score matrix."""
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    assert torch.cuda.is_available()
    return mod


@pytest.mark.parametrize("d,b,h,row0,chunk", [
    (64, 0, 0, 0, 0), (64, 1, 1, 256, 0), (64, 0, 2, 299, 0),
    (128, 0, 0, 0, 0), (128, 1, 2, 128, 1), (128, 1, 1, 256, 0), (128, 0, 2, 299, 1),
])
def test_tma_box_load_matches_source(fa, d, b, h, row0, chunk):
    B, N, H = 2, 300, 3
    x = synthetic.draw(B, N, H, d, 8100 + d, "bf16")["q"].cuda()
    y = torch.full((128, 64), float("nan"), device="cuda", dtype=torch.bfloat16)
    assert fa.fa_debug_tma_tile(x, y, B, N, H, d, b, h, row0, chunk) == 0
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    ref = torch.zeros((128, 64), dtype=torch.bfloat16)
    rows = min(128, N - row0)
    ref[:rows] = x[b, row0:row0 + rows, h, 64 * chunk:64 * chunk + 64].cpu()
    assert torch.equal(y.cpu(), ref)  # bitwise, zero fill past N


@pytest.mark.parametrize("ncols", [32, 64, 128, 256])
def test_tmem_store_load_round_trip(fa, ncols):
    g = torch.Generator().manual_seed(ncols)
    src = torch.randint(0, 2 ** 31 - 1, (128, ncols), generator=g, dtype=torch.int64)
    inp = src.to(torch.int32).cuda()
    out = torch.zeros_like(inp)
    assert fa.fa_debug_tmem_roundtrip(inp, out, ncols) == 0
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), inp.cpu())


def _schedule_model(B, H, N, causal, G):
    """The forward's unit order as the kernel's comments state it: round r hands CTA c the
    unit r*G + c (even r) or r*G + G-1-c (odd r); causal units are sorted longest first
    (query-tile pair index descending, heads inside a band), otherwise head-major."""
    num_pairs = (N + 255) // 256
    BH = B * H
    U = BH * num_pairs
    out = []
    for c in range(G):
        seq, r = [], 0
        while True:
            u = r * G + ((G - 1 - c) if r & 1 else c)
            if u >= U:
                break
            if causal:
                pair, bh = num_pairs - 1 - u // BH, u % BH
            else:
                bh, pair = u // num_pairs, u % num_pairs
            seq.append(bh * num_pairs + pair)
            r += 1
        out.append(seq)
    return out, num_pairs, U


@pytest.mark.parametrize("B,H,N,causal,G", [
    (1, 16, 16384, True, 148), (4, 16, 4096, False, 148), (2, 3, 1000, True, 7), (1, 1, 128, False, 5),
])
def test_forward_schedule_matches_model_and_covers_every_unit(fa, B, H, N, causal, G):
    model, num_pairs, U = _schedule_model(B, H, N, causal, G)
    R = max(len(s) for s in model) + 1
    units = torch.full((G, R), -7, device="cuda", dtype=torch.int32)
    assert fa.fa_debug_fwd_schedule(B, H, N, causal, G, units, R) == 0
    got = units.cpu().numpy()
    seen = []
    for c in range(G):
        seq = list(got[c, :len(model[c])])
        assert seq == model[c]
        assert got[c, len(model[c])] == -1
        seen += seq
        if causal:  # longest first: the pair index never grows along a CTA's rounds
            pairs = [s % num_pairs for s in seq]
            assert all(a >= b for a, b in zip(pairs, pairs[1:]))
    assert sorted(seen) == list(range(U))  # every (head, query-tile pair) exactly once


def test_forward_and_backward_memory_is_linear_in_n(fa):
    """16 heads of 16k tokens: one head's N x N fp32 scores alone would be 1 GiB; the whole
    forward + backward must stay within inputs + outputs + the documented workspace."""
    B, N, H, d = 1, 16384, 16, 128
    t = synthetic.draw(B, N, H, d, 8200, "bf16", with_grad=True)
    q, k, v, dO = (t[n].cuda() for n in ("q", "k", "v", "dO"))
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    o, lse = fa.attention_forward(q, k, v, causal=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, dO, causal=True)
    torch.cuda.synchronize()
    extra = torch.cuda.max_memory_allocated() - base
    tensor = q.numel() * q.element_size()
    allowed = 4 * tensor + lse.numel() * 4 + fa.fa_bwd_workspace_bytes(B, H, N, d)
    assert extra <= allowed + (8 << 20), (extra, allowed)
    assert extra < (1 << 30)
