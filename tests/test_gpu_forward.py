"""GPU parity of the forward kernels against the fp64 oracle (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests._helpers import (F32_MAX_ABS, LSE_MAX_ABS, O_MAX_ABS, O_REL_L2, cuda, max_abs, rel_l2,
                            to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    assert torch.cuda.is_available()
    return mod


# ------------------------------------------------------------------ primitive self-tests

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("n,k", [(128, 64), (128, 128), (64, 128), (64, 64)])
def test_umma_tile(fa, mode, n, k):
    g = torch.Generator().manual_seed(100 + 10 * mode + n + k)
    A = torch.randn(128, k, generator=g).to(torch.bfloat16)
    Bm = torch.randn(n, k, generator=g).to(torch.bfloat16) if mode == 0 else \
        torch.randn(k, n, generator=g).to(torch.bfloat16)
    ref = A.double() @ (Bm.double().T if mode == 0 else Bm.double())
    dA, dB = A.cuda(), Bm.cuda()
    C = torch.full((128, n), float("nan"), device="cuda")
    assert fa.fa_debug_umma_tile(dA, dB, C, n, k, mode) == 0
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    np.testing.assert_allclose(C.double().cpu().numpy(), ref.numpy(), atol=2e-3, rtol=1e-5)


def test_software_exp2_within_its_error_bound(fa):
    # Range the kernels feed it: logits minus a running max, i.e. <= 8 (stale max) and down
    # to the clamp at -125; plus the exact integers where the reduction is trivial.
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_003), np.arange(-125, 9, dtype=np.float64),
                        np.random.default_rng(0).uniform(-30, 8, 100_000)]).astype(np.float32)
    dx = torch.from_numpy(x).cuda()
    yp, yh = torch.empty_like(dx), torch.empty_like(dx)
    assert fa.fa_debug_exp2(dx, yp, yh, x.size) == 0
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    rel_poly = np.abs(yp.cpu().numpy().astype(np.float64) / exact - 1.0)
    rel_hw = np.abs(yh.cpu().numpy().astype(np.float64) / exact - 1.0)
    # minimax bound of the polynomial (7.5e-5) plus fp32 rounding of the reduction
    assert rel_poly.max() < 1e-4, rel_poly.max()
    # the hardware exp2 is the reference scale for what the kernels accept elsewhere
    assert rel_hw.max() < 1e-5
    # bf16 (the precision P is stored in) cannot tell them apart most of the time
    assert np.mean(rel_poly < 2.0 ** -9) == 1.0


def test_bounded_wait_times_out_and_reports(fa):
    assert fa.fa_debug_wait_timeout(50_000_000) == 0
    assert fa.fa_read_device_status() == fa.FA_ERR_TIMEOUT
    # The context is still usable and the word was cleared.
    assert fa.fa_read_device_status() == fa.FA_OK
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0


# ------------------------------------------------------------------ fp32 path

def _f32_case(fa, B, N, H, d, causal, seed):
    t = synthetic.draw(B, N, H, d, seed, "f32")
    q, k, v = cuda(t, ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    O_ref, L_ref = oracle.forward(*(synthetic.to_f64(t[n]) for n in ("q", "k", "v")), scale, causal)
    return to_np(o), to_np(lse), O_ref, L_ref


@pytest.mark.parametrize("causal", [False, True])
def test_f32_tiny_config(fa, causal):
    w = synthetic.tiny_f32(causal)
    O, L, O_ref, L_ref = _f32_case(fa, w.B, w.N, w.H, w.d, causal, w.seed)
    assert max_abs(O, O_ref) <= F32_MAX_ABS
    assert max_abs(L, L_ref) <= F32_MAX_ABS


@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 64), (2, 37, 3, 32), (1, 200, 2, 128), (1, 65, 1, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_f32_ragged(fa, B, N, H, d, causal):
    O, L, O_ref, L_ref = _f32_case(fa, B, N, H, d, causal, 11)
    assert max_abs(O, O_ref) <= F32_MAX_ABS
    assert max_abs(L, L_ref) <= F32_MAX_ABS


# ------------------------------------------------------------------ bf16 tensor-core path

def _bf16_case(fa, B, N, H, d, causal, seed):
    t = synthetic.draw(B, N, H, d, seed, "bf16")
    q, k, v = cuda(t, ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    O_ref, L_ref = oracle.forward(*(synthetic.to_f64(t[n]) for n in ("q", "k", "v")), scale, causal)
    return to_np(o), to_np(lse), O_ref, L_ref


@pytest.mark.parametrize("B,N,H,d", [
    (1, 128, 2, 64), (1, 128, 2, 128),      # one tile
    (2, 1000, 3, 128), (3, 300, 2, 64),    # several tiles + ragged tail
    (1, 1, 1, 64), (1, 127, 2, 128), (1, 129, 1, 64), (1, 640, 4, 64),
])
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_forward_parity(fa, B, N, H, d, causal):
    O, L, O_ref, L_ref = _bf16_case(fa, B, N, H, d, causal, 1000 + N + d)
    assert max_abs(O, O_ref) <= O_MAX_ABS, max_abs(O, O_ref)
    assert rel_l2(O, O_ref) <= O_REL_L2, rel_l2(O, O_ref)
    assert max_abs(L, L_ref) <= LSE_MAX_ABS, max_abs(L, L_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_forward_is_deterministic(fa, d):
    t = synthetic.draw(2, 1024, 4, d, 5, "bf16")
    q, k, v = cuda(t, ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    o2, l2 = fa.attention_forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bf16_forward_gpu_invariants(fa):
    # identical keys -> O_i is the mean of the visible values; causal row 0 is exactly v_0
    B, N, H, d = 1, 384, 2, 128
    t = synthetic.draw(B, N, H, d, 9, "bf16")
    t["k"] = t["k"][:, :1].expand(B, N, H, d).contiguous()
    q, k, v = cuda(t, ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    V = synthetic.to_f64(t["v"])
    O = to_np(o)
    means = np.cumsum(V, axis=1) / np.arange(1, N + 1)[None, :, None, None]
    assert max_abs(O, means) <= O_MAX_ABS
    np.testing.assert_array_equal(O[:, 0], V[:, 0])


# Every (head dim, causal) instantiation of the dense forward runs here at a size where each
# persistent CTA takes many units (B*H*ceil(N/256) units on at most 148 CTAs), so the hand-over
# of the O columns and of the K/V ring from one unit to the next is checked against the oracle:
# d=64 non-causal 4k (1024 units), d=64 causal 16k (2048) and 512 (2048 one-pair units),
# d=128 non-causal 16k (1024) and 512 (1024), d=128 causal 16k (1024) and 64k (256).
FULL_SIZE = [synthetic.fwd_sweep(64, 4096, False), synthetic.fwd_sweep(64, 16384, True),
             synthetic.fwd_sweep(64, 512, True), synthetic.fwd_sweep(128, 16384, False),
             synthetic.fwd_sweep(128, 512, False), synthetic.fwd_sweep(128, 16384, True),
             synthetic.long_context()]


@pytest.mark.parametrize("w", FULL_SIZE, ids=lambda w: w.label())
def test_bf16_forward_full_size_sampled_rows(fa, w):
    t = synthetic.draw_workload(w, with_grad=False)
    q, k, v = cuda(t, ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    rng = np.random.default_rng(w.seed)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, w.N - 1], rng.integers(0, w.N, 57)]))
    # First and last head, plus two from the middle of the unit order (other batch entries
    # and heads land on other CTAs and rounds of the persistent schedule).
    heads = sorted({(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 3), ((w.B - 1) // 3, w.H - 2)})
    for b, h in heads:
        Q, K, V = (synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v"))
        O_ref, L_ref = oracle.forward_rows(Q, K, V, w.scale, w.causal, rows)
        O = to_np(o[b, rows, h])
        L = to_np(lse[b, h, rows])
        assert max_abs(O, O_ref) <= O_MAX_ABS
        assert rel_l2(O, O_ref) <= O_REL_L2
        assert max_abs(L, L_ref) <= LSE_MAX_ABS
