"""GPU parity of the backward pass against the fp64 oracle (through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests._helpers import GRAD_REL_L2, cuda, grad_err, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    assert torch.cuda.is_available()
    return mod


def _workspace(fa, q):
    B, N, H, d = q.shape
    return torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), device=q.device, dtype=torch.uint8)


def _run(fa, t, causal, scale):
    q, k, v, dO = cuda(t, ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    ws = _workspace(fa, q)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, dO, causal=causal, scale=scale,
                                       workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0      # the forward's (library-owned) word
    assert fa.fa_read_device_status(ws) == 0    # the backward call's own word
    return dq, dk, dv


@pytest.mark.parametrize("B,N,H,d", [
    (1, 128, 2, 64), (1, 128, 2, 128),     # one tile
    (2, 1000, 3, 128), (3, 300, 2, 64),    # several tiles + ragged tail
    (1, 1, 1, 64), (1, 129, 1, 128), (1, 640, 4, 64), (1, 200, 2, 128),
])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_parity(fa, B, N, H, d, causal):
    t = synthetic.draw(B, N, H, d, 2000 + N + d, "bf16", with_grad=True)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = _run(fa, t, causal, scale)
    refs = oracle.backward(*(synthetic.to_f64(t[n]) for n in ("q", "k", "v", "dO")), scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        assert grad_err(to_np(g), r) <= GRAD_REL_L2, (name, grad_err(to_np(g), r))


def test_backward_repeatable_within_tolerance(fa):
    t = synthetic.draw(2, 512, 4, 128, 17, "bf16", with_grad=True)
    a = _run(fa, t, True, 1 / math.sqrt(128))
    b = _run(fa, t, True, 1 / math.sqrt(128))
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # dK, dV: fixed order
    assert rel_l2(to_np(a[0]), to_np(b[0])) < 1e-3             # dQ: fp32 atomics


def _sampled_checks(fa, w, n_rows, tail):
    t = synthetic.draw_workload(w, with_grad=True)
    dq, dk, dv = _run(fa, t, w.causal, w.scale)
    rng = np.random.default_rng(w.seed)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N - 1], rng.integers(0, w.N, n_rows)]))
    for b, h in [(0, 0), (w.B - 1, w.H - 1)]:
        Q, K, V, dO = (synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v", "dO"))
        ref = oracle.dq_rows(Q, K, V, dO, w.scale, w.causal, rows)
        assert rel_l2(to_np(dq[b, rows, h]), ref) <= GRAD_REL_L2
        if w.causal:
            tk, tv = oracle.kv_grad_tail(Q, K, V, dO, w.scale, w.N - tail)
            assert rel_l2(to_np(dk[b, w.N - tail:, h]), tk) <= GRAD_REL_L2
            assert rel_l2(to_np(dv[b, w.N - tail:, h]), tv) <= GRAD_REL_L2
        # properties that hold at any size: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0
        sdv = to_np(dv[b, :, h]).sum(0)
        assert np.abs(sdv - dO.sum(0)).max() <= 2e-3 * np.abs(to_np(dv[b, :, h])).sum(0).max()
        sdk = to_np(dk[b, :, h]).sum(0)
        assert np.abs(sdk).max() <= 2e-3 * np.abs(to_np(dk[b, :, h])).sum(0).max()


@pytest.mark.parametrize("N", [4096, 16384])
def test_backward_full_size_sampled(fa, N):
    _sampled_checks(fa, synthetic.fwdbwd(N), 59, 64)


def test_backward_long_context_sampled(fa):
    _sampled_checks(fa, synthetic.long_context(), 27, 64)


def test_backward_full_head_at_4k(fa):
    w = synthetic.fwdbwd(4096)
    t = synthetic.draw_workload(w, with_grad=True)
    dq, dk, dv = _run(fa, t, True, w.scale)
    b, h = 1, 5
    refs = oracle.backward_head(*(synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v", "dO")),
                                w.scale, True)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        assert rel_l2(to_np(g[b, :, h]), r) <= GRAD_REL_L2, name


# ------------------------------------------------------------------ deterministic variant

@pytest.mark.parametrize("B,N,H,d", [(2, 1000, 3, 128), (3, 300, 2, 64), (1, 1, 1, 64),
                                     (1, 129, 1, 128), (1, 640, 4, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_deterministic_backward_parity(fa, B, N, H, d, causal):
    t = synthetic.draw(B, N, H, d, 3000 + N + d, "bf16", with_grad=True)
    scale = 1.0 / math.sqrt(d)
    q, k, v, dO = cuda(t, ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    ws = _workspace(fa, q)
    got = fa.attention_backward(q, k, v, o, lse, dO, causal=causal, scale=scale, deterministic=True,
                                workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    assert fa.fa_read_device_status(ws) == 0
    refs = oracle.backward(*(synthetic.to_f64(t[n]) for n in ("q", "k", "v", "dO")), scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), got, refs):
        assert grad_err(to_np(g), r) <= GRAD_REL_L2, (name, grad_err(to_np(g), r))


@pytest.mark.parametrize("w", [synthetic.fwdbwd(4096), synthetic.long_context()], ids=lambda w: w.label())
def test_deterministic_backward_is_bitwise_repeatable_at_full_size(fa, w):
    t = synthetic.draw_workload(w, with_grad=True)
    q, k, v, dO = cuda(t, ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    a = fa.attention_backward(q, k, v, o, lse, dO, causal=w.causal, scale=w.scale, deterministic=True)
    b = fa.attention_backward(q, k, v, o, lse, dO, causal=w.causal, scale=w.scale, deterministic=True)
    c = fa.attention_backward(q, k, v, o, lse, dO, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # and it agrees with the atomic-reduction variant within the gradient tolerance
    for x, y in zip(a, c):
        assert rel_l2(to_np(x), to_np(y)) <= 2e-3
    rng = np.random.default_rng(w.seed)
    rows = np.unique(rng.integers(0, w.N, 32))
    Q, K, V, DO = (synthetic.to_f64(t[n][0, :, 0]) for n in ("q", "k", "v", "dO"))
    ref = oracle.dq_rows(Q, K, V, DO, w.scale, w.causal, rows)
    assert rel_l2(to_np(a[0][0, rows, 0]), ref) <= GRAD_REL_L2


# ------------------------------------------------------------------ per-call status word

def test_backward_status_word_is_per_call(fa):
    # Two backward calls run on two streams, each with its own workspace, so each has its
    # own status word (the workspace's first int).  A bounded wait that runs out on the
    # first stream, recorded into the first call's word, shows up there only: the second
    # call's word and the library-owned word stay clear.
    B, N, H, d = 1, 512, 2, 128
    scale = 1.0 / math.sqrt(d)
    t = synthetic.draw(B, N, H, d, 41, "bf16", with_grad=True)
    q, k, v, dO = cuda(t, ("q", "k", "v", "dO"))
    o, lse = fa.attention_forward(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == fa.FA_OK
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    wss = (_workspace(fa, q), _workspace(fa, q))
    outs = [[torch.full_like(q, float("nan")) for _ in range(3)] for _ in range(2)]
    for s, ws, (dq, dk, dv) in zip(streams, wss, outs):
        rc = fa.fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, True, scale, ws, ws.numel(),
                       stream=s)
        assert rc == fa.FA_OK, fa.status_string(rc)
    assert fa.fa_debug_wait_timeout(20_000_000, wss[0], stream=streams[0]) == fa.FA_OK
    assert fa.fa_read_device_status(wss[0], stream=streams[0]) == fa.FA_ERR_TIMEOUT
    assert fa.fa_read_device_status(wss[1], stream=streams[1]) == fa.FA_OK
    assert fa.fa_read_device_status() == fa.FA_OK
    assert fa.fa_read_device_status(wss[0], stream=streams[0]) == fa.FA_OK  # read clears it
    # Both calls computed the same gradients (dK, dV bit for bit: fixed accumulation order).
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][2], outs[1][2])
    assert rel_l2(to_np(outs[0][0]), to_np(outs[1][0])) <= 1e-3
