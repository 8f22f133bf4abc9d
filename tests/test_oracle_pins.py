"""Pins for the fp64 oracle: closed forms, invariants, brute force and a library special case.

Each test checks the oracle against something other than itself, chosen so that a
plausible slip (dropped scale, wrong mask direction, transposed operand, wrong sign in the
softmax Jacobian, log2 instead of ln) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.attention import backward_head, forward_head, scalar_loop_head

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- hand-worked fixture

@pytest.mark.parametrize("causal", [False, True])
def test_two_token_hand_example(causal):
    g = json.load(open(os.path.join(GOLDEN, "two_token_example.json")))
    inp = g["inputs"]
    col = lambda xs: np.array(xs, np.float64)[:, None]
    Q, K, V, dO = col(inp["q"]), col(inp["k"]), col(inp["v"]), col(inp["dO"])
    O, lse = forward_head(Q, K, V, inp["scale"], causal)
    dQ, dK, dV = backward_head(Q, K, V, dO, inp["scale"], causal)
    exp = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(O[:, 0], exp["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, exp["LSE"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dQ[:, 0], exp["dQ"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dK[:, 0], exp["dK"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dV[:, 0], exp["dV"], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_visible_values(causal):
    N, d = 37, 8
    scale = 0.3
    Q, V = rnd(1, N, d), rnd(2, N, d)
    k = rnd(3, d)
    K = np.tile(k, (N, 1))
    O, lse = forward_head(Q, K, V, scale, causal)
    for i in range(N):
        vis = i + 1 if causal else N
        np.testing.assert_allclose(O[i], V[:vis].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(lse[i] - (scale * Q[i] @ k + math.log(vis))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_dominant_logit_reproduces_that_value_row(causal):
    # Key j* = 3 outscores every other visible key by more than 800 in the logits, so
    # exp(-800) underflows to zero in fp64 and P is exactly one-hot.
    N, d = 12, 4
    Q = np.zeros((N, d))
    Q[:, 0] = 1.0
    K = rnd(5, N, d) * 0.1
    K[3, 0] = 1000.0
    V = rnd(6, N, d)
    O, lse = forward_head(Q, K, V, 1.0, causal)
    for i in (range(3, N) if causal else range(N)):
        np.testing.assert_array_equal(O[i], V[3])
        assert abs(lse[i] - Q[i] @ K[3]) < 1e-12
    if causal:  # rows before j* cannot see it
        assert not np.allclose(O[0], V[3])


def test_single_key_and_causal_row_zero():
    d, scale = 5, 0.7
    Q, K, V = rnd(7, 1, d), rnd(8, 1, d), rnd(9, 1, d)
    O, lse = forward_head(Q, K, V, scale, False)
    np.testing.assert_array_equal(O[0], V[0])
    assert abs(lse[0] - scale * Q[0] @ K[0]) < 1e-14
    Q, K, V = rnd(10, 9, d), rnd(11, 9, d), rnd(12, 9, d)
    O, lse = forward_head(Q, K, V, scale, True)
    np.testing.assert_array_equal(O[0], V[0])
    assert abs(lse[0] - scale * Q[0] @ K[0]) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    # With V = identity (N x N) the output row i is exactly row i of P.
    N, d = 20, 6
    Q, K = rnd(13, N, d), rnd(14, N, d)
    O, _ = forward_head(Q, K, np.eye(N), 0.5, causal)
    np.testing.assert_allclose(O.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (O >= 0).all()
    if causal:
        assert np.all(np.triu(O, 1) == 0.0)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance_with_large_logits(causal):
    N, d, scale = 33, 8, 1.0 / math.sqrt(8)
    Q, K, V = rnd(15, N, d), rnd(16, N, d), rnd(17, N, d)
    u = rnd(18, d) * 300.0  # logits of order 1e3: overflow-safe softmax required
    O0, l0 = forward_head(Q, K, V, scale, causal)
    O1, l1 = forward_head(Q, K + u, V, scale, causal)
    assert np.isfinite(O1).all()
    np.testing.assert_allclose(O1, O0, rtol=0, atol=1e-9)
    np.testing.assert_allclose(l1 - l0, scale * Q @ u, rtol=1e-10, atol=1e-9)


def test_noncausal_joint_permutation_of_keys_and_values():
    N, d = 29, 7
    Q, K, V = rnd(19, N, d), rnd(20, N, d), rnd(21, N, d)
    perm = np.random.default_rng(22).permutation(N)
    O0, l0 = forward_head(Q, K, V, 0.4, False)
    O1, l1 = forward_head(Q, K[perm], V[perm], 0.4, False)
    np.testing.assert_allclose(O1, O0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l0, rtol=0, atol=1e-13)


def test_causal_row_equals_noncausal_attention_over_its_prefix():
    N, d = 17, 5
    Q, K, V = rnd(23, N, d), rnd(24, N, d), rnd(25, N, d)
    Oc, lc = forward_head(Q, K, V, 0.6, True)
    for i in (0, 5, 16):
        Op, lp = forward_head(Q[i:i + 1], K[:i + 1], V[:i + 1], 0.6, False)
        np.testing.assert_allclose(Oc[i], Op[0], rtol=0, atol=1e-14)
        assert abs(lc[i] - lp[0]) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_rules(causal):
    N, d = 40, 8
    Q, K, V, dO = (rnd(s, N, d) for s in (26, 27, 28, 29))
    dQ, dK, dV = backward_head(Q, K, V, dO, 0.35, causal)
    # each row of P sums to one:  sum_j dV_j = sum_i dO_i
    np.testing.assert_allclose(dV.sum(axis=0), dO.sum(axis=0), rtol=0, atol=1e-12)
    # each row of dS sums to zero:  sum_j dK_j = 0
    np.testing.assert_allclose(dK.sum(axis=0), 0.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- online softmax claim

def _blockwise_rescaled(Q, K, V, scale, causal, bk):
    """Independent restatement of the rescaling argument: running max / sum per row,
    partial output rescaled whenever the max moves, normalised once at the end."""
    N = Q.shape[0]
    O = np.zeros((N, V.shape[1]))
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    for j0 in range(0, N, bk):
        S = scale * Q @ K[j0:j0 + bk].T
        if causal:
            S = np.where(np.arange(j0, j0 + S.shape[1])[None, :] <= np.arange(N)[:, None], S, -np.inf)
        m_new = np.maximum(m, S.max(axis=1))
        alpha = np.where(np.isfinite(m), np.exp(m - m_new), 0.0)
        Pt = np.exp(S - m_new[:, None])
        l = alpha * l + Pt.sum(axis=1)
        O = alpha[:, None] * O + Pt @ V[j0:j0 + bk]
        m = m_new
    return O / l[:, None], m + np.log(l)


def _blockwise_naive(Q, K, V, scale, bk):
    """Normalise each block on its own and add the pieces: NOT the same computation."""
    O = np.zeros((Q.shape[0], V.shape[1]))
    for j0 in range(0, Q.shape[0], bk):
        S = scale * Q @ K[j0:j0 + bk].T
        P = np.exp(S - S.max(axis=1, keepdims=True))
        O += (P / P.sum(axis=1, keepdims=True)) @ V[j0:j0 + bk]
    return O


@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_equals_whole_row_softmax(causal):
    N, d = 96, 16
    Q, K, V = rnd(30, N, d), rnd(31, N, d), rnd(32, N, d)
    O, lse = forward_head(Q, K, V, 0.25, causal)
    Ot, lt = _blockwise_rescaled(Q, K, V, 0.25, causal, 16)
    np.testing.assert_allclose(Ot, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lt, lse, rtol=0, atol=1e-13)
    if not causal:
        assert np.abs(_blockwise_naive(Q, K, V, 0.25, 16) - O).max() > 1e-2


# ---------------------------------------------------------------- brute force / library

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (3, 4), (8, 1), (8, 4)])
def test_gradients_match_central_finite_differences(N, d, causal):
    Q, K, V, dO = (rnd(40 + s, N, d) for s in range(4))
    scale, h = 0.8, 1e-6
    dQ, dK, dV = backward_head(Q, K, V, dO, scale, causal)

    def loss(Q_, K_, V_):
        return float((forward_head(Q_, K_, V_, scale, causal)[0] * dO).sum())

    for which, grad in ((0, dQ), (1, dK), (2, dV)):
        fd = np.zeros((N, d))
        for i in range(N):
            for t in range(d):
                args_p = [Q.copy(), K.copy(), V.copy()]
                args_m = [Q.copy(), K.copy(), V.copy()]
                args_p[which][i, t] += h
                args_m[which][i, t] -= h
                fd[i, t] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.abs(fd - grad).max() / max(1.0, np.abs(grad).max())
        assert err < 1e-7, (which, err)


@pytest.mark.parametrize("causal", [False, True])
def test_scalar_loop_twin_agrees(causal):
    N, d = 11, 3
    Q, K, V, dO = (rnd(50 + s, N, d) for s in range(4))
    O, lse = forward_head(Q, K, V, 0.9, causal)
    dQ, dK, dV = backward_head(Q, K, V, dO, 0.9, causal)
    Os, ls, dQs, dKs, dVs = scalar_loop_head(Q.tolist(), K.tolist(), V.tolist(), dO.tolist(), 0.9, causal)
    for a, b in ((O, Os), (lse, ls), (dQ, dQs), (dK, dKs), (dV, dVs)):
        np.testing.assert_allclose(a, np.array(b), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,d", [(2, 5, 3, 4), (1, 130, 2, 16)])
def test_matches_torch_sdpa_fp64_with_autograd(B, N, H, d, causal):
    g = torch.Generator().manual_seed(60)
    q, k, v, dO = (torch.randn(B, N, H, d, generator=g, dtype=torch.float64) for _ in range(4))
    scale = 1.0 / math.sqrt(d)
    qt, kt, vt = (x.transpose(1, 2).clone().requires_grad_(True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    out.backward(dO.transpose(1, 2))
    O, lse = oracle.forward(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    dQ, dK, dV = oracle.backward(q.numpy(), k.numpy(), v.numpy(), dO.numpy(), scale, causal)
    np.testing.assert_allclose(O, out.detach().transpose(1, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dQ, qt.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK, kt.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, vt.grad.transpose(1, 2).numpy(), rtol=0, atol=1e-12)
    # LSE against torch.logsumexp of the explicitly masked logits
    S = scale * torch.einsum("bihd,bjhd->bhij", q, k)
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(S, dim=-1).numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- sampled-row helpers

def test_row_sampled_helpers_match_whole_head():
    N, d, scale = 300, 8, 0.3
    Q, K, V, dO = (rnd(70 + s, N, d) for s in range(4))
    rows = np.array([0, 1, 127, 128, 299])
    for causal in (False, True):
        O, lse = forward_head(Q, K, V, scale, causal, slab=64)
        dQ, dK, dV = backward_head(Q, K, V, dO, scale, causal, slab=64)
        Or, lr = oracle.forward_rows(Q, K, V, scale, causal, rows)
        np.testing.assert_allclose(Or, O[rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lr, lse[rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(oracle.dq_rows(Q, K, V, dO, scale, causal, rows), dQ[rows], rtol=0, atol=1e-12)
    dQ, dK, dV = backward_head(Q, K, V, dO, scale, True)
    tk, tv = oracle.kv_grad_tail(Q, K, V, dO, scale, 250)
    np.testing.assert_allclose(tk, dK[250:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(tv, dV[250:], rtol=0, atol=1e-12)


def test_slab_size_does_not_change_results():
    N, d = 200, 4
    Q, K, V, dO = (rnd(80 + s, N, d) for s in range(4))
    for causal in (False, True):
        a = forward_head(Q, K, V, 0.5, causal, slab=N)
        b = forward_head(Q, K, V, 0.5, causal, slab=7)
        np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-14)
        ga = backward_head(Q, K, V, dO, 0.5, causal, slab=N)
        gb = backward_head(Q, K, V, dO, 0.5, causal, slab=7)
        for x, y in zip(ga, gb):
            np.testing.assert_allclose(x, y, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- fewer queries than keys

def test_single_last_query_sees_every_key():
    # Decoding one token: with the causal mask aligned to the last key, the only query sees
    # all keys, i.e. it equals the non-causal result.
    Nk, d = 57, 6
    Q, K, V = rnd(90, 1, d), rnd(91, Nk, d), rnd(92, Nk, d)
    Oc, lc = forward_head(Q, K, V, 0.4, True)
    On, ln = forward_head(Q, K, V, 0.4, False)
    np.testing.assert_allclose(Oc, On, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lc, ln, rtol=0, atol=1e-14)


def test_bottom_right_causal_row_equals_noncausal_over_its_visible_keys():
    Nq, Nk, d = 9, 40, 5
    Q, K, V = rnd(93, Nq, d), rnd(94, Nk, d), rnd(95, Nk, d)
    O, l = forward_head(Q, K, V, 0.7, True)
    for i in range(Nq):
        vis = i + Nk - Nq + 1
        Op, lp = forward_head(Q[i:i + 1], K[:vis], V[:vis], 0.7, False)
        np.testing.assert_allclose(O[i], Op[0], rtol=0, atol=1e-14)
        assert abs(l[i] - lp[0]) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_key_split_merge_rule(causal):
    # Splitting the keys, attending to each part and merging with the logsumexp rule
    # (O = sum_s exp(L_s - L) O_s, L = log sum_s exp L_s) reproduces attention over all keys.
    Nq, Nk, d = 7, 61, 8
    Q, K, V = rnd(96, Nq, d), rnd(97, Nk, d), rnd(98, Nk, d)
    O, L = forward_head(Q, K, V, 0.3, causal)
    off = Nk - Nq
    parts = []
    for a, b in [(0, 20), (20, 47), (47, Nk)]:
        S = 0.3 * Q @ K[a:b].T
        if causal:
            S = np.where(np.arange(a, b)[None, :] <= np.arange(Nq)[:, None] + off, S, -np.inf)
        m = S.max(axis=1)
        E = np.exp(S - m[:, None])
        parts.append((E @ V[a:b] / E.sum(1)[:, None], m + np.log(E.sum(1))))
    Ls = np.stack([p[1] for p in parts])
    Lm = np.log(np.exp(Ls - Ls.max(0)).sum(0)) + Ls.max(0)
    Om = sum(np.exp(p[1] - Lm)[:, None] * p[0] for p in parts)
    np.testing.assert_allclose(Om, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lm, L, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- block-sparse reference

def test_block_sparse_all_ones_is_dense():
    N, d = 300, 8
    Q, K, V = rnd(100, N, d), rnd(101, N, d), rnd(102, N, d)
    m = np.ones((3, 3), np.uint8)
    for causal in (False, True):
        O, L = oracle.forward_head_block_sparse(Q, K, V, 0.3, causal, m)
        Od, Ld = forward_head(Q, K, V, 0.3, causal)
        np.testing.assert_allclose(O, Od, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-13)


def test_block_diagonal_mask_is_independent_blocks():
    # Only diagonal blocks: each 128-row block attends to itself alone.
    N, d = 300, 8
    Q, K, V = rnd(103, N, d), rnd(104, N, d), rnd(105, N, d)
    O, L = oracle.forward_head_block_sparse(Q, K, V, 0.3, False, np.eye(3, dtype=np.uint8))
    for a in range(0, N, 128):
        b = min(N, a + 128)
        Ob, Lb = forward_head(Q[a:b], K[a:b], V[a:b], 0.3, False)
        np.testing.assert_allclose(O[a:b], Ob, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L[a:b], Lb, rtol=0, atol=1e-13)


def test_block_sparse_empty_rows_and_brute_force():
    N, d = 260, 4
    Q, K, V = rnd(106, N, d), rnd(107, N, d), rnd(108, N, d)
    m = np.array([[0, 1, 0], [0, 0, 0], [1, 0, 1]], np.uint8)
    O, L = oracle.forward_head_block_sparse(Q, K, V, 0.5, False, m)
    assert np.all(O[128:256] == 0) and np.all(np.isneginf(L[128:256]))   # block row 1 is empty
    for i in (0, 100, 256, 259):                                           # brute force rows
        keys = [j for j in range(N) if m[i // 128, j // 128]]
        s = np.array([0.5 * Q[i] @ K[j] for j in keys])
        p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
        np.testing.assert_allclose(O[i], p @ V[keys], rtol=0, atol=1e-13)
        assert abs(L[i] - (s.max() + np.log(np.exp(s - s.max()).sum()))) < 1e-12
    # causal: block (0,1) lies above the diagonal, so rows 0..127 see nothing
    Oc, Lc = oracle.forward_head_block_sparse(Q, K, V, 0.5, True, m)
    assert np.all(Oc[:128] == 0) and np.all(np.isneginf(Lc[:128]))


def test_block_sparse_rows_all_ones_equal_dense_rows():
    # With every block active the sampled-rows form is dense attention at those rows.
    N, d = 300, 8
    Q, K, V = rnd(109, N, d), rnd(110, N, d), rnd(111, N, d)
    rows = np.array([0, 1, 127, 128, 200, 299])
    for causal in (False, True):
        O, L = oracle.forward_rows_block_sparse(Q, K, V, 0.3, causal, np.ones((3, 3), np.uint8), rows)
        Od, Ld = forward_head(Q, K, V, 0.3, causal)
        np.testing.assert_allclose(O, Od[rows], rtol=0, atol=1e-13)
        np.testing.assert_allclose(L, Ld[rows], rtol=0, atol=1e-13)


def test_block_sparse_rows_one_block_is_dense_attention_over_that_block():
    # Block row r sees only key block p(r): its rows are non-causal dense attention over
    # K, V rows [128 p, 128 p + 128) (the last block is ragged); block row 1 sees nothing.
    N, d = 300, 8
    Q, K, V = rnd(112, N, d), rnd(113, N, d), rnd(114, N, d)
    m = np.zeros((3, 3), np.uint8)
    m[0, 2] = 1
    m[2, 0] = 1
    rows = np.array([0, 50, 127, 128, 255, 256, 299])
    O, L = oracle.forward_rows_block_sparse(Q, K, V, 0.7, False, m, rows)
    for n, i in enumerate(rows):
        if i // 128 == 1:
            assert np.all(O[n] == 0) and np.isneginf(L[n])
            continue
        a = 256 if i // 128 == 0 else 0
        Ob, Lb = forward_head(Q[i:i + 1], K[a:a + 128], V[a:a + 128], 0.7, False)
        np.testing.assert_allclose(O[n], Ob[0], rtol=0, atol=1e-13)
        assert abs(L[n] - Lb[0]) < 1e-12
    # causal: block (0, 2) lies above the diagonal, so block row 0 sees nothing either
    Oc, Lc = oracle.forward_rows_block_sparse(Q, K, V, 0.7, True, m, rows[:3])
    assert np.all(Oc == 0) and np.all(np.isneginf(Lc))


def test_block_sparse_rows_match_the_whole_head_form():
    N, d = 390, 4
    Q, K, V = rnd(115, N, d), rnd(116, N, d), rnd(117, N, d)
    m = (np.random.default_rng(118).random((4, 4)) < 0.5).astype(np.uint8)
    rows = np.arange(0, N, 7)
    for causal in (False, True):
        O, L = oracle.forward_rows_block_sparse(Q, K, V, 0.4, causal, m, rows)
        Oh, Lh = oracle.forward_head_block_sparse(Q, K, V, 0.4, causal, m)
        np.testing.assert_allclose(O, Oh[rows], rtol=0, atol=1e-13)
        assert np.array_equal(np.isneginf(L), np.isneginf(Lh[rows]))
        live = np.isfinite(L)
        np.testing.assert_allclose(L[live], Lh[rows][live], rtol=0, atol=1e-12)
