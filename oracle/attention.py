"""fp64 CPU oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the library's product path may import, call or
execute this module: only the test-suite, the package's smoke check and the bench's
CPU-baseline / reference leg use it.  It shares no code with the CUDA path.

What it computes (the plain definition, written out):

* Forward, from the formula ``Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V`` and the
  three-step "standard" evaluation of it in "Flash Attention 2で打破するローカルLLMの
  「メモリの壁」" (section "標準的なAttention機構のメモリ挙動"): materialise
  S = scale * Q K^T, then P = softmax(S) row by row, then O = P V.  The scale is an
  explicit argument (the pages' 1/sqrt(d_k) is what the workloads pass).
* The causal mask: key j is visible to query i iff j <= i (square problems only).
* The per-row logsumexp LSE_i = m_i + ln(sum_j exp(S_ij - m_i)), natural log, over the
  visible keys, including the scale.  The pages do not define it; it is the statistic
  that lets the backward pass rebuild P ("タイリング（Tiling）と再計算（Recomputation）の
  仕組み" on the same page).
* Backward: the textbook softmax Jacobian applied to the materialised P:
  dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij;  dS = P o (dP - D);
  dQ = scale dS K;  dK = scale dS^T Q.
  D is formed from P and dP here on purpose; it shares no shortcut with the GPU
  kernels' rowsum(dO o O) (equal in exact arithmetic).

Precision: float64 throughout.  Inputs are whatever float arrays the caller passes
(the bf16 / fp32 test tensors upcast exactly).

Blocking: for long sequences a head is processed in slabs of query rows.  Every row
still forms its full row of S and its full two-pass softmax; slabs only bound the memory
held at once, and dK / dV sum the slabs' contributions (fp64 rounding order only).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

DEFAULT_SLAB = 1024


def _mask_rows(S: np.ndarray, rows: np.ndarray, causal: bool, offset: int = 0) -> np.ndarray:
    """Set S[r, j] = -inf where key j is not visible to query rows[r]: under the causal mask
    query i sees keys j <= i + offset (offset = Nk - Nq aligns the last query with the last
    key when there are fewer queries than keys; 0 for square problems)."""
    if causal:
        cols = np.arange(S.shape[1])
        S = np.where(cols[None, :] <= rows[:, None] + offset, S, -np.inf)
    return S


def _softmax_rows(S: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Explicit two-pass row softmax of a materialised score block.

    Returns P (same shape as S) and the natural-log logsumexp of each row.
    """
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    P = E / l[:, None]
    return P, m + np.log(l)


def forward_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, causal: bool,
                 slab: int = DEFAULT_SLAB) -> Tuple[np.ndarray, np.ndarray]:
    """One (batch, head): Q is [Nq, d], K and V are [Nk, d] (Nq = Nk for the square problems
    of the main path; Nq <= Nk for decoding, where the causal mask is aligned to the last
    key: query i sees keys j <= i + Nk - Nq).  Returns O [Nq, d] and LSE [Nq]."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    offset = K.shape[0] - N
    O = np.empty((N, V.shape[1]), np.float64)
    lse = np.empty(N, np.float64)
    for r0 in range(0, N, slab):
        rows = np.arange(r0, min(N, r0 + slab))
        S = scale * (Q[rows] @ K.T)              # step 1: S = scale * Q K^T
        S = _mask_rows(S, rows, causal, offset)
        P, lse[rows] = _softmax_rows(S)          # step 2: P = softmax(S)
        O[rows] = P @ V                          # step 3: O = P V
    return O, lse


def backward_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray, scale: float,
                  causal: bool, slab: int = DEFAULT_SLAB):
    """Gradients of sum(O o dO) for one (batch, head).  Returns dQ, dK, dV ([N, d] each)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dO = np.asarray(dO, np.float64)
    N = Q.shape[0]
    dQ = np.empty_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for r0 in range(0, N, slab):
        rows = np.arange(r0, min(N, r0 + slab))
        S = _mask_rows(scale * (Q[rows] @ K.T), rows, causal)
        P, _ = _softmax_rows(S)
        dV += P.T @ dO[rows]
        dP = dO[rows] @ V.T
        D = (P * dP).sum(axis=1)
        dS = P * (dP - D[:, None])
        dQ[rows] = scale * (dS @ K)
        dK += scale * (dS.T @ Q[rows])
    return dQ, dK, dV


def _heads(x: np.ndarray):
    """Iterate (b, h, x[b, :, h, :]) over a [B, N, H, d] array."""
    B, _, H, _ = x.shape
    for b in range(B):
        for h in range(H):
            yield b, h


def forward(q, k, v, scale: float, causal: bool, heads: Optional[Sequence[Tuple[int, int]]] = None):
    """q [B, Nq, H, d], k and v [B, Nk, H, d].  Returns O [B, Nq, H, d] and LSE [B, H, Nq]
    (float64).  ``heads`` restricts the work to the listed (b, h) pairs; other entries stay
    NaN.
    """
    q = np.asarray(q, np.float64)
    B, N, H, _ = q.shape
    O = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    lse = np.full((B, H, N), np.nan)
    for b, h in (heads if heads is not None else _heads(q)):
        O[b, :, h, :], lse[b, h] = forward_head(q[b, :, h], k[b, :, h], v[b, :, h], scale, causal)
    return O, lse


def backward(q, k, v, dO, scale: float, causal: bool,
             heads: Optional[Sequence[Tuple[int, int]]] = None):
    """[B, N, H, d] inputs.  Returns dQ, dK, dV ([B, N, H, d] float64)."""
    q = np.asarray(q, np.float64)
    dQ = np.full(q.shape, np.nan)
    dK = np.full(q.shape, np.nan)
    dV = np.full(np.shape(v), np.nan)
    for b, h in (heads if heads is not None else _heads(q)):
        dQ[b, :, h], dK[b, :, h], dV[b, :, h] = backward_head(
            q[b, :, h], k[b, :, h], v[b, :, h], dO[b, :, h], scale, causal)
    return dQ, dK, dV


# ----------------------------------------------------------------------------------------
# Row-sampled evaluation for problems too large to run whole on the CPU.  Each function is
# the same definition restricted to the requested rows; nothing is approximated.
# ----------------------------------------------------------------------------------------

def forward_rows(Q, K, V, scale: float, causal: bool, rows) -> Tuple[np.ndarray, np.ndarray]:
    """O and LSE of the selected query rows of one head ([N, d] inputs)."""
    rows = np.asarray(rows)
    Q = np.asarray(Q, np.float64)
    S = _mask_rows(scale * (Q[rows] @ np.asarray(K, np.float64).T), rows, causal)
    P, lse = _softmax_rows(S)
    return P @ np.asarray(V, np.float64), lse


def dq_rows(Q, K, V, dO, scale: float, causal: bool, rows) -> np.ndarray:
    """dQ of the selected query rows of one head: row i needs only row i of P and dP."""
    rows = np.asarray(rows)
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    S = _mask_rows(scale * (Q[rows] @ K.T), rows, causal)
    P, _ = _softmax_rows(S)
    dP = np.asarray(dO, np.float64)[rows] @ np.asarray(V, np.float64).T
    D = (P * dP).sum(axis=1)
    return scale * ((P * (dP - D[:, None])) @ K)


def kv_grad_tail(Q, K, V, dO, scale: float, j0: int) -> Tuple[np.ndarray, np.ndarray]:
    """Causal only: dK, dV of keys j >= j0 of one head.

    Under the causal mask key j is seen by queries i >= j alone, so the keys of the
    sequence tail need only the query rows i >= j0 (each a full row of P and dP).
    """
    Q = np.asarray(Q, np.float64)
    N = Q.shape[0]
    rows = np.arange(j0, N)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    dOr = np.asarray(dO, np.float64)[rows]
    S = _mask_rows(scale * (Q[rows] @ K.T), rows, True)
    P, _ = _softmax_rows(S)
    dP = dOr @ V.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dK = scale * (dS[:, j0:].T @ Q[rows])
    dV = P[:, j0:].T @ dOr
    return dK, dV


# ----------------------------------------------------------------------------------------
# Scalar-loop twin: the same definition as nested Python loops over scalars (math.exp,
# math.log).  Used only to cross-check the array version on tiny problems (N <= 16).
# ----------------------------------------------------------------------------------------

def scalar_loop_head(Q, K, V, dO, scale: float, causal: bool):
    """Returns O, LSE, dQ, dK, dV as nested lists for one head."""
    N, d = len(Q), len(Q[0])
    dv = len(V[0])
    O = [[0.0] * dv for _ in range(N)]
    LSE = [0.0] * N
    P = [[0.0] * N for _ in range(N)]
    for i in range(N):
        vis = [j for j in range(N) if (not causal) or j <= i]
        s = {j: scale * sum(Q[i][t] * K[j][t] for t in range(d)) for j in vis}
        m = max(s.values())
        e = {j: math.exp(s[j] - m) for j in vis}
        l = sum(e.values())
        for j in vis:
            P[i][j] = e[j] / l
        LSE[i] = m + math.log(l)
        for c in range(dv):
            O[i][c] = sum(P[i][j] * V[j][c] for j in vis)
    dQ = [[0.0] * d for _ in range(N)]
    dK = [[0.0] * d for _ in range(N)]
    dV = [[0.0] * dv for _ in range(N)]
    if dO is None:
        return O, LSE, None, None, None
    for i in range(N):
        dP = [sum(dO[i][c] * V[j][c] for c in range(dv)) for j in range(N)]
        D = sum(P[i][j] * dP[j] for j in range(N))
        for j in range(N):
            dS = P[i][j] * (dP[j] - D)
            for c in range(dv):
                dV[j][c] += P[i][j] * dO[i][c]
            for t in range(d):
                dQ[i][t] += scale * dS * K[j][t]
                dK[j][t] += scale * dS * Q[i][t]
    return O, LSE, dQ, dK, dV


# ----------------------------------------------------------------------------------------
# Block-sparse attention: the FlashAttention summary's extension ("FlashAttention――GPUメモリ
# の読み書きを減らし、注意機構を正確なまま高速・省メモリに", section 手法): whole blocks of S are
# skipped.  Key j is visible to query i iff block_mask[i // bq, j // bk] is set (and, under the
# causal mask, j <= i).  A query that sees no key at all gets O = 0 and LSE = -inf (the
# empty sum): the pages leave that case open.
# ----------------------------------------------------------------------------------------

def forward_head_block_sparse(Q, K, V, scale: float, causal: bool, block_mask, bq: int = 128,
                              bk: int = 128):
    """Q, K, V [N, d]; block_mask [ceil(N/bq), ceil(N/bk)] of 0/1.  Returns O [N, d], LSE [N]."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    mask = np.asarray(block_mask).astype(bool)
    vis = np.repeat(np.repeat(mask, bq, axis=0), bk, axis=1)[:N, :K.shape[0]]
    if causal:
        vis &= np.arange(K.shape[0])[None, :] <= np.arange(N)[:, None]
    S = np.where(vis, scale * (Q @ K.T), -np.inf)
    O = np.zeros((N, V.shape[1]))
    lse = np.full(N, -np.inf)
    live = vis.any(axis=1)
    if live.any():
        P, lse[live] = _softmax_rows(S[live])
        O[live] = P @ V
    return O, lse


def forward_rows_block_sparse(Q, K, V, scale: float, causal: bool, block_mask, rows,
                              bq: int = 128, bk: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """O [len(rows), d] and LSE [len(rows)] of the block-sparse attention above at the selected
    query rows, without the N x N matrix (for long sequences): query i attends to the keys of
    the active blocks of its block row (and, causal, j <= i), with the plain two-pass softmax
    over that key set; a row with no such key gets O = 0, LSE = -inf."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    mask = np.asarray(block_mask).astype(bool)
    nk = K.shape[0]
    rows = np.asarray(rows)
    O = np.zeros((len(rows), V.shape[1]))
    lse = np.full(len(rows), -np.inf)
    for n, i in enumerate(rows):
        blocks = np.nonzero(mask[i // bq])[0]
        if blocks.size == 0:
            continue
        keys = np.concatenate([np.arange(b * bk, min(nk, (b + 1) * bk)) for b in blocks])
        if causal:
            keys = keys[keys <= i]
        if keys.size == 0:
            continue
        s = scale * (K[keys] @ Q[i])
        m = s.max()
        e = np.exp(s - m)
        O[n] = (e @ V[keys]) / e.sum()
        lse[n] = m + math.log(e.sum())
    return O, lse
