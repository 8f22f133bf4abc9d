"""fp64 CPU oracle for the FP8 forward path with incoherent processing.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.attention``): the test-suite, the smoke
check and the bench's CPU legs may use it; the library's product path never does.  It
shares no code with the CUDA kernels.

What the pages fix ("FlashAttention-3 — FlashAttention-3", section FlashAttention-3の技術的
革新, item 3, 量子化誤差を低減した低精度（FP8）):
  * before attention, the query and key feature vectors are multiplied by a random
    orthogonal matrix, a Hadamard matrix being the example named;
  * this spreads rare large entries over all coordinates, and quantising to FP8 afterwards
    loses less;
  * the matrix is orthogonal, so it cancels in Q K^T and the attention result is unchanged
    up to the quantisation error;
  * the pages report about 2.6x lower error than FP8 without the transform.

Readings where the pages are silent (each one is also listed with the design notes):
  * The matrix is M = diag(s) H_d / sqrt(d): H_d the Sylvester Hadamard matrix of order d,
    s a random +-1 vector passed in by the caller.  Rows are transformed as x -> x M, so
    (Q M)(K M)^T = Q M M^T K^T = Q K^T exactly.
  * FP8 is the OCP E4M3 format (bias 7, largest finite 448, no infinities), rounding to
    nearest, ties to even, saturating to +-448.
  * One scale per (batch, head) and tensor, a power of two: the smallest 2^e with
    448 * 2^e >= max |x| over the head (1 for an all-zero head).  A power of two keeps the
    division by the scale exact.
  * Q and K are transformed then quantised; V is quantised without a transform (it does
    not meet K's transform in P V).
  * The codes are decided in fp32, the kernel's precision: the transform is evaluated as
    the textbook fast Walsh-Hadamard transform in fp32 (sign flips, then butterfly stages
    (a + b, a - b) on pairs 1, 2, 4, ... apart, then one multiply by the fp32 value of
    1/sqrt(d)).  ``transform`` below is the exact fp64 definition; ``transform_f32`` is
    pinned to it within fp32 rounding.
  * The attention itself: softmax(scale * (s_q Q8)(s_k K8)^T)(s_v V8) in exact arithmetic is
    what the FP8 kernel approximates; its own further rounding (P to E4M3 for the second
    product) is an implementation error measured against this, not a reading.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np

from .attention import forward_head

E4M3_MAX = 448.0


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order d (a power of two): H_1 = [1],
    H_2n = [[H_n, H_n], [H_n, -H_n]].  Entries +-1, H H^T = d I."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def transform(X: np.ndarray, signs: Optional[np.ndarray]) -> np.ndarray:
    """Rows of X (last axis d) times M = diag(signs) H_d / sqrt(d).  signs=None: identity."""
    if signs is None:
        return np.asarray(X, dtype=np.float64)
    d = X.shape[-1]
    M = np.asarray(signs, dtype=np.float64)[:, None] * hadamard(d) / math.sqrt(d)
    return np.asarray(X, dtype=np.float64) @ M


def transform_f32(X: np.ndarray, signs: Optional[np.ndarray]) -> np.ndarray:
    """The transform as evaluated in fp32: x * s, log2(d) butterfly stages, times fp32
    1/sqrt(d).  Returns fp32.  signs=None: the identity (values cast to fp32)."""
    x = np.asarray(X, dtype=np.float32)
    if signs is None:
        return x
    d = x.shape[-1]
    x = x * np.asarray(signs, dtype=np.float32)
    h = 1
    while h < d:
        y = x.reshape(*x.shape[:-1], d // (2 * h), 2, h)
        a, b = y[..., 0, :], y[..., 1, :]
        x = np.stack([a + b, a - b], axis=-2).reshape(*x.shape[:-1], d)
        h *= 2
    inv = np.float32(1.0) / np.sqrt(np.float32(d))
    return x * inv


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Values of x rounded to E4M3: nearest, ties to even, saturating at +-448.  Normal
    numbers (1 + m/8) 2^(e-7), e = 1..15 (e = 15, m = 7 is NaN), subnormals m/8 * 2^-6."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros_like(a)
    nz = a > 0
    _, ex = np.frexp(a[nz])                 # a = f 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)              # floor(log2 a), subnormals share 2^-6's quantum
    quantum = np.ldexp(1.0, e - 3)          # 3 mantissa bits
    out[nz] = np.round(a[nz] / quantum) * quantum   # numpy rounds half to even
    out = np.minimum(out, E4M3_MAX)
    return np.copysign(out, x)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """uint8 codes S EEEE MMM of e4m3_round(x).  A value that rounds to zero keeps its sign
    bit (0x80 for negative)."""
    r = e4m3_round(x)
    a = np.abs(r)
    code = np.zeros(a.shape, dtype=np.int64)
    sub = (a > 0) & (a < 2.0 ** -6)
    code[sub] = np.rint(a[sub] / 2.0 ** -9).astype(np.int64)
    nrm = a >= 2.0 ** -6
    _, ex = np.frexp(a[nrm])
    e = ex - 1
    mant = np.rint((a[nrm] / np.ldexp(1.0, e) - 1.0) * 8).astype(np.int64)
    code[nrm] = ((e + 7) << 3) | mant
    code |= np.where(np.signbit(np.asarray(x, dtype=np.float64)), 0x80, 0)
    return code.astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """fp64 values of E4M3 codes (0x7F / 0xFF, the NaN codes, decode to NaN)."""
    c = np.asarray(codes, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def pow2_scale(amax: float) -> float:
    """Smallest power of two 2^e with 448 * 2^e >= amax (1.0 when amax is 0), e clamped
    to [-126, 127] so that the scale is a normal fp32 number."""
    if not amax > 0:
        return 1.0
    e = math.ceil(math.log2(amax / E4M3_MAX))
    while E4M3_MAX * 2.0 ** (e - 1) >= amax:  # guard the log2 rounding at exact powers
        e -= 1
    while E4M3_MAX * 2.0 ** e < amax:
        e += 1
    return 2.0 ** max(-126, min(127, e))  # kept a normal fp32 number


def quantize_head(X: np.ndarray, signs: Optional[np.ndarray]) -> Tuple[np.ndarray, float, float]:
    """One (batch, head) slice X [N, d]: transform (in fp32, see the module notes),
    per-head power-of-two scale, E4M3 codes.  Returns (codes [N, d] uint8, scale, amax of
    the transformed values)."""
    Xt = transform_f32(X, signs).astype(np.float64)
    amax = float(np.max(np.abs(Xt))) if Xt.size else 0.0
    sc = pow2_scale(amax)
    return e4m3_encode(Xt / sc), sc, amax


def quantize(q: np.ndarray, k: np.ndarray, v: np.ndarray, signs: Optional[np.ndarray]
             ) -> Dict[str, np.ndarray]:
    """All heads of [B, N, H, d] inputs.  Returns q8, k8 [B, N, H, d] codes, vt8 [B, H, d, N]
    codes (V per head, transposed), scales [3, B*H] (q, k, v) and amax [3, B*H]."""
    B, N, H, d = q.shape
    q8 = np.zeros((B, N, H, d), np.uint8)
    k8 = np.zeros((B, N, H, d), np.uint8)
    vt8 = np.zeros((B, H, d, N), np.uint8)
    scales = np.zeros((3, B * H))
    amax = np.zeros((3, B * H))
    for b in range(B):
        for h in range(H):
            i = b * H + h
            q8[b, :, h], scales[0, i], amax[0, i] = quantize_head(q[b, :, h], signs)
            k8[b, :, h], scales[1, i], amax[1, i] = quantize_head(k[b, :, h], signs)
            c, scales[2, i], amax[2, i] = quantize_head(v[b, :, h], None)
            vt8[b, h] = c.T
    return {"q8": q8, "k8": k8, "vt8": vt8, "scales": scales, "amax": amax}


def attention_head(q8: np.ndarray, k8: np.ndarray, vt8: np.ndarray, sq: float, sk: float,
                   sv: float, scale: float, causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention of one head on the dequantised operands: q8, k8 [N, d] codes,
    vt8 [d, N] codes.  Returns (O [N, d], LSE [N]) in fp64."""
    Q = e4m3_decode(q8) * sq
    K = e4m3_decode(k8) * sk
    V = e4m3_decode(vt8).T * sv
    return forward_head(Q, K, V, scale, causal)
