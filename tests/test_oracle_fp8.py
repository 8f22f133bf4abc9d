"""Pins for the FP8 / incoherent-processing oracle (oracle.fp8) against facts that do not
come from the oracle itself: the E4M3 format's definition, an independent library
conversion, closed forms of the Hadamard transform, and the direction of the pages'
error claim ("FlashAttention-3 — FlashAttention-3", section 技術的革新 3)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from oracle import fp8


# ------------------------------------------------------------------ E4M3 format facts
@pytest.mark.parametrize("code,value", [
    (0x38, 1.0), (0x7E, 448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
    (0x40, 2.0), (0x3C, 1.5), (0xB8, -1.0), (0x00, 0.0), (0x77, 240.0),
])
def test_e4m3_decode_known_codes(code, value):
    assert fp8.e4m3_decode(np.array([code]))[0] == value


def test_e4m3_nan_codes():
    assert np.isnan(fp8.e4m3_decode(np.array([0x7F, 0xFF]))).all()


@pytest.mark.parametrize("x,expect", [
    (1.0625, 1.0),          # halfway between 1 (m=0) and 1.125 (m=1): even -> 1
    (1.1875, 1.25),         # halfway between 1.125 (m=1) and 1.25 (m=2): even -> 1.25
    (2.0 ** -10, 0.0),      # halfway between 0 and the smallest subnormal: even -> 0
    (3 * 2.0 ** -10, 2.0 ** -8),  # halfway between m=1 and m=2 subnormals -> m=2
    (500.0, 448.0),         # saturates
    (-1e9, -448.0),
    (450.0, 448.0),
    (0.3, 0.3125),          # nearest of 0.28125 / 0.3125
])
def test_e4m3_rounding_special_cases(x, expect):
    assert fp8.e4m3_round(np.array([x]))[0] == expect


def test_e4m3_every_finite_code_round_trips():
    codes = np.arange(256)
    vals = fp8.e4m3_decode(codes)
    fin = np.isfinite(vals)
    assert fin.sum() == 254
    assert np.array_equal(fp8.e4m3_encode(vals[fin]), codes[fin].astype(np.uint8))


def test_e4m3_rounding_matches_torch_float8():
    """torch's float8_e4m3fn cast is an independent round-to-nearest-even implementation;
    inside the finite range the two must agree exactly."""
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-440, 440, 20000), rng.normal(0, 1e-2, 20000),
                        rng.normal(0, 3, 20000)])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(fp8.e4m3_round(x), ref)


# ------------------------------------------------------------------ Hadamard transform
def test_hadamard_small_and_orthogonality():
    assert np.array_equal(fp8.hadamard(2), np.array([[1.0, 1.0], [1.0, -1.0]]))
    for d in (4, 64, 128):
        H = fp8.hadamard(d)
        assert np.all(np.abs(H) == 1)
        assert np.array_equal(H @ H.T, d * np.eye(d))


def _fwht(x):
    """Butterfly fast Walsh-Hadamard transform of rows (an algorithm independent of the
    oracle's explicit matrix): log2(d) stages of (a + b, a - b) on pairs `h` apart."""
    x = np.array(x, dtype=np.float64)
    d = x.shape[-1]
    h = 1
    while h < d:
        y = x.reshape(*x.shape[:-1], d // (2 * h), 2, h)
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        x = y.reshape(*x.shape[:-1], d)
        h *= 2
    return x


@pytest.mark.parametrize("d", [64, 128])
def test_transform_matches_butterfly_and_preserves_qk(d):
    rng = np.random.default_rng(d)
    X = rng.normal(size=(37, d))
    Y = rng.normal(size=(29, d))
    s = synthetic.to_f64(synthetic.draw_signs(d, 3))
    Xt = fp8.transform(X, s)
    assert np.allclose(Xt, _fwht(X * s) / math.sqrt(d), rtol=0, atol=1e-12)
    assert np.allclose(np.linalg.norm(Xt, axis=1), np.linalg.norm(X, axis=1), rtol=1e-13)
    assert np.allclose(Xt @ fp8.transform(Y, s).T, X @ Y.T, rtol=0, atol=1e-11)


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_transform_is_the_definition_within_fp32_rounding(d):
    rng = np.random.default_rng(d + 1)
    X = (rng.normal(size=(50, d)) * np.where(rng.random((50, d)) < 0.01, 10, 1)).astype(np.float32)
    s = synthetic.to_f64(synthetic.draw_signs(d, 4))
    ref = fp8.transform(X.astype(np.float64), s)
    got = fp8.transform_f32(X, s)
    assert got.dtype == np.float32
    # log2(d) + 2 roundings of |values| <= sqrt(d) max|x|
    assert np.max(np.abs(got - ref)) <= (np.log2(d) + 2) * 2.0 ** -24 * math.sqrt(d) * np.abs(X).max()
    assert np.array_equal(fp8.transform_f32(X, None), X)


def test_transform_spreads_a_single_outlier():
    d = 128
    x = np.zeros((1, d))
    x[0, 17] = 40.0
    s = synthetic.to_f64(synthetic.draw_signs(d, 3))
    assert np.allclose(np.abs(fp8.transform(x, s)), 40.0 / math.sqrt(d), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ scales and quantisation
@pytest.mark.parametrize("amax,scale", [
    (448.0, 1.0), (449.0, 2.0), (224.0, 0.5), (224.0001, 1.0), (0.0, 1.0), (1.0, 2.0 ** -8),
    (448.0 * 2 ** -20, 2.0 ** -20), (3584.0, 8.0),
])
def test_pow2_scale_rule(amax, scale):
    assert fp8.pow2_scale(amax) == scale


def test_quantize_layout_and_bounds():
    t = synthetic.draw_outliers(2, 70, 3, 64, 9)
    q, k, v = (synthetic.to_f64(t[n]) for n in ("q", "k", "v"))
    s = synthetic.to_f64(synthetic.draw_signs(64, 2))
    r = fp8.quantize(q, k, v, s)
    assert r["q8"].shape == (2, 70, 3, 64) and r["vt8"].shape == (2, 3, 64, 70)
    # Every head's largest transformed |value| lands in [224, 448] after scaling.
    for i in range(6):
        b, h = divmod(i, 3)
        qd = fp8.e4m3_decode(r["q8"][b, :, h])
        assert 224.0 <= np.max(np.abs(qd)) <= 448.0
        vd = fp8.e4m3_decode(r["vt8"][b, h]).T * r["scales"][2, i]
        assert np.max(np.abs(vd - v[b, :, h]) / np.maximum(np.abs(v[b, :, h]), 2.0 ** -6 * r["scales"][2, i])) <= 2.0 ** -4 + 1e-12


def test_incoherent_processing_lowers_fp8_attention_error():
    """The direction of the pages' claim: with rare large entries in Q, K, V, FP8 attention
    after the random Hadamard transform is closer to exact attention than FP8 without it.
    (The pages report about 2.6x; the ratio depends on the outlier model, so only the
    direction and a clear margin are pinned.)"""
    B, N, H, d = 1, 384, 2, 128
    t = synthetic.draw_outliers(B, N, H, d, 7)
    q, k, v = (synthetic.to_f64(t[n]) for n in ("q", "k", "v"))
    s = synthetic.to_f64(synthetic.draw_signs(d, 11))
    sc = 1.0 / math.sqrt(d)
    err = {}
    for name, signs in (("plain", None), ("hadamard", s)):
        r = fp8.quantize(q, k, v, signs)
        e = []
        for h in range(H):
            O, _ = fp8.attention_head(r["q8"][0, :, h], r["k8"][0, :, h], r["vt8"][0, h],
                                      *r["scales"][:, h], sc, False)
            Or, _ = oracle.forward_head(q[0, :, h], k[0, :, h], v[0, :, h], sc, False)
            e.append(np.sqrt(np.mean((O - Or) ** 2)))
        err[name] = float(np.mean(e))
    assert err["plain"] / err["hadamard"] > 1.25, err


def test_lossless_operands_give_exact_attention():
    """Inputs whose values are exact in E4M3 after the per-head power-of-two scaling are
    quantised without loss, so attention on the dequantised codes must equal exact attention
    on the inputs.  Here Q takes values in {0, +-0.5, +-1, +-1.5, +-2} (max 2, scale 2^-7),
    K the same times 4 (scale 2^-5) and V times 1/4 (scale 2^-9): each maps to E4M3 numbers
    exactly, and the three scales differ, so this pins the scale bookkeeping (s_q, s_k, s_v),
    the transposed V layout and the decoding together."""
    rng = np.random.default_rng(21)
    B, N, H, d = 1, 150, 2, 64
    vals = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 1.5, -1.5, 2.0, -2.0])
    q, k, v = (vals[rng.integers(0, len(vals), size=(B, N, H, d))] for _ in range(3))
    for x in (q, k, v):
        x[0, 0, :, 0] = 2.0  # every head's max |x| is 2 before the factors below
    k, v = 4.0 * k, 0.25 * v
    r = fp8.quantize(q, k, v, None)
    assert np.all(r["scales"][0] == 2.0 ** -7) and np.all(r["scales"][1] == 2.0 ** -5)
    assert np.all(r["scales"][2] == 2.0 ** -9)
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        for causal in (False, True):
            O, L = fp8.attention_head(r["q8"][0, :, h], r["k8"][0, :, h], r["vt8"][0, h],
                                      *r["scales"][:, h], scale, causal)
            Or, Lr = oracle.forward_head(q[0, :, h], k[0, :, h], v[0, :, h], scale, causal)
            np.testing.assert_allclose(O, Or, rtol=0, atol=1e-12)
            np.testing.assert_allclose(L, Lr, rtol=0, atol=1e-12)
