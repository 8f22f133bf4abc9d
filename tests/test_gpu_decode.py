"""GPU parity of the split-KV (decoding) forward against the fp64 oracle, bf16 and fp16."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from tests._helpers import LSE_MAX_ABS, O_MAX_ABS, O_REL_L2, max_abs, rel_l2, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    assert torch.cuda.is_available()
    return mod


def _case(fa, B, Nq, Nk, H, d, causal, dtype, seed):
    t = synthetic.draw_decode(B, Nq, Nk, H, d, seed, dtype)
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_decode(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    O_ref, L_ref = oracle.forward(*(synthetic.to_f64(t[n]) for n in ("q", "k", "v")), scale, causal)
    return to_np(o), to_np(lse), O_ref, L_ref


@pytest.mark.parametrize("B,Nq,Nk,H,d", [
    (2, 1, 1, 3, 64), (2, 1, 300, 3, 128), (1, 4, 1000, 2, 128), (2, 37, 700, 2, 64),
    (1, 128, 2048, 4, 128), (1, 200, 1000, 2, 128), (1, 100, 100, 2, 64), (3, 16, 4096, 2, 64),
])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_splitkv_parity(fa, B, Nq, Nk, H, d, causal, dtype):
    O, L, O_ref, L_ref = _case(fa, B, Nq, Nk, H, d, causal, dtype, 4000 + Nq + Nk + d)
    assert max_abs(O, O_ref) <= O_MAX_ABS, max_abs(O, O_ref)
    assert rel_l2(O, O_ref) <= O_REL_L2, rel_l2(O, O_ref)
    assert max_abs(L, L_ref) <= LSE_MAX_ABS, max_abs(L, L_ref)


def test_splitkv_square_causal_matches_forward_kernel(fa):
    # Nq = Nk: the bottom-right causal alignment coincides with the square mask of fa_fwd.
    t = synthetic.draw(2, 640, 3, 128, 77, "bf16")
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    o2, l2 = fa.attention_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert max_abs(to_np(o1), to_np(o2)) <= 8e-3
    assert max_abs(to_np(l1), to_np(l2)) <= 1e-4


@pytest.mark.parametrize("Nk", [16384, 65536])
def test_splitkv_decode_one_token_full_size(fa, Nk):
    B, Nq, H, d = 8, 1, 16, 128
    O, L, O_ref, L_ref = None, None, None, None
    t = synthetic.draw_decode(B, Nq, Nk, H, d, 5000 + Nk, "bf16")
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (B - 1, H - 1), (3, 7)]:
        Q, K, V = (synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v"))
        Or, Lr = oracle.forward_head(Q, K, V, 1.0 / math.sqrt(d), True)
        assert max_abs(to_np(o[b, :, h]), Or) <= O_MAX_ABS
        assert abs(float(lse[b, h, 0]) - Lr[0]) <= LSE_MAX_ABS


def test_splitkv_rejects_bad_arguments(fa):
    a16 = 1 << 20
    p = [a16] * 5
    nb = fa.fa_fwd_splitkv_workspace_bytes(1, 1, 4, 100, 128)
    assert nb > 0
    # causal needs Nq <= Nk
    assert fa.fa_fwd_splitkv(*p, 1, 1, 200, 100, 128, 1, 0.1, 0, a16, 1 << 30, stream=0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_splitkv(*p, 1, 1, 4, 100, 96, 0, 0.1, 0, a16, 1 << 30, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_splitkv(*p, 1, 1, 4, 100, 128, 0, 0.1, 7, a16, 1 << 30, stream=0) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_splitkv(*p, 1, 1, 4, 100, 128, 0, 0.1, 0, a16, nb - 1, stream=0) == fa.FA_ERR_WORKSPACE


# ------------------------------------------------------------------ block-sparse forward

def _bs_case(fa, B, N, H, d, causal, mask, seed):
    t = synthetic.draw(B, N, H, d, seed, "bf16")
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_block_sparse(q, k, v, torch.from_numpy(mask), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    for b in range(B):
        for h in range(H):
            Or, Lr = oracle.forward_head_block_sparse(*(synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v")),
                                                      scale, causal, mask)
            O, L = to_np(o[b, :, h]), to_np(lse[b, h])
            assert max_abs(O, Or) <= O_MAX_ABS
            if np.linalg.norm(Or) > 0:
                assert rel_l2(O, Or) <= O_REL_L2
            live = np.isfinite(Lr)
            assert np.all(np.isneginf(L[~live])) and np.all(O[~live] == 0)
            assert max_abs(L[live], Lr[live]) <= LSE_MAX_ABS


@pytest.mark.parametrize("N,d", [(1000, 128), (700, 64), (129, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_random_masks(fa, N, d, causal):
    nt = (N + 127) // 128
    mask = (np.random.default_rng(N + d).random((nt, nt)) < 0.5).astype(np.uint8)
    mask[0, 0] = 1
    _bs_case(fa, 2, N, 2, d, causal, mask, 6000 + N)


def test_block_sparse_all_ones_equals_dense_and_empty_rows(fa):
    N, d = 640, 128
    _bs_case(fa, 1, N, 3, d, True, np.ones((5, 5), np.uint8), 6100)
    m = np.eye(5, dtype=np.uint8)
    m[2, 2] = 0  # block row 2 sees nothing: O = 0, lse = -inf
    _bs_case(fa, 1, N, 2, d, False, m, 6101)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_block_sparse_empty_query_tiles_with_several_units_per_cta(fa, d, causal):
    """More units than SMs (32 heads x 8 query-tile pairs = 256 on 148 persistent CTAs, so
    most CTAs take two units) with every third query tile seeing no key: a query tile with
    nothing to accumulate follows, in the same CTA, one that had work, and its empty O must
    be signalled only after the previous O was read."""
    N, H = 2048, 32
    nt = N // 128
    rng = np.random.default_rng(300 + d)
    m = (rng.random((nt, nt)) < 0.4).astype(np.uint8)
    m[np.arange(nt), np.arange(nt)] = 1
    m[np.arange(nt) % 3 == 1, :] = 0
    _bs_case(fa, 1, N, H, d, causal, m, 6300 + d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_interleaved_and_odd_tile_counts(fa, d, causal):
    """Masks that make the two query tiles of a pair take turns (tile 2p on even key tiles,
    tile 2p+1 on odd ones, so most of each tile's next products wait for a later key tile),
    an odd number of query tiles (the last pair has one tile), and a pair with one tile
    empty."""
    N = 1100  # 9 query tiles
    nt = (N + 127) // 128
    m = np.zeros((nt, nt), np.uint8)
    for i in range(nt):
        m[i, (i % 2)::2] = 1
        m[i, i] = 1
    m[3, :] = 0  # tile 3 sees nothing: O = 0, lse = -inf (its pair partner is tile 2)
    _bs_case(fa, 1, N, 3, d, causal, m, 6200 + d)



def _bs_sampled(fa, B, N, H, d, causal, mask, seed, heads, rows):
    """Block-sparse forward at full size, checked at sampled rows of a few heads."""
    t = synthetic.draw(B, N, H, d, seed, "bf16")
    q, k, v = (t[n].cuda() for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_block_sparse(q, k, v, torch.from_numpy(mask), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_read_device_status() == 0
    for b, h in heads:
        Or, Lr = oracle.forward_rows_block_sparse(*(synthetic.to_f64(t[n][b, :, h]) for n in ("q", "k", "v")),
                                                  scale, causal, mask, rows)
        O, L = to_np(o[b, rows, h]), to_np(lse[b, h, rows])
        live = np.isfinite(Lr)
        assert np.all(np.isneginf(L[~live])) and np.all(O[~live] == 0)
        assert max_abs(O, Or) <= O_MAX_ABS
        assert rel_l2(O[live], Or[live]) <= O_REL_L2
        assert max_abs(L[live], Lr[live]) <= LSE_MAX_ABS


@pytest.mark.parametrize("d,causal", [(128, False), (128, True), (64, False)])
def test_block_sparse_full_size_sampled_rows(fa, d, causal):
    """The benchmark's block-sparse size (N = 16384, H*d = 2048, a random mask of density 0.5
    with the diagonal kept): 128 query tiles per head, so each persistent CTA walks many units
    with different active-tile counts; sampled rows of four heads."""
    N, H = 16384, 2048 // d
    nt = N // 128
    m = (np.random.default_rng(400 + d).random((nt, nt)) < 0.5).astype(np.uint8)
    m[np.arange(nt), np.arange(nt)] = 1
    rng = np.random.default_rng(401 + d)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, N - 129, N - 1], rng.integers(0, N, 41)]))
    heads = [(0, 0), (0, H // 3), (0, H // 2), (0, H - 1)]
    _bs_sampled(fa, 1, N, H, d, causal, m, 7000 + d, heads, rows)


def test_block_sparse_longest_supported_sequence(fa):
    """N = 131072, the documented limit (1024 key tiles: every one of a query tile's 32 bitmask
    words is in use), with a causal band of 8 key tiles plus the first key tile, and a query
    tile whose band is cut out; rows from the first, a middle and the last query tiles."""
    N, H, d = 131072, 2, 128
    nt = N // 128
    m = np.zeros((nt, nt), np.uint8)
    for i in range(nt):
        m[i, max(0, i - 7):i + 1] = 1
        m[i, 0] = 1
    m[700, :] = 0  # this query tile sees nothing: O = 0, LSE = -inf
    rows = np.array([0, 1, 127, 128, 700 * 128, 700 * 128 + 127, 701 * 128 + 5, 65535, 65536,
                     N - 130, N - 129, N - 128, N - 2, N - 1])
    _bs_sampled(fa, 1, N, H, d, True, m, 7100, [(0, 0), (0, 1)], rows)
