"""Host-side checks of the Python binding's convenience wrappers: every tensor handed to the
library is checked for shape, dtype, layout and device before any pointer crosses the C ABI
(the kernels read and write whole extents through raw pointers).  CPU tensors only: each
case is rejected before a CUDA call is made."""
import pytest
import torch


@pytest.fixture(autouse=True)
def _host_only(no_visible_gpu):
    """The wrappers must refuse every case below before a CUDA call (see no_visible_gpu)."""


@pytest.fixture(scope="module")
def fa():
    import __graft_entry__
    __graft_entry__.build()
    from exact_io_aware_88_b200 import fa as mod
    return mod


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


B, N, H, D = 2, 300, 3, 64


def test_forward_checks_every_tensor(fa):
    q = bf(B, N, H, D)
    with pytest.raises(ValueError, match="expected \\[B, N, H, d\\]"):
        fa.attention_forward(bf(N, H, D), q, q)
    with pytest.raises(ValueError, match="k: expected shape"):
        fa.attention_forward(q, bf(B, N - 1, H, D), q)
    with pytest.raises(ValueError, match="v: expected dtype"):
        fa.attention_forward(q, q, q.to(torch.float16))
    with pytest.raises(ValueError, match="q: expected dtype"):
        fa.attention_forward(q.to(torch.float16), q, q)
    with pytest.raises(ValueError, match="k must be contiguous"):
        fa.attention_forward(q, bf(B, H, N, D).transpose(1, 2), q)
    with pytest.raises(ValueError, match="out: expected shape"):
        fa.attention_forward(q, q, q, out=bf(B, N, H, D + 1))
    with pytest.raises(ValueError, match="lse: expected dtype"):
        fa.attention_forward(q, q, q, lse=torch.zeros(B, H, N, dtype=torch.float64))
    with pytest.raises(ValueError, match="lse: expected shape"):
        fa.attention_forward(q, q, q, lse=torch.zeros(B, N, H))
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_forward(q, q, q)


def test_backward_checks_every_tensor(fa):
    q = bf(B, N, H, D)
    lse = torch.zeros(B, H, N)
    with pytest.raises(ValueError, match="dO: expected shape"):
        fa.attention_backward(q, q, q, q, lse, bf(B, N, H, 2 * D))
    with pytest.raises(ValueError, match="o: expected dtype"):
        fa.attention_backward(q, q, q, q.float(), lse, q)
    with pytest.raises(ValueError, match="lse: expected shape"):
        fa.attention_backward(q, q, q, q, torch.zeros(B, N, H), q)
    with pytest.raises(ValueError, match="q: expected dtype"):
        fa.attention_backward(q.float(), q, q, q, lse, q)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_backward(q, q, q, q, lse, q)


def test_decode_checks_kv_against_q(fa):
    q = bf(B, 1, H, D)
    kv = bf(B, 500, H, D)
    with pytest.raises(ValueError, match="v: expected shape"):
        fa.attention_decode(q, kv, bf(B, 499, H, D))
    with pytest.raises(ValueError, match="k: expected shape"):
        fa.attention_decode(q, bf(B, 500, H + 1, D), kv)
    with pytest.raises(ValueError, match="unsupported dtype"):
        fa.attention_decode(q.float(), kv, kv)
    with pytest.raises(ValueError, match="k: expected dtype"):
        fa.attention_decode(q.half(), kv, kv.half())
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_decode(q, kv, kv)


def test_block_sparse_checks_the_mask(fa):
    q = bf(B, N, H, D)
    nt = (N + 127) // 128
    with pytest.raises(ValueError, match="block_mask: expected shape"):
        fa.attention_block_sparse(q, q, q, torch.ones(nt, nt - 1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="block_mask: expected shape"):
        fa.attention_block_sparse(q, q, q, torch.ones(nt * nt, dtype=torch.uint8))
    with pytest.raises(ValueError, match="block_mask: expected an integer or bool dtype"):
        fa.attention_block_sparse(q, q, q, torch.ones(nt, nt))
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.attention_block_sparse(q, q, q, torch.ones(nt, nt, dtype=torch.bool))


def test_fp8_wrappers_check_operands(fa):
    q = bf(B, N, H, 128)
    with pytest.raises(ValueError, match="signs: expected shape"):
        fa.fp8_quantize(q, q, q, torch.ones(64))
    with pytest.raises(ValueError, match="k: expected shape"):
        fa.fp8_quantize(q, bf(B, N, H, 64), q, None)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        fa.fp8_quantize(q, q, q, torch.ones(128))
    u8 = torch.zeros(B, N, H, 128, dtype=torch.uint8)
    npad = (N + 15) // 16 * 16
    vt8 = torch.zeros(B, H, 128, npad, dtype=torch.uint8)
    sc = torch.ones(3, B * H)
    with pytest.raises(ValueError, match="vt8: expected shape"):
        fa.attention_forward_fp8(u8, u8, torch.zeros(B, H, 128, N, dtype=torch.uint8), sc)
    with pytest.raises(ValueError, match="scales: expected shape"):
        fa.attention_forward_fp8(u8, u8, vt8, torch.ones(3, B))
    with pytest.raises(ValueError, match="k8: expected dtype"):
        fa.attention_forward_fp8(u8, q, vt8, sc)
    with pytest.raises(ValueError, match="q8 must be a CUDA tensor"):
        fa.attention_forward_fp8(u8, u8, vt8, sc)
