"""ctypes binding of libfa.so (include/fa.h, include/fa_debug.h).

Argument marshalling only: every step of the attention path runs in the library's CUDA
kernels.  There is no CPU fallback; if libfa.so is missing or cannot be loaded, importing
this module raises.

The ``fa_*`` functions mirror the C entry points one to one and accept either raw device
addresses (ints) or torch tensors (their ``data_ptr()`` is passed).  ``attention_forward``
and ``attention_backward`` are conveniences that allocate outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_WORKSPACE = 4
FA_ERR_CUDA = 5
FA_ERR_TIMEOUT = 6
FA_ERR_INTERNAL = 7
FA_DTYPE_BF16 = 0
FA_DTYPE_FP16 = 1


class FAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it first "
                          "(python -c 'import __graft_entry__ as g; g.build()')")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_lib.fa_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]
_lib.fa_fwd.restype = _I
_lib.fa_bwd_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.fa_bwd_workspace_bytes.restype = _SZ
_lib.fa_bwd.argtypes = [_P] * 9 + [_I, _I, _I, _I, _I, _F, _P, _SZ, _P]
_lib.fa_bwd.restype = _I
_lib.fa_bwd_deterministic.argtypes = [_P] * 9 + [_I, _I, _I, _I, _I, _F, _P, _SZ, _P]
_lib.fa_bwd_deterministic.restype = _I
_lib.fa_bwd_preprocess.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P]
_lib.fa_bwd_preprocess.restype = _I
_lib.fa_bwd_kv.argtypes = [_P] * 6 + [_I, _I, _I, _I, _I, _F, _P, _SZ, _P]
_lib.fa_bwd_kv.restype = _I
_lib.fa_bwd_dq_convert.argtypes = [_P, _I, _I, _I, _I, _F, _P, _SZ, _P]
_lib.fa_bwd_dq_convert.restype = _I
_lib.fa_bwd_noalloc.argtypes = [_P] * 9 + [_I, _I, _I, _I, _I, _F, _P]
_lib.fa_bwd_noalloc.restype = _I
_lib.fa_fwd_splitkv_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
_lib.fa_fwd_splitkv_workspace_bytes.restype = _SZ
_lib.fa_fwd_splitkv.argtypes = [_P] * 5 + [_I] * 6 + [_F, _I, _P, _SZ, _P]
_lib.fa_fwd_splitkv.restype = _I
_lib.fa_fwd_block_sparse_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.fa_fwd_block_sparse_workspace_bytes.restype = _SZ
_lib.fa_fwd_block_sparse.argtypes = [_P] * 5 + [_I] * 5 + [_F, _P, _P, _SZ, _P]
_lib.fa_fwd_block_sparse.restype = _I
_lib.fa_fp8_quantize_workspace_bytes.argtypes = [_I, _I]
_lib.fa_fp8_quantize_workspace_bytes.restype = _SZ
_lib.fa_fp8_quantize.argtypes = [_P] * 8 + [_I] * 4 + [_P, _SZ, _P]
_lib.fa_fp8_quantize.restype = _I
_lib.fa_fwd_fp8.argtypes = [_P] * 6 + [_I] * 5 + [_F, _P]
_lib.fa_fwd_fp8.restype = _I
_lib.fa_fwd_f32.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]
_lib.fa_fwd_f32.restype = _I
_lib.fa_read_device_status.argtypes = [_P, _P]
_lib.fa_read_device_status.restype = _I
_lib.fa_status_string.argtypes = [_I]
_lib.fa_status_string.restype = ctypes.c_char_p
_lib.fa_version.argtypes = []
_lib.fa_version.restype = _I
_lib.fa_debug_umma_tile.argtypes = [_P, _P, _P, _I, _I, _I, _P]
_lib.fa_debug_umma_tile.restype = _I
_lib.fa_debug_exp2.argtypes = [_P, _P, _P, _I, _P]
_lib.fa_debug_exp2.restype = _I
_lib.fa_debug_wait_timeout.argtypes = [ctypes.c_longlong, _P, _P]
_lib.fa_debug_wait_timeout.restype = _I
_lib.fa_debug_tma_tile.argtypes = [_P, _P] + [_I] * 8 + [_P]
_lib.fa_debug_tma_tile.restype = _I
_lib.fa_debug_tmem_roundtrip.argtypes = [_P, _P, _I, _P]
_lib.fa_debug_tmem_roundtrip.restype = _I
_lib.fa_debug_fwd_schedule.argtypes = [_I] * 5 + [_P, _I, _P]
_lib.fa_debug_fwd_schedule.restype = _I

# Every symbol the C headers declare, for the ABI self-check.
EXPORTED = sorted(["fa_fwd", "fa_bwd_workspace_bytes", "fa_bwd", "fa_bwd_deterministic", "fa_bwd_preprocess", "fa_bwd_kv",
                   "fa_bwd_dq_convert", "fa_bwd_noalloc", "fa_fwd_f32", "fa_fwd_splitkv",
                   "fa_fwd_splitkv_workspace_bytes", "fa_fwd_block_sparse",
                   "fa_fp8_quantize_workspace_bytes", "fa_fp8_quantize", "fa_fwd_fp8",
                   "fa_fwd_block_sparse_workspace_bytes", "fa_read_device_status", "fa_status_string",
                   "fa_version", "fa_debug_umma_tile", "fa_debug_wait_timeout",
                   "fa_debug_exp2", "fa_debug_tma_tile", "fa_debug_tmem_roundtrip",
                   "fa_debug_fwd_schedule"])


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def status_string(code: int) -> str:
    return _lib.fa_status_string(int(code)).decode()


def version() -> int:
    return _lib.fa_version()


def fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, stream=None) -> int:
    return _lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal),
                       float(scale), _stream(stream))


def fa_bwd_workspace_bytes(B, H, N, d) -> int:
    return _lib.fa_bwd_workspace_bytes(B, H, N, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, workspace,
           workspace_bytes, stream=None) -> int:
    return _lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                       _ptr(dk), _ptr(dv), B, H, N, d, int(causal), float(scale),
                       _ptr(workspace), int(workspace_bytes), _stream(stream))


def fa_bwd_deterministic(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, workspace,
                         workspace_bytes, stream=None) -> int:
    return _lib.fa_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
                                     _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, int(causal),
                                     float(scale), _ptr(workspace), int(workspace_bytes),
                                     _stream(stream))


def fa_bwd_preprocess(o, lse, dO, B, H, N, d, workspace, workspace_bytes, stream=None) -> int:
    return _lib.fa_bwd_preprocess(_ptr(o), _ptr(lse), _ptr(dO), B, H, N, d, _ptr(workspace),
                                  int(workspace_bytes), _stream(stream))


def fa_bwd_kv(q, k, v, dO, dk, dv, B, H, N, d, causal, scale, workspace, workspace_bytes,
              stream=None) -> int:
    return _lib.fa_bwd_kv(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dk), _ptr(dv), B, H, N, d,
                          int(causal), float(scale), _ptr(workspace), int(workspace_bytes),
                          _stream(stream))


def fa_bwd_dq_convert(dq, B, H, N, d, scale, workspace, workspace_bytes, stream=None) -> int:
    return _lib.fa_bwd_dq_convert(_ptr(dq), B, H, N, d, float(scale), _ptr(workspace),
                                  int(workspace_bytes), _stream(stream))


# Size of the library's built-in workspace used by fa_bwd_noalloc (FA_NOALLOC_WORKSPACE_BYTES).
NOALLOC_WORKSPACE_BYTES = 64 * 1024 * 1024


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, stream=None) -> int:
    """fa_bwd without a caller-provided workspace, for callers that may not allocate device
    memory (see include/fa.h).  Calls whose GPU work overlaps share one library array and
    race; serialise them."""
    return _lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(dq),
                               _ptr(dk), _ptr(dv), B, H, N, d, int(causal), float(scale),
                               _stream(stream))


def fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d) -> int:
    return _lib.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, dtype, workspace,
                   workspace_bytes, stream=None) -> int:
    return _lib.fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                               int(causal), float(scale), int(dtype), _ptr(workspace),
                               int(workspace_bytes), _stream(stream))


def fa_fp8_quantize_workspace_bytes(B, H) -> int:
    return _lib.fa_fp8_quantize_workspace_bytes(B, H)


def fa_fp8_quantize(q, k, v, signs, q8, k8, vt8, scales, B, H, N, d, workspace, workspace_bytes,
                    stream=None) -> int:
    return _lib.fa_fp8_quantize(_ptr(q), _ptr(k), _ptr(v), _ptr(signs), _ptr(q8), _ptr(k8),
                                _ptr(vt8), _ptr(scales), B, H, N, d, _ptr(workspace),
                                int(workspace_bytes), _stream(stream))


def fa_fwd_fp8(q8, k8, vt8, scales, o, lse, B, H, N, d, causal, scale, stream=None) -> int:
    return _lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(scales), _ptr(o), _ptr(lse), B, H,
                           N, d, int(causal), float(scale), _stream(stream))


def fa_fwd_block_sparse_workspace_bytes(B, H, N, d) -> int:
    return _lib.fa_fwd_block_sparse_workspace_bytes(B, H, N, d)


def fa_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, causal, scale, block_mask, workspace,
                        workspace_bytes, stream=None) -> int:
    return _lib.fa_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                    int(causal), float(scale), _ptr(block_mask), _ptr(workspace),
                                    int(workspace_bytes), _stream(stream))


def fa_fwd_f32(q, k, v, o, lse, B, H, N, d, causal, scale, stream=None) -> int:
    return _lib.fa_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                           int(causal), float(scale), _stream(stream))


def fa_read_device_status(status_word=None, stream=None) -> int:
    """Synchronises `stream` and returns (and clears) a device status word: the library-owned
    one when `status_word` is None, else the word at the start of a backward workspace."""
    return _lib.fa_read_device_status(_ptr(status_word), _stream(stream))


def fa_debug_umma_tile(a, b, c, n, k, mode, stream=None) -> int:
    return _lib.fa_debug_umma_tile(_ptr(a), _ptr(b), _ptr(c), n, k, mode, _stream(stream))


def fa_debug_exp2(x, y_poly, y_hw, n, stream=None) -> int:
    return _lib.fa_debug_exp2(_ptr(x), _ptr(y_poly), _ptr(y_hw), int(n), _stream(stream))


def fa_debug_tma_tile(x, y, B, N, H, d, b, h, row0, chunk, stream=None) -> int:
    return _lib.fa_debug_tma_tile(_ptr(x), _ptr(y), B, N, H, d, b, h, row0, chunk, _stream(stream))


def fa_debug_tmem_roundtrip(inp, out, ncols, stream=None) -> int:
    return _lib.fa_debug_tmem_roundtrip(_ptr(inp), _ptr(out), int(ncols), _stream(stream))


def fa_debug_fwd_schedule(B, H, N, causal, grid, units, max_rounds, stream=None) -> int:
    return _lib.fa_debug_fwd_schedule(B, H, N, int(causal), grid, _ptr(units), max_rounds,
                                      _stream(stream))


def fa_debug_wait_timeout(timeout_ns, status_word=None, stream=None) -> int:
    return _lib.fa_debug_wait_timeout(int(timeout_ns), _ptr(status_word), _stream(stream))


# ------------------------------------------------------------------ tensor conveniences

def _check(fn: str, rc: int):
    if rc != FA_OK:
        raise FAError(fn, rc)


def _shape(q) -> Tuple[int, int, int, int]:
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("expected [B, N, H, d] tensors")
    return tuple(q.shape)


def _require(*specs) -> None:
    """Each spec is (name, tensor, shape, dtypes).  Raises ValueError unless every tensor is
    contiguous, exactly `shape`, one of `dtypes`, and on the same CUDA device as the first.
    Shapes, dtypes and layouts are checked for all tensors before devices.  The kernels read
    and write whole extents through raw pointers, so a tensor that fails any of these would
    be read or written out of bounds."""
    for name, t, shape, dtypes in specs:
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a torch.Tensor")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        if t.dtype not in dtypes:
            raise ValueError(f"{name}: expected dtype {' or '.join(map(str, dtypes))}, "
                             f"got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    dev = specs[0][1].device
    for name, t, _, _ in specs:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")


def attention_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                      scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O, LSE for [B, N, H, d] CUDA tensors (bf16 -> fa_fwd, fp32 -> fa_fwd_f32)."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    x = (B, N, H, d)
    specs = [("q", q, x, (torch.bfloat16, torch.float32)), ("k", k, x, (q.dtype,)),
             ("v", v, x, (q.dtype,))]
    if out is not None:
        specs.append(("out", out, x, (q.dtype,)))
    if lse is not None:
        specs.append(("lse", lse, (B, H, N), (torch.float32,)))
    _require(*specs)
    with torch.cuda.device(q.device):
        o = torch.empty_like(q) if out is None else out
        l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
        if q.dtype == torch.bfloat16:
            _check("fa_fwd", fa_fwd(q, k, v, o, l, B, H, N, d, causal, scale))
        else:
            _check("fa_fwd_f32", fa_fwd_f32(q, k, v, o, l, B, H, N, d, causal, scale))
    return o, l


def attention_backward(q, k, v, o, lse, dO, causal: bool = False, scale: Optional[float] = None,
                       workspace: Optional[torch.Tensor] = None, deterministic: bool = False):
    """dQ, dK, dV for bf16 [B, N, H, d] CUDA tensors (fa_bwd, or fa_bwd_deterministic)."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    x, bf = (B, N, H, d), (torch.bfloat16,)
    specs = [("q", q, x, bf), ("k", k, x, bf), ("v", v, x, bf), ("o", o, x, bf),
             ("lse", lse, (B, H, N), (torch.float32,)), ("dO", dO, x, bf)]
    if workspace is not None:
        specs.append(("workspace", workspace, tuple(getattr(workspace, "shape", ())),
                      (getattr(workspace, "dtype", None),)))
    _require(*specs)
    nbytes = fa_bwd_workspace_bytes(B, H, N, d)
    with torch.cuda.device(q.device):
        if workspace is None:
            workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fn = fa_bwd_deterministic if deterministic else fa_bwd
        _check(fn.__name__, fn(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale,
                               workspace, workspace.numel() * workspace.element_size()))
    return dq, dk, dv


def attention_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True,
                     scale: Optional[float] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O, LSE for q [B, Nq, H, d] against k, v [B, Nk, H, d] (bf16 or fp16), split-KV."""
    B, Nq, H, d = _shape(q)
    Nk = _shape(k)[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dt = {torch.bfloat16: FA_DTYPE_BF16, torch.float16: FA_DTYPE_FP16}.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _require(("q", q, (B, Nq, H, d), (q.dtype,)), ("k", k, (B, Nk, H, d), (q.dtype,)),
             ("v", v, (B, Nk, H, d), (q.dtype,)))
    with torch.cuda.device(q.device):
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32)
        nb = fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d)
        ws = torch.empty(max(nb, 256), device=q.device, dtype=torch.uint8)
        _check("fa_fwd_splitkv", fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale,
                                                dt, ws, ws.numel()))
    return o, lse


def attention_block_sparse(q, k, v, block_mask: torch.Tensor, causal: bool = False,
                           scale: Optional[float] = None):
    """O, LSE for bf16 [B, N, H, d] tensors with a [ceil(N/128), ceil(N/128)] mask (nonzero =
    block active; any integer or bool dtype, on any device)."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nt = (N + 127) // 128
    if not isinstance(block_mask, torch.Tensor) or tuple(block_mask.shape) != (nt, nt):
        got = tuple(block_mask.shape) if isinstance(block_mask, torch.Tensor) else type(block_mask)
        raise ValueError(f"block_mask: expected shape {(nt, nt)}, got {got}")
    if block_mask.is_floating_point() or block_mask.is_complex():
        raise ValueError(f"block_mask: expected an integer or bool dtype, got {block_mask.dtype}")
    x, bf = (B, N, H, d), (torch.bfloat16,)
    _require(("q", q, x, bf), ("k", k, x, bf), ("v", v, x, bf))
    with torch.cuda.device(q.device):
        m = (block_mask != 0).to(device=q.device, dtype=torch.uint8).contiguous()
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
        nb = fa_fwd_block_sparse_workspace_bytes(B, H, N, d)
        ws = torch.empty(max(nb, 256), device=q.device, dtype=torch.uint8)
        _check("fa_fwd_block_sparse", fa_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, causal,
                                                          scale, m, ws, ws.numel()))
    return o, lse


def fp8_quantize(q, k, v, signs: Optional[torch.Tensor]):
    """E4M3 operands for attention_forward_fp8 from bf16 [B, N, H, d] q, k, v; signs is the
    [d] +-1 diagonal of the Hadamard transform (None: no transform).  Returns
    (q8, k8, vt8, scales) as uint8 [B, N, H, d], uint8 [B, N, H, d], uint8 [B, H, d, Npad]
    and fp32 [3, B*H]."""
    B, N, H, d = _shape(q)
    if signs is not None and (not isinstance(signs, torch.Tensor) or tuple(signs.shape) != (d,)):
        got = tuple(signs.shape) if isinstance(signs, torch.Tensor) else type(signs)
        raise ValueError(f"signs: expected shape {(d,)}, got {got}")
    x, bf = (B, N, H, d), (torch.bfloat16,)
    _require(("q", q, x, bf), ("k", k, x, bf), ("v", v, x, bf))
    npad = (N + 15) // 16 * 16
    dev = q.device
    with torch.cuda.device(dev):
        q8 = torch.empty((B, N, H, d), device=dev, dtype=torch.uint8)
        k8 = torch.empty_like(q8)
        vt8 = torch.empty((B, H, d, npad), device=dev, dtype=torch.uint8)
        scales = torch.empty((3, B * H), device=dev, dtype=torch.float32)
        nb = fa_fp8_quantize_workspace_bytes(B, H)
        ws = torch.empty(max(nb, 256), device=dev, dtype=torch.uint8)
        sg = None if signs is None else signs.to(device=dev, dtype=torch.float32).contiguous()
        _check("fa_fp8_quantize", fa_fp8_quantize(q, k, v, sg, q8, k8, vt8, scales, B, H, N, d,
                                                  ws, ws.numel()))
    return q8, k8, vt8, scales


def attention_forward_fp8(q8, k8, vt8, scales, causal: bool = False,
                          scale: Optional[float] = None):
    """O (bf16 [B, N, H, d]) and LSE (fp32 [B, H, N]) from fp8_quantize's operands."""
    B, N, H, d = _shape(q8)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    npad = (N + 15) // 16 * 16
    u8 = (torch.uint8,)
    _require(("q8", q8, (B, N, H, d), u8), ("k8", k8, (B, N, H, d), u8),
             ("vt8", vt8, (B, H, d, npad), u8), ("scales", scales, (3, B * H), (torch.float32,)))
    with torch.cuda.device(q8.device):
        o = torch.empty((B, N, H, d), device=q8.device, dtype=torch.bfloat16)
        lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
        _check("fa_fwd_fp8", fa_fwd_fp8(q8, k8, vt8, scales, o, lse, B, H, N, d, causal, scale))
    return o, lse
