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
_lib.fa_read_device_status.argtypes = [ctypes.POINTER(_I), _P]
_lib.fa_read_device_status.restype = _I
_lib.fa_status_string.argtypes = [_I]
_lib.fa_status_string.restype = ctypes.c_char_p
_lib.fa_version.argtypes = []
_lib.fa_version.restype = _I
_lib.fa_debug_umma_tile.argtypes = [_P, _P, _P, _I, _I, _I, _P]
_lib.fa_debug_umma_tile.restype = _I
_lib.fa_debug_exp2.argtypes = [_P, _P, _P, _I, _P]
_lib.fa_debug_exp2.restype = _I
_lib.fa_debug_wait_timeout.argtypes = [ctypes.c_longlong, _P]
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


def fa_read_device_status(stream=None) -> int:
    word = _I(0)
    return _lib.fa_read_device_status(ctypes.byref(word), _stream(stream))


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


def fa_debug_wait_timeout(timeout_ns, stream=None) -> int:
    return _lib.fa_debug_wait_timeout(int(timeout_ns), _stream(stream))


# ------------------------------------------------------------------ tensor conveniences

def _check(fn: str, rc: int):
    if rc != FA_OK:
        raise FAError(fn, rc)


def _shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, N, H, d] tensors")
    return q.shape


def attention_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                      scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """O, LSE for [B, N, H, d] CUDA tensors (bf16 -> fa_fwd, fp32 -> fa_fwd_f32)."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    for t in (q, k, v):
        if not (t.is_cuda and t.is_contiguous() and t.shape == q.shape and t.dtype == q.dtype):
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    if q.dtype == torch.bfloat16:
        _check("fa_fwd", fa_fwd(q, k, v, o, l, B, H, N, d, causal, scale))
    elif q.dtype == torch.float32:
        _check("fa_fwd_f32", fa_fwd_f32(q, k, v, o, l, B, H, N, d, causal, scale))
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return o, l


def attention_backward(q, k, v, o, lse, dO, causal: bool = False, scale: Optional[float] = None,
                       workspace: Optional[torch.Tensor] = None, deterministic: bool = False):
    """dQ, dK, dV for bf16 [B, N, H, d] CUDA tensors (fa_bwd, or fa_bwd_deterministic)."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = fa_bwd_workspace_bytes(B, H, N, d)
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
    Nk = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dt = {torch.bfloat16: FA_DTYPE_BF16, torch.float16: FA_DTYPE_FP16}.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32)
    nb = fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d)
    ws = torch.empty(max(nb, 256), device=q.device, dtype=torch.uint8)
    _check("fa_fwd_splitkv", fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, dt,
                                            ws, ws.numel()))
    return o, lse


def attention_block_sparse(q, k, v, block_mask: torch.Tensor, causal: bool = False,
                           scale: Optional[float] = None):
    """O, LSE for bf16 [B, N, H, d] tensors with a [ceil(N/128), ceil(N/128)] uint8 mask."""
    B, N, H, d = _shape(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    m = block_mask.to(device=q.device, dtype=torch.uint8).contiguous()
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    nb = fa_fwd_block_sparse_workspace_bytes(B, H, N, d)
    ws = torch.empty(max(nb, 256), device=q.device, dtype=torch.uint8)
    _check("fa_fwd_block_sparse", fa_fwd_block_sparse(q, k, v, o, lse, B, H, N, d, causal, scale,
                                                      m, ws, ws.numel()))
    return o, lse


def fp8_quantize(q, k, v, signs: Optional[torch.Tensor]):
    """E4M3 operands for attention_forward_fp8 from bf16 [B, N, H, d] q, k, v; signs is the
    [d] +-1 diagonal of the Hadamard transform (None: no transform).  Returns
    (q8, k8, vt8, scales) as uint8 [B, N, H, d], uint8 [B, N, H, d], uint8 [B, H, d, Npad]
    and fp32 [3, B*H]."""
    B, N, H, d = _shape(q)
    npad = (N + 15) // 16 * 16
    dev = q.device
    q8 = torch.empty((B, N, H, d), device=dev, dtype=torch.uint8)
    k8 = torch.empty_like(q8)
    vt8 = torch.empty((B, H, d, npad), device=dev, dtype=torch.uint8)
    scales = torch.empty((3, B * H), device=dev, dtype=torch.float32)
    nb = fa_fp8_quantize_workspace_bytes(B, H)
    ws = torch.empty(max(nb, 256), device=dev, dtype=torch.uint8)
    sg = None if signs is None else signs.to(device=dev, dtype=torch.float32).contiguous()
    _check("fa_fp8_quantize", fa_fp8_quantize(q, k, v, sg, q8, k8, vt8, scales, B, H, N, d, ws,
                                              ws.numel()))
    return q8, k8, vt8, scales


def attention_forward_fp8(q8, k8, vt8, scales, causal: bool = False,
                          scale: Optional[float] = None):
    """O (bf16 [B, N, H, d]) and LSE (fp32 [B, H, N]) from fp8_quantize's operands."""
    B, N, H, d = q8.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty((B, N, H, d), device=q8.device, dtype=torch.bfloat16)
    lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
    _check("fa_fwd_fp8", fa_fwd_fp8(q8, k8, vt8, scales, o, lse, B, H, N, d, causal, scale))
    return o, lse
