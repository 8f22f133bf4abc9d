"""Seeded synthetic workloads shared by the tests, the bench and the oracle runs.

This module holds no attention arithmetic: it only names the benchmark shapes and
draws the random tensors.  Both the CUDA path and the fp64 CPU oracle are fed from
here, so the two sides see bit-identical inputs.

Workload geometry follows the attention-kernel sweep described in "FlashAttention-2を読む"
(section "約2倍という数値の対象を確認する"): sequence length 512 .. 16k, head dim 64 / 128,
causal on and off, the total number of tokens per batch fixed at 16k.  The hidden size
H*d = 2048 and the long-context / fp32-tiny cases are this library's own choices.

Recipe: every value is an iid standard normal drawn in fp32 by a CPU
``torch.Generator`` seeded with ``seed``, in the order q, k, v, dO, each of shape
[B, N, H, d] (the (batch, seq, heads, head_dim) layout used by ``flash_attn_func``);
bf16 workloads then round to bf16 (round to nearest even).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import torch

TOTAL_TOKENS = 16384
SWEEP_N = [512, 1024, 2048, 4096, 8192, 16384]


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, precision, masking and seed."""

    name: str
    B: int
    N: int
    H: int
    d: int
    causal: bool
    dtype: str  # "bf16" or "f32"
    backward: bool
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved under the causal mask (the usual attention FLOP count)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()

    def label(self) -> str:
        return (f"{self.name}:B{self.B}xN{self.N}xH{self.H}xd{self.d}"
                f"{'-causal' if self.causal else ''}-{self.dtype}")


def tiny_f32(causal: bool) -> Workload:
    return Workload("tiny_f32", 1, 128, 2, 64, causal, "f32", False, 1000)


def fwd_sweep(d: int, N: int, causal: bool) -> Workload:
    H = 2048 // d
    return Workload(f"fwd_d{d}", TOTAL_TOKENS // N, N, H, d, causal, "bf16", False,
                    1001 if d == 64 else 1002)


def fwdbwd(N: int) -> Workload:
    return Workload("fwdbwd_d128", TOTAL_TOKENS // N, N, 16, 128, True, "bf16", True, 1003)


def long_context() -> Workload:
    return Workload("long_64k", 1, 65536, 16, 128, True, "bf16", True, 1004)


def all_workloads() -> List[Workload]:
    out = [tiny_f32(False), tiny_f32(True)]
    for d in (64, 128):
        for N in SWEEP_N:
            for c in (False, True):
                out.append(fwd_sweep(d, N, c))
    for N in SWEEP_N[1:]:
        out.append(fwdbwd(N))
    out.append(long_context())
    return out


def draw(B: int, N: int, H: int, d: int, seed: int, dtype: str = "bf16",
         with_grad: bool = False) -> Dict[str, torch.Tensor]:
    """Draw q, k, v (and dO) on the CPU.  Returns contiguous [B, N, H, d] tensors."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    names = ["q", "k", "v"] + (["dO"] if with_grad else [])
    out = {}
    for nm in names:
        t = torch.randn((B, N, H, d), generator=g, dtype=torch.float32)
        if dtype == "bf16":
            t = t.to(torch.bfloat16)
        elif dtype == "f16":
            t = t.to(torch.float16)
        elif dtype != "f32":
            raise ValueError(f"unknown dtype {dtype}")
        out[nm] = t.contiguous()
    return out


def draw_workload(w: Workload, with_grad: Optional[bool] = None) -> Dict[str, torch.Tensor]:
    return draw(w.B, w.N, w.H, w.d, w.seed, w.dtype,
                w.backward if with_grad is None else with_grad)


def to_f64(t: torch.Tensor):
    """Exact upcast of a bf16/fp32 tensor to a float64 numpy array."""
    return t.to(torch.float64).numpy()


def draw_decode(B: int, Nq: int, Nk: int, H: int, d: int, seed: int, dtype: str = "bf16"
                ) -> Dict[str, torch.Tensor]:
    """q [B, Nq, H, d] and k, v [B, Nk, H, d] for decoding workloads (q drawn first)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = {}
    for nm, n in (("q", Nq), ("k", Nk), ("v", Nk)):
        t = torch.randn((B, n, H, d), generator=g, dtype=torch.float32)
        t = t.to({"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype])
        out[nm] = t.contiguous()
    return out


def decode_workloads():
    """Decoding shapes (not among the pages' prefill sweep): a batch of 8 sequences, 16 heads
    of dim 128, one new query token (and 16 for speculative-style multi-token steps) against
    4k / 16k / 64k cached keys, causal, bf16.  Returns (name, B, Nq, Nk, H, d, seed)."""
    out = []
    for Nq in (1, 16):
        for Nk in (4096, 16384, 65536):
            out.append((f"decode_q{Nq}_k{Nk}", 8, Nq, Nk, 16, 128, 1005))
    return out


def draw_outliers(B: int, N: int, H: int, d: int, seed: int, frac: float = 1e-3,
                  mag: float = 10.0) -> Dict[str, torch.Tensor]:
    """q, k, v [B, N, H, d] bf16 with rare large entries, for the FP8 error study: every entry
    is a standard normal, and an entry chosen with probability `frac` is multiplied by
    `mag`.  Drawn in the order q, k, v; for each tensor the normals first, then the uniforms
    that pick the outliers."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out = {}
    for nm in ("q", "k", "v"):
        t = torch.randn((B, N, H, d), generator=g, dtype=torch.float32)
        u = torch.rand((B, N, H, d), generator=g, dtype=torch.float32)
        t = torch.where(u < frac, t * mag, t)
        out[nm] = t.to(torch.bfloat16).contiguous()
    return out


def draw_signs(d: int, seed: int) -> torch.Tensor:
    """The random +-1 diagonal of the incoherent-processing transform, fp32 [d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    bits = torch.randint(0, 2, (d,), generator=g, dtype=torch.int64)
    return (1.0 - 2.0 * bits.to(torch.float32)).contiguous()


def fp8_workloads():
    """FP8 forward shapes: the head-dim-128 rows of the prefill sweep at 4k and 16k tokens
    per sequence, causal and not (B*N = 16384, H = 16).  Returns (name, B, N, H, d, causal,
    seed)."""
    out = []
    for N in (4096, 16384):
        for causal in (False, True):
            nm = f"fwd_fp8:B{TOTAL_TOKENS // N}xN{N}xH16xd128" + ("-causal" if causal else "")
            out.append((nm, TOTAL_TOKENS // N, N, 16, 128, causal, 1006))
    return out
