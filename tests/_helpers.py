"""Shared helpers for the GPU parity tests (comparison metrics, device transfer)."""
import numpy as np
import torch

# Tolerances for bf16 inputs with fp32 accumulation, and for the fp32 path.
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2
F32_MAX_ABS = 1e-5


def rel_l2(x, ref):
    return float(np.linalg.norm(np.asarray(x) - ref) / np.linalg.norm(ref))


def max_abs(x, ref):
    return float(np.abs(np.asarray(x) - ref).max())


def to_np(t: torch.Tensor):
    return t.detach().to(torch.float64).cpu().numpy()


def cuda(tensors, names):
    return [tensors[n].to("cuda:0") for n in names]


def grad_err(x, ref):
    """Relative L2 error; where the exact gradient is identically zero (e.g. dQ and dK of a
    single-key problem, whose softmax is constant) the max-abs error is returned instead."""
    n = float(np.linalg.norm(ref))
    if n == 0.0:
        return float(np.abs(np.asarray(x)).max())
    return rel_l2(x, ref)
