"""Shared helpers for the GPU parity tests: moving generator outputs to the
device, slicing heads for the oracle, and the two error metrics.

Tolerances (stated by the operator's accuracy targets):
  fp32 I/O : max|gpu - oracle| / max|oracle| <= 1e-4, per tensor;
  bf16 I/O : ||gpu - oracle||_F / ||oracle||_F <= 2e-2, per tensor.
"""
import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def to_dev(inp, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def rel_max(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def err(a, b, io_dtype):
    return rel_max(a, b) if io_dtype == torch.float32 else rel_fro(a, b)


def tol(io_dtype):
    return TOL_F32 if io_dtype == torch.float32 else TOL_BF16


def head_slice(inp, heads):
    """CPU copies of the prefill inputs restricted to the given heads (for the oracle)."""
    hs = list(heads)
    out = {k: inp[k][:, hs].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
    out["S0"] = None if inp["S0"] is None else inp["S0"][:, hs].contiguous()
    out["cu_seqlens"] = inp["cu_seqlens"]
    return out


def as_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)
