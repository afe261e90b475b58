"""Seeded synthetic inputs for the KDA operator.

This module only draws random numbers and shapes them; it holds none of the
operator's arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  Every draw comes from ``numpy.random.default_rng(seed)`` (PCG64) in
float32, in a fixed order: sequence lengths (varlen workloads only), q, k, v,
beta logits, log_alpha, initial state.

Distributions (the workloads the KDA operator is measured on):
  q, k      ~ N(0, 1), then L2-normalised per (token, head) over d_k in fp32,
              then cast to the I/O dtype;
  v         ~ N(0, 1);
  beta      = sigmoid(N(0, 1));
  log_alpha ~ U[ln(alpha_min), 0] per channel (alpha_min is the workload's
              lower bound on the decay);
  S0        ~ N(0, s0_std) in fp32, or zero.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    io_dtype: str                 # "f32" or "bf16" (q, k, v, out, log_alpha, beta)
    lengths: tuple                # per-sequence token counts
    H: int
    Dk: int
    Dv: int
    alpha_min: float              # log_alpha ~ U[ln(alpha_min), 0]
    s0_std: Optional[float]       # None -> zero initial state
    seed: int
    varlen_range: Optional[tuple] = None   # (lo, hi) inclusive, drawn lengths
    n_varlen: int = 0
    decode_steps: int = 0         # > 0: recurrent decode workload

    @property
    def torch_dtype(self):
        return torch.float32 if self.io_dtype == "f32" else torch.bfloat16


# The five measured workloads of the KDA operator.
WORKLOADS = {
    0: Workload("kda_fwd_f32_B1_T256_H2_d64", "f32", (256,), 2, 64, 64, 0.5, None, 0),
    1: Workload("kda_prefill_bf16_B2_T4096_H16_d128", "bf16", (4096, 4096), 16, 128, 128,
                0.9, 0.02, 1),
    2: Workload("kda_prefill_bf16_B1_T65536_H32_d128", "bf16", (65536,), 32, 128, 128,
                0.95, None, 2),
    3: Workload("kda_varlen_bf16_N8_U1024_32768_H32_d128", "bf16", (), 32, 128, 128,
                0.95, 0.02, 3, varlen_range=(1024, 32768), n_varlen=8),
    4: Workload("kda_decode_N256_H32_d128_64steps", "bf16", (1,) * 256, 32, 128, 128,
                0.9, 0.02, 4, decode_steps=64),
}


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _l2norm(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-20))).astype(np.float32)


def _cast(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def resolve_lengths(w: Workload, rng) -> List[int]:
    if w.varlen_range is not None:
        lo, hi = w.varlen_range
        return [int(x) for x in rng.integers(lo, hi + 1, size=w.n_varlen)]
    return list(w.lengths)


def forward_inputs(w: Workload, lengths: Optional[List[int]] = None, H: Optional[int] = None,
                   seed: Optional[int] = None, s0: Optional[bool] = None):
    """Packed prefill inputs as CPU tensors.

    ``lengths``/``H``/``seed`` override the workload's (for reduced-size parity
    cases with the same distributions); ``s0`` forces (True) or drops (False)
    the initial state.  Returns a dict with q, k, v, log_alpha [T, H, D] and
    beta [T, H] in the I/O dtype, S0 [N, H, Dk, Dv] fp32 or None, cu_seqlens
    int32 [N+1], and ``lengths``.
    """
    rng = np.random.default_rng(w.seed if seed is None else seed)
    drawn = resolve_lengths(w, rng)
    lens = list(lengths) if lengths is not None else drawn
    H = w.H if H is None else H
    T = int(sum(lens))
    N = len(lens)
    q = _l2norm(_normal(rng, (T, H, w.Dk)))
    k = _l2norm(_normal(rng, (T, H, w.Dk)))
    v = _normal(rng, (T, H, w.Dv))
    beta = 1.0 / (1.0 + np.exp(-_normal(rng, (T, H))))
    la = rng.uniform(math.log(w.alpha_min), 0.0, size=(T, H, w.Dk)).astype(np.float32)
    use_s0 = (w.s0_std is not None) if s0 is None else s0
    S0 = None
    if use_s0:
        std = w.s0_std if w.s0_std is not None else 0.02
        S0 = torch.from_numpy(_normal(rng, (N, H, w.Dk, w.Dv)) * np.float32(std))
    dt = w.torch_dtype
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return dict(q=_cast(q, dt), k=_cast(k, dt), v=_cast(v, dt), log_alpha=_cast(la, dt),
                beta=_cast(beta.astype(np.float32), dt), S0=S0, cu_seqlens=cu, lengths=lens)


def decode_inputs(w: Workload, steps: Optional[int] = None, N: Optional[int] = None,
                  H: Optional[int] = None, seed: Optional[int] = None):
    """Recurrent-decode inputs: per-step q, k, log_alpha [steps, N, H, Dk],
    v [steps, N, H, Dv], beta [steps, N, H] in the I/O dtype, and the fp32
    state S [N, H, Dk, Dv]."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    steps = w.decode_steps if steps is None else steps
    N = len(w.lengths) if N is None else N
    H = w.H if H is None else H
    q = _l2norm(_normal(rng, (steps, N, H, w.Dk)))
    k = _l2norm(_normal(rng, (steps, N, H, w.Dk)))
    v = _normal(rng, (steps, N, H, w.Dv))
    beta = 1.0 / (1.0 + np.exp(-_normal(rng, (steps, N, H))))
    la = rng.uniform(math.log(w.alpha_min), 0.0, size=(steps, N, H, w.Dk)).astype(np.float32)
    std = w.s0_std if w.s0_std is not None else 0.02
    S = torch.from_numpy(_normal(rng, (N, H, w.Dk, w.Dv)) * np.float32(std))
    dt = w.torch_dtype
    return dict(q=_cast(q, dt), k=_cast(k, dt), v=_cast(v, dt), log_alpha=_cast(la, dt),
                beta=_cast(beta.astype(np.float32), dt), S=S)
