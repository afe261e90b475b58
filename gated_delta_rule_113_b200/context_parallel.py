"""Context-parallel prefill of one long sequence over several GPUs.

The sequence is cut into consecutive segments, one per rank.  The recurrence
of the page "Kimi K3: Open Frontier Intelligence and Implementation
Framework" (section "Hybrid Attention Mechanism", KDA bullet) makes the
state the only thing a segment needs from the tokens before it, so rank r
runs ``kda_forward`` on its segment starting from the state rank r - 1 ends
with.  To keep every rank busy the heads are processed in groups: rank r
starts head group g as soon as rank r - 1 has sent the state after its
segment for that group, then sends its own state for g on to rank r + 1.
With G groups and W ranks each rank is idle for W - 1 group-steps of the
G + W - 1; ``choose_group_size`` picks G from H, W and the SM count.

The exchange is one fp32 state per head of a group (Hg x 64 KiB at
d_k = d_v = 128), sent point to point with ``torch.distributed.send`` /
``recv`` into the receiving rank's own memory.  All arithmetic runs in the
library's kernels; this module only schedules calls and moves states.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def choose_group_size(H: int, world: int, n_sms: int = 148, ctas_per_head: int = 4) -> int:
    """Heads per group for ``cp_prefill`` on ``world`` ranks of ``n_sms`` SMs.

    One group call runs the chain pass over ``ctas_per_head`` CTAs per head
    (32-wide value slices) and each of those walks the rank's whole segment:
    its time is set by the chain's per-chunk latency, not by the number of
    heads, until the call has enough heads to fill the GPU (about n_sms /
    ctas_per_head).  The rank pipeline over G groups keeps each rank busy for
    G of G + W - 1 group steps, so the job takes (G + W - 1) t(H / G) with
    t(h) = max(t_latency, h t_head).  Below the fill point t is flat and one
    group is fastest (the split then serves memory capacity: every rank holds
    only its segment); above it, groups of about the fill size balance the
    two terms.
    """
    if H < 1 or world < 1 or n_sms < 1 or ctas_per_head < 1:
        raise ValueError("H, world, n_sms and ctas_per_head must be positive")
    fill = max(1, -(-n_sms // ctas_per_head))   # heads that fill the GPU in one call
    if H <= fill or world == 1:
        return H
    groups = -(-H // fill)
    return -(-H // groups)                         # equal groups of at most `fill` heads


def busy_fraction(H: int, group_size: int, world: int) -> float:
    """Fraction of group steps each rank computes in the pipeline: G / (G + W - 1)."""
    G = len(head_groups(H, group_size))
    return G / (G + world - 1)


def head_groups(H: int, group_size: int):
    """[(h0, h1), ...] covering 0..H in groups of at most ``group_size`` heads."""
    if group_size < 1:
        raise ValueError("group_size must be positive")
    return [(h0, min(H, h0 + group_size)) for h0 in range(0, H, group_size)]


def cp_prefill(q, k, v, log_alpha, beta, S0=None, *, rank: int, world: int,
               group_size: Optional[int] = None,
               send_state: Callable[[torch.Tensor, int], None],
               recv_state: Callable[[torch.Tensor, int], None],
               forward: Optional[Callable] = None, state_dtype=torch.float32):
    """This rank's share of a context-parallel prefill of one sequence.

    q, k, log_alpha [T_r, H, Dk]; v [T_r, H, Dv]; beta [T_r, H]: the tokens of
    this rank's segment (segment r follows segment r - 1 in the sequence).
    S0 [1, H, Dk, Dv] fp32 is the sequence's initial state, used by rank 0
    only (None: zero).  ``send_state(t, peer)`` / ``recv_state(t, peer)`` move
    one contiguous state tensor; ``forward`` defaults to the library's
    prefill with the signature of ``gated_delta_rule_113_b200.forward``
    (states in ``state_dtype``, fp32 for the library).  ``group_size`` None:
    ``choose_group_size(H, world)`` (the same on every rank).

    Returns (out [T_r, H, Dv], S_final [1, H, Dk, Dv] on the last rank, None
    elsewhere).
    """
    if forward is None:
        from . import forward as library_forward   # the library's kernels
        forward = library_forward
    T, H, Dk = q.shape
    Dv = v.shape[-1]
    if group_size is None:
        group_size = choose_group_size(H, world)
    out = torch.empty((T, H, Dv), dtype=q.dtype, device=q.device)
    S_last = torch.empty((1, H, Dk, Dv), dtype=state_dtype, device=q.device) \
        if rank == world - 1 else None
    cu = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    for h0, h1 in head_groups(H, group_size):
        hs = slice(h0, h1)
        if rank == 0:
            s_in = None if S0 is None else S0[:, hs].contiguous()
        else:
            s_in = torch.empty((1, h1 - h0, Dk, Dv), dtype=state_dtype, device=q.device)
            recv_state(s_in, rank - 1)
        o_g, s_out = forward(q[:, hs].contiguous(), k[:, hs].contiguous(), v[:, hs].contiguous(),
                             log_alpha[:, hs].contiguous(), beta[:, hs].contiguous(), s_in, cu)
        out[:, hs] = o_g
        if rank < world - 1:
            send_state(s_out.contiguous(), rank + 1)
        else:
            S_last[:, hs] = s_out
    return out, S_last


def torch_distributed_transport():
    """send_state / recv_state over the default torch.distributed process group."""
    import torch.distributed as dist

    def send_state(t, peer):
        dist.send(t, dst=peer)

    def recv_state(t, peer):
        dist.recv(t, src=peer)

    return send_state, recv_state
