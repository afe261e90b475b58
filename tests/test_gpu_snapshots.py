"""GPU parity of the prefix-cache state snapshots (kda_forward_snapshots)
against the fp64 oracle's snapshots, on the same seeded inputs.

A snapshot is a chain's state right after every `every`-th token of its
sequence (page "Kimi K3: Open Frontier Intelligence and Implementation
Framework", section "Inference Serving", KDA-aware prefix caching at
512-token boundaries); the library writes snapshot m of sequence n to pool
slot slot_base[n] + m and can start a sequence from a pool slot.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs
from helpers import TOL_BF16, as_np, rel_fro, to_dev

pytestmark = pytest.mark.gpu

KDA_ERR_SLOT = 8


def _inputs(lengths, H=3, seed=None):
    return forward_inputs(WORKLOADS[1], lengths=lengths, H=H, seed=seed)


def _oracle_snaps(inp, every):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                          inp["cu_seqlens"].numpy(), snapshot_every=every)


def _pool(n_slots, H, guard=2):
    """Pool with NaN guard slots on both sides; returns (full buffer, usable view)."""
    buf = torch.full((n_slots + 2 * guard, H, 128, 128), float("nan"), dtype=torch.float32,
                     device="cuda")
    return buf, buf[guard:guard + n_slots]


def _workspace(inp):
    T, H = inp["q"].shape[:2]
    N = inp["cu_seqlens"].numel() - 1
    return torch.empty(kda.forward_workspace_size(N, T, H, 128, 128, torch.bfloat16),
                       dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("every,lengths,H", [
    (512, [1100, 600, 100, 1536, 0, 513], 3),
    (128, [1100, 600, 100, 1536, 0, 513], 3),
    (512, [1100, 600], 80),          # enough chains for the 64-wide chain slices
    (128, [700, 300, 130], 40),      # more: the transposed full-width chain
    (512, [0, 700, 0, 1024], 3),     # empty sequences own no slot, first one included
])
def test_snapshots_match_oracle(every, lengths, H):
    inp = _inputs(lengths, H=H)
    ro, rs, rsn, roff = _oracle_snaps(inp, every)
    n_snap = rsn.shape[0]
    shift = 3                               # slots need not start at 0
    buf, pool = _pool(n_snap + shift + 1, H)
    base = torch.tensor(roff + shift, dtype=torch.int32, device="cuda")
    d = to_dev(inp)
    ws = _workspace(inp)
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], workspace=ws, snapshot_pool=pool,
                          snapshot_slot_base=base, snapshot_every=every)
    assert kda.workspace_status(ws) == 0
    got = as_np(pool[shift:shift + n_snap])
    for n, L in enumerate(lengths):
        for m in range(L // every):
            e = rel_fro(got[roff[n] + m], rsn[roff[n] + m])
            assert e <= TOL_BF16, f"snapshot {m} of sequence {n}: error {e:.3e}"
    # slots nobody owns stay untouched (NaN), inside and around the pool
    assert torch.isnan(pool[:shift]).all() and torch.isnan(pool[shift + n_snap:]).all()
    assert torch.isnan(buf[:2]).all() and torch.isnan(buf[-2:]).all()
    assert rel_fro(as_np(out), ro) <= TOL_BF16 and rel_fro(as_np(sf), rs) <= TOL_BF16


def test_snapshots_leave_outputs_bit_identical():
    inp = _inputs([1030, 700])
    d = to_dev(inp)
    out0, sf0 = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                            d["cu_seqlens"])
    _, pool = _pool(4, inp["q"].shape[1])
    base = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    out1, sf1 = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                            d["cu_seqlens"], snapshot_pool=pool, snapshot_slot_base=base,
                            snapshot_every=512)
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(sf0, sf1)
    # the state at the end of a sequence whose length is a multiple of `every`
    # is its final state, bit for bit
    inp2 = _inputs([1024])
    d2 = to_dev(inp2)
    _, pool2 = _pool(2, inp2["q"].shape[1])
    _, sf2 = kda.forward(d2["q"], d2["k"], d2["v"], d2["log_alpha"], d2["beta"], d2["S0"],
                         d2["cu_seqlens"], snapshot_pool=pool2,
                         snapshot_slot_base=torch.zeros(1, dtype=torch.int32, device="cuda"),
                         snapshot_every=512)
    torch.cuda.synchronize()
    assert torch.equal(pool2[1], sf2[0])


@pytest.mark.parametrize("H", [None, 40])   # 40 heads: the transposed full-width chain
def test_resume_from_snapshot_matches_uninterrupted_run(H):
    """Prefill a prefix with snapshots, then prefill the rest of each sequence
    starting from a pool slot: outputs and final states match the oracle's
    uninterrupted run."""
    lengths = [1300, 700]
    inp = _inputs(lengths) if H is None else _inputs(lengths, H=H)
    H = inp["q"].shape[1]
    every = 512
    ro, rs = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["S0"], inp["cu_seqlens"].numpy())
    d = to_dev(inp)
    _, pool = _pool(4, H)
    base = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"],
                snapshot_pool=pool, snapshot_slot_base=base, snapshot_every=every)
    # resume sequence 0 after 1024 tokens (slot 1) and sequence 1 after 512 (slot 2)
    cu = inp["cu_seqlens"].numpy()
    starts = [cu[0] + 1024, cu[1] + 512]
    idx = np.concatenate([np.arange(starts[0], cu[1]), np.arange(starts[1], cu[2])])
    tails = [cu[1] - starts[0], cu[2] - starts[1]]
    sub = {k: d[k][idx].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
    cu_t = torch.tensor([0, tails[0], tails[0] + tails[1]], dtype=torch.int32, device="cuda")
    s0_slots = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    out_t, sf_t = kda.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], None,
                              cu_t, snapshot_pool=pool, s0_slots=s0_slots)
    torch.cuda.synchronize()
    assert rel_fro(as_np(out_t), ro[idx]) <= TOL_BF16
    assert rel_fro(as_np(sf_t), rs) <= TOL_BF16
    # a negative start slot falls back to S0
    s0_mixed = torch.tensor([-1, 2], dtype=torch.int32, device="cuda")
    S0 = torch.zeros((2, H, 128, 128), dtype=torch.float32, device="cuda")
    S0[0] = pool[1]
    out_m, sf_m = kda.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], S0,
                              cu_t, snapshot_pool=pool, s0_slots=s0_mixed)
    torch.cuda.synchronize()
    assert torch.equal(out_m, out_t) and torch.equal(sf_m, sf_t)


def test_out_of_range_slots_are_reported_not_written():
    inp = _inputs([1100, 1100])
    H = inp["q"].shape[1]
    d = to_dev(inp)
    buf, pool = _pool(3, H)
    base = torch.tensor([0, 2], dtype=torch.int32, device="cuda")   # sequence 1 needs slots 2, 3
    ws = _workspace(inp)
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], d["cu_seqlens"],
                workspace=ws, snapshot_pool=pool, snapshot_slot_base=base, snapshot_every=512)
    assert kda.workspace_status(ws) == KDA_ERR_SLOT
    assert not torch.isnan(pool).any()                 # slots 0..2 written
    assert torch.isnan(buf[:2]).all() and torch.isnan(buf[-2:]).all()   # nothing outside
    # a start slot past the pool is reported too, and that chain starts from zero
    ws2 = _workspace(inp)
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, d["cu_seqlens"],
                workspace=ws2, snapshot_pool=pool,
                s0_slots=torch.tensor([-1, 7], dtype=torch.int32, device="cuda"))
    assert kda.workspace_status(ws2) == KDA_ERR_SLOT


def test_snapshots_need_the_two_pass_path():
    inp = _inputs([256])
    d = to_dev(inp)
    _, pool = _pool(1, inp["q"].shape[1])
    base = torch.zeros(1, dtype=torch.int32, device="cuda")
    for kw in (dict(force_simt=True), dict(fused_tc=True)):
        with pytest.raises(kda.KDAError, match="UNSUPPORTED"):
            kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                        d["cu_seqlens"], snapshot_pool=pool, snapshot_slot_base=base,
                        snapshot_every=512, **kw)
