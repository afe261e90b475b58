"""GPU parity of kda_backward (gradients through the recurrence) against the
fp64 backward oracle, on the same seeded inputs.

The recurrence is that of the page "Kimi K3: Open Frontier Intelligence and
Implementation Framework" (section "Hybrid Attention Mechanism", KDA bullet).
Both sides see identical input values (the oracle takes the device inputs'
bf16 or fp32 values as fp64).  The kernel computes in fp32 throughout, so each
gradient tensor must match within 1e-4 relative (Frobenius): fp32 rounding
(about 6e-8 per operation) accumulated through sums of at most 128 terms per
step and a recurrence that contracts (alpha <= 1) stays near 1e-6.
"""
import dataclasses

import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs
from helpers import as_np, rel_fro, to_dev

pytestmark = pytest.mark.gpu

TOL_GRAD = 1e-4
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def _case(w, lengths, H, s0, dsf, seed=7):
    inp = forward_inputs(w, lengths=lengths, H=H, s0=s0)
    g = torch.Generator().manual_seed(seed)
    T, N = sum(lengths), len(lengths)
    inp["d_out"] = torch.randn((T, H, w.Dv), generator=g).to(inp["v"].dtype)
    inp["dS_final"] = torch.randn((N, H, w.Dk, w.Dv), generator=g) if dsf else None
    return inp


def _run(inp, need_dS0=True):
    d = to_dev(inp)
    dsf = inp["dS_final"].cuda() if inp["dS_final"] is not None else None
    g = kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                     d["cu_seqlens"], d_out=inp["d_out"].cuda(), dS_final=dsf,
                     need_dS0=need_dS0, force_simt=True)
    torch.cuda.synchronize()
    return g


def _oracle(inp):
    return oracle.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["S0"], inp["cu_seqlens"].numpy(), inp["d_out"], inp["dS_final"])


def _check(inp, g):
    ref = _oracle(inp)
    for name in GRADS:
        e = rel_fro(as_np(g[name]), ref[name])
        assert e <= TOL_GRAD, f"{name}: relative error {e:.3e}"


@pytest.mark.parametrize("widx,lengths,H,s0,dsf", [
    (1, [300, 201], 2, True, True),          # bf16, d = 128, ragged multi-chunk
    (1, [1, 63, 64, 65, 0, 130], 2, True, False),
    (0, [256], 2, False, True),              # fp32, d = 64
    (1, [129], 3, False, False),             # no initial state, no final-state gradient
])
def test_backward_matches_oracle(widx, lengths, H, s0, dsf):
    inp = _case(WORKLOADS[widx], lengths, H, s0, dsf)
    _check(inp, _run(inp))


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_backward_mixed_widths(dk, dv):
    w = dataclasses.replace(WORKLOADS[1], Dk=dk, Dv=dv)
    inp = _case(w, [190, 64], 3, True, True)
    _check(inp, _run(inp))


def test_backward_without_dS0_and_on_empty_sequences():
    inp = _case(WORKLOADS[1], [0, 77, 0], 2, True, True)
    g_full = _run(inp)
    g_part = _run(inp, need_dS0=False)
    assert g_part["dS0"] is None
    # every gradient is a fixed sequence of operations: leaving dS0 out changes none
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        assert torch.equal(g_full[name], g_part[name]), name
    # an empty sequence passes dS_final straight to dS0
    assert torch.equal(g_full["dS0"][0].cpu(), inp["dS_final"][0])
    _check(inp, g_full)


def test_backward_malformed_seqlens_reported_not_faulting():
    w = WORKLOADS[1]
    T, H = 256, 2
    inp = _case(w, [T], H, False, False)
    d = to_dev(inp)
    cu = torch.tensor([0, T, 0, T, 0, T, 0, T, 0, T], dtype=torch.int32, device="cuda")
    N = cu.numel() - 1
    for simt in (True, False):
        n_ws = kda.backward_workspace_size(N, T, H, 128, 128, force_simt=simt)
        buf = torch.zeros(n_ws + (1 << 20), dtype=torch.uint8, device="cuda")
        kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, cu,
                     d_out=inp["d_out"].cuda(), workspace=buf[:n_ws], force_simt=simt)
        assert kda.workspace_status(buf[:n_ws]) == 7
        assert not buf[n_ws:].any()            # nothing written past the workspace


def test_backward_fp32_io_bf16_gates():
    w = WORKLOADS[0]
    inp = _case(w, [150, 90], 2, True, True)
    inp["log_alpha"] = inp["log_alpha"].to(torch.bfloat16)
    inp["beta"] = inp["beta"].to(torch.bfloat16)
    _check(inp, _run(inp))


def test_backward_full_size_sampled_chains():
    """The benchmark's workload (bf16, B=2, T=4096, H=16, d=128) in one call on
    the GPU; the oracle recomputes two whole chains (one per sequence, heads 0
    and 11) from the same inputs and the sampled gradients must match."""
    w = WORKLOADS[1]
    inp = forward_inputs(w)
    g = torch.Generator().manual_seed(21)
    T, H = inp["q"].shape[:2]
    N = inp["cu_seqlens"].numel() - 1
    inp["d_out"] = torch.randn((T, H, w.Dv), generator=g).to(inp["v"].dtype)
    inp["dS_final"] = torch.randn((N, H, w.Dk, w.Dv), generator=g)
    got = _run(inp)
    cu = inp["cu_seqlens"].numpy()
    for n, h in ((0, 0), (1, 11)):
        a, b = int(cu[n]), int(cu[n + 1])
        one = {k: inp[k][a:b, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha",
                                                               "d_out")}
        one["beta"] = inp["beta"][a:b, h:h + 1].contiguous()
        one["S0"] = inp["S0"][n:n + 1, h:h + 1] if inp["S0"] is not None else None
        one["dS_final"] = inp["dS_final"][n:n + 1, h:h + 1]
        one["cu_seqlens"] = torch.tensor([0, b - a], dtype=torch.int32)
        ref = _oracle(one)
        sl = {"dq": got["dq"][a:b, h], "dk": got["dk"][a:b, h], "dv": got["dv"][a:b, h],
              "dlog_alpha": got["dlog_alpha"][a:b, h], "dbeta": got["dbeta"][a:b, h],
              "dS0": got["dS0"][n, h]}
        for name, x in sl.items():
            e = rel_fro(as_np(x), ref[name].reshape(as_np(x).shape))
            assert e <= TOL_GRAD, f"chain ({n}, {h}) {name}: relative error {e:.3e}"


def test_backward_with_no_tokens_passes_dS_final_to_dS0():
    H, D = 2, 128
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    e = torch.empty((0, H, D), dtype=torch.bfloat16, device="cuda")
    dSf = torch.randn((2, H, D, D), device="cuda")
    for simt in (True, False):
        g = kda.backward(e, e, e, e, torch.empty((0, H), dtype=torch.bfloat16, device="cuda"),
                         None, cu, d_out=e, dS_final=dSf, force_simt=simt)
        torch.cuda.synchronize()
        assert torch.equal(g["dS0"], dSf)
        g0 = kda.backward(e, e, e, e, torch.empty((0, H), dtype=torch.bfloat16, device="cuda"),
                          None, cu, d_out=e, force_simt=simt)
        torch.cuda.synchronize()
        assert torch.equal(g0["dS0"], torch.zeros_like(dSf))


def test_backward_is_bitwise_reproducible():
    """Every gradient is a fixed sequence of fp32 operations (per-slice partial
    sums added in slice order, no atomics), so two calls on the same inputs
    agree to the last bit."""
    w = WORKLOADS[1]
    inp = _case(w, [300, 129, 64], 4, True, True)
    g1 = _run(inp)
    g2 = _run(inp)
    for name in GRADS:
        assert torch.equal(g1[name], g2[name]), name
    _check(inp, g1)
