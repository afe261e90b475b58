"""Parity at the measured workloads' full sizes, in the launch configuration the
benchmark times (one ``kda.forward`` / ``kda.decode_step`` call over the whole
problem).  The oracle recomputes sampled (sequence, head) chains in full;
chains are independent, so each sampled chain is checked exactly as it sits
inside the full problem."""
import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, decode_inputs, forward_inputs
from helpers import as_np, err, head_slice, rel_fro, to_dev, tol

pytestmark = pytest.mark.gpu


def _full(widx, heads):
    w = WORKLOADS[widx]
    inp = forward_inputs(w)
    d = to_dev(inp)
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"])
    torch.cuda.synchronize()
    hs = list(heads)
    out_h = as_np(out[:, hs])
    sf_h = as_np(sf[:, hs])
    del d, out, sf
    ref = head_slice(inp, hs)
    ro, rs = oracle.forward(ref["q"], ref["k"], ref["v"], ref["log_alpha"], ref["beta"],
                            ref["S0"], ref["cu_seqlens"].numpy())
    e_o, e_s = err(out_h, ro, w.torch_dtype), err(sf_h, rs, w.torch_dtype)
    assert e_o <= tol(w.torch_dtype), f"out error {e_o:.3e}"
    assert e_s <= tol(w.torch_dtype), f"S_final error {e_s:.3e}"
    # every sampled chain individually, too
    cu = inp["cu_seqlens"].numpy()
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        for i in range(len(hs)):
            if b > a:
                assert rel_fro(out_h[a:b, i], ro[a:b, i]) <= tol(w.torch_dtype)
            assert rel_fro(sf_h[n, i], rs[n, i]) <= tol(w.torch_dtype)


def test_workload1_full_all_heads():
    _full(1, range(16))


def test_workload2_full_sampled_heads():
    _full(2, [0, 13, 31])


def test_workload3_varlen_full_sampled_heads():
    _full(3, [0, 21])


def test_workload4_decode_full_sampled_sequences():
    w = WORKLOADS[4]
    inp = decode_inputs(w)
    S = inp["S"].cuda()
    outs = []
    for t in range(w.decode_steps):
        outs.append(kda.decode_step(*(inp[n][t].cuda() for n in ("q", "k", "v", "log_alpha",
                                                                  "beta")), S).cpu())
    torch.cuda.synchronize()
    seqs = [0, 1, 77, 128, 200, 255]
    S_ref = inp["S"][seqs].double().numpy()
    for t in range(w.decode_steps):
        ro, S_ref = oracle.decode_step(*(inp[n][t][seqs] for n in ("q", "k", "v", "log_alpha",
                                                                    "beta")), S_ref)
        assert rel_fro(as_np(outs[t][seqs]), ro) <= 2e-2
    assert rel_fro(as_np(S[seqs]), S_ref) <= 2e-2
