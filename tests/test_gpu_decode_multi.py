"""GPU parity of the multi-token decode (kda_decode_multi): n consecutive
tokens per sequence with the state read once and the state after every token
kept, as the verify step of speculative decoding needs for rollback.

The oracle side is the plain recurrence over each sequence's n tokens from
the given state, with a snapshot after every token (snapshot_every = 1)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, decode_inputs
from helpers import TOL_BF16, TOL_F32, as_np, rel_fro, rel_max

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "beta")


def _to_multi(inp):
    """decode_inputs gives [steps, N, ...]; the multi-token call takes [N, steps, ...]."""
    return {n: inp[n].transpose(0, 1).contiguous() for n in NAMES}


def _oracle(inp, n):
    m = _to_multi(inp)
    N, H = m["q"].shape[0], m["q"].shape[2]
    flat = {k: m[k].reshape(N * n, H, -1) if k != "beta" else m[k].reshape(N * n, H) for k in NAMES}
    cu = np.arange(0, N * n + 1, n)
    out, sf, snaps, off = oracle.forward(flat["q"], flat["k"], flat["v"], flat["log_alpha"],
                                         flat["beta"], inp["S"], cu, snapshot_every=1)
    return out.reshape(N, n, H, -1), snaps.reshape(N, n, H, *snaps.shape[2:])


@pytest.mark.parametrize("n", [1, 4, 7])
def test_decode_multi_matches_oracle_bf16(n):
    inp = decode_inputs(WORKLOADS[4], steps=n, N=5, H=3, seed=7)
    m = {k: v.cuda() for k, v in _to_multi(inp).items()}
    out, S_tok = kda.decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"],
                                  inp["S"].cuda())
    torch.cuda.synchronize()
    ro, rs = _oracle(inp, n)
    assert rel_fro(as_np(out), ro) <= TOL_BF16
    for t in range(n):
        assert rel_fro(as_np(S_tok[:, t]), rs[:, t]) <= TOL_BF16


def test_decode_multi_matches_oracle_fp32_small_dims():
    from dataclasses import replace
    w = replace(WORKLOADS[0], Dk=64, Dv=64)
    inp = decode_inputs(w, steps=3, N=4, H=2, seed=3)
    m = {k: v.cuda() for k, v in _to_multi(inp).items()}
    S = inp["S"].cuda()
    S_copy = S.clone()
    out, S_tok = kda.decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], S)
    torch.cuda.synchronize()
    ro, rs = _oracle(inp, 3)
    assert rel_max(as_np(out), ro) <= TOL_F32
    assert rel_max(as_np(S_tok), rs) <= TOL_F32
    assert torch.equal(S, S_copy)          # the input state is only read


def test_decode_multi_equals_successive_single_steps_bitwise():
    n = 5
    inp = decode_inputs(WORKLOADS[4], steps=n, N=6, H=4, seed=11)
    S = inp["S"].cuda()
    m = {k: v.cuda() for k, v in _to_multi(inp).items()}
    out, S_tok = kda.decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"], S)
    S1 = S.clone()
    for t in range(n):
        o1 = kda.decode_step(*(inp[k][t].cuda() for k in NAMES), S1)
        torch.cuda.synchronize()
        assert torch.equal(o1, out[:, t])
        assert torch.equal(S1, S_tok[:, t])


def test_decode_multi_full_size_sampled_sequences():
    """Workload 4's 256 x 32 state with 4 draft tokens; every output and state of
    sampled sequences checked (the oracle computes them independently)."""
    n = 4
    inp = decode_inputs(WORKLOADS[4], steps=n)
    m = {k: v.cuda() for k, v in _to_multi(inp).items()}
    out, S_tok = kda.decode_multi(m["q"], m["k"], m["v"], m["log_alpha"], m["beta"],
                                  inp["S"].cuda())
    torch.cuda.synchronize()
    seqs = [0, 77, 255]
    sub = {k: inp[k][:, seqs].contiguous() for k in NAMES}
    sub["S"] = inp["S"][seqs].contiguous()
    ro, rs = _oracle(sub, n)
    assert rel_fro(as_np(out[seqs]), ro) <= TOL_BF16
    assert rel_fro(as_np(S_tok[seqs]), rs) <= TOL_BF16
