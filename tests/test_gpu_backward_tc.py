"""GPU parity of the chunked tensor-core backward (kda_backward for bf16 q, k,
v and gates with d_k = d_v = 128) against the fp64 backward oracle.

The path runs the forward's two passes keeping every chunk's entering state,
a reverse state chain on the transposed packet tiles, and a chunk-parallel
gradient assembly with bf16 tensor-core products and fp32 accumulation (the
chunk form of the recurrence of the page "Kimi K3: Open Frontier
Intelligence and Implementation Framework", section "Hybrid Attention
Mechanism", KDA bullet, run backwards).  Its operands are rounded to bf16 like
the forward's, so every gradient tensor is held to the bf16 tolerance of the
forward: ||gpu - oracle||_F / ||oracle||_F <= 2e-2.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs
from helpers import TOL_BF16, as_np, rel_fro, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def _case(lengths, H, s0, dsf, seed=7, w=WORKLOADS[1]):
    inp = forward_inputs(w, lengths=lengths, H=H, s0=s0, seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    T, N = sum(lengths), len(lengths)
    inp["d_out"] = torch.randn((T, H, w.Dv), generator=g).to(torch.bfloat16)
    inp["dS_final"] = torch.randn((N, H, w.Dk, w.Dv), generator=g) if dsf else None
    return inp


def _run(inp, workspace=None):
    d = to_dev(inp)
    dsf = inp["dS_final"].cuda() if inp["dS_final"] is not None else None
    g = kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                     d["cu_seqlens"], d_out=inp["d_out"].cuda(), dS_final=dsf,
                     workspace=workspace)
    torch.cuda.synchronize()
    return g


def _oracle(inp):
    return oracle.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["S0"], inp["cu_seqlens"].numpy(), inp["d_out"], inp["dS_final"])


def _check(inp, g, tol=TOL_BF16):
    ref = _oracle(inp)
    errs = {}
    for name in GRADS:
        if ref[name].size == 0:
            continue
        errs[name] = rel_fro(as_np(g[name]), ref[name])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"relative errors above {tol}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("lengths,H,s0,dsf", [
    ([64], 1, False, False),                 # one full chunk
    ([128], 1, True, True),                  # two chunks, both state gradients
    ([300, 201], 2, True, True),             # ragged multi-chunk
    ([1, 63, 64, 65, 0, 130], 2, True, False),   # edge lengths and an empty sequence
    ([129], 3, False, False),
    ([200, 77, 64], 30, True, True),         # enough chains for the transposed forward chain
])
def test_chunked_backward_matches_oracle(lengths, H, s0, dsf):
    inp = _case(lengths, H, s0, dsf)
    _check(inp, _run(inp))


def test_chunked_backward_is_bitwise_reproducible():
    inp = _case([300, 129, 64], 4, True, True, seed=11)
    g1, g2 = _run(inp), _run(inp)
    for name in GRADS:
        assert torch.equal(g1[name], g2[name]), name


def test_chunked_backward_agrees_with_the_fp32_path():
    """The two backward kernels on the same inputs: the fp32 CUDA-core one is
    within 1e-4 of the oracle, so the tensor-core one must sit within the bf16
    tolerance of it as well."""
    inp = _case([200, 77], 2, True, True, seed=3)
    tc = _run(inp)
    d = to_dev(inp)
    f32 = kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                       d["cu_seqlens"], d_out=inp["d_out"].cuda(),
                       dS_final=inp["dS_final"].cuda(), force_simt=True)
    torch.cuda.synchronize()
    for name in GRADS:
        assert rel_fro(as_np(tc[name]), as_np(f32[name])) <= TOL_BF16, name


def test_chunked_backward_reports_out_of_range_decay():
    inp = _case([128, 64], 2, True, True, seed=5)
    la = inp["log_alpha"].clone()
    la[64:128, 1, :] = -2.0          # cumulative -128 over the second chunk of sequence 0
    inp["log_alpha"] = la
    n_ws = kda.backward_workspace_size(2, 192, 2, 128, 128)
    ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
    _run(inp, workspace=ws)
    assert kda.workspace_status(ws) == 9


def test_chunked_backward_full_size_sampled_chains():
    """The B=2, T=4096, H=16, d=128 workload in one call; the oracle recomputes
    two whole chains (heads 0 and 11 of the two sequences) and all six
    gradients of those chains must match."""
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
            assert e <= TOL_BF16, f"chain ({n}, {h}) {name}: relative error {e:.3e}"
