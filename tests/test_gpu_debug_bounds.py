"""The bounds-checking build of the library (-DKDA_DEBUG_BOUNDS) on ragged
problems: every checked global index stays inside its buffer (the device
status word stays KDA_OK; an index that left its buffer would be skipped and
recorded as KDA_ERR_BOUNDS, without a trap), and the results are those of the
regular build.  Covered: the two-pass prefill with snapshots (narrow and
full-width chains), the fused and CUDA-core prefills, and both backward
paths."""
import contextlib

import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
from gated_delta_rule_113_b200 import build as kbuild
from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs
from helpers import as_np, rel_fro, to_dev

pytestmark = pytest.mark.gpu

KDA_OK = 0


@contextlib.contextmanager
def debug_library():
    """Route the Python binding through libkda_debug_bounds.so for the block."""
    import os
    if not os.path.exists(kbuild.LIB_DEBUG_BOUNDS):
        kbuild.build(debug_bounds=True)
    regular = kda.load_library()
    kda._lib = kda.load_library(kbuild.LIB_DEBUG_BOUNDS)
    try:
        yield
    finally:
        kda._lib = regular


def _forward(d, lens, H, **kw):
    N, T = len(lens), sum(lens)
    ws = torch.empty(max(kda.forward_workspace_size(N, T, H, 128, 128), 1 << 16),
                     dtype=torch.uint8, device="cuda")
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], workspace=ws, **kw)
    return out, sf, kda.workspace_status(ws)


@pytest.mark.parametrize("path", ["two_pass", "two_pass_full_width", "fused_tc", "simt"])
def test_debug_bounds_build_prefill(path):
    # 40 heads: enough chains for the transposed full-width chain kernel
    lens, H = [300, 1, 64, 0, 130], (40 if path == "two_pass_full_width" else 2)
    inp = forward_inputs(WORKLOADS[1], lengths=lens, H=H, s0=True)
    d = to_dev(inp)
    kw = {"fused_tc": path == "fused_tc", "force_simt": path == "simt"}
    if path.startswith("two_pass"):
        n_snap = sum(n // 64 for n in lens)
        pool = torch.zeros((n_snap, H, 128, 128), device="cuda")
        base = torch.tensor([sum(n // 64 for n in lens[:i]) for i in range(len(lens))],
                            dtype=torch.int32, device="cuda")
        kw.update(snapshot_pool=pool, snapshot_slot_base=base, snapshot_every=64)
    out_r, sf_r, st_r = _forward(d, lens, H, **kw)
    with debug_library():
        out_d, sf_d, st_d = _forward(d, lens, H, **kw)
    assert st_r == KDA_OK and st_d == KDA_OK
    assert torch.equal(out_d, out_r) and torch.equal(sf_d, sf_r)


@pytest.mark.parametrize("simt", [False, True])
def test_debug_bounds_build_backward(simt):
    lens, H = [200, 0, 77, 64], 2
    inp = forward_inputs(WORKLOADS[1], lengths=lens, H=H, s0=True)
    d = to_dev(inp)
    g = torch.Generator().manual_seed(9)
    d_out = torch.randn((sum(lens), H, 128), generator=g).to(torch.bfloat16).cuda()
    dSf = torch.randn((len(lens), H, 128, 128), generator=g).cuda()

    def run():
        n_ws = kda.backward_workspace_size(len(lens), sum(lens), H, 128, 128, force_simt=simt)
        ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
        gr = kda.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], d_out=d_out, dS_final=dSf, workspace=ws,
                          force_simt=simt)
        return gr, kda.workspace_status(ws)

    g_r, st_r = run()
    with debug_library():
        g_d, st_d = run()
    assert st_r == KDA_OK and st_d == KDA_OK
    for name in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        assert torch.equal(g_d[name], g_r[name]), name
