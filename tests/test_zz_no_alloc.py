"""The allocation-free prefill entry point (for callers that cannot allocate
device memory, e.g. engines with a fixed memory plan or plug-ins inside an
application that owns the allocator) must give the same results as the
workspace-taking entry point.

This file is collected last so that a run stopping at its first failure has
already run every other test; it passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2   # ||a - b||_F / ||b||_F, the bf16 tolerance of the parity tests
KDA_ERR_UNSUPPORTED = 2


def _noalloc_fn():
    lib = kda.load_library()
    fn = lib.kda_forward_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 9 + [ctypes.POINTER(kda.Params), ctypes.c_void_p]
    return fn


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    fn = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, lens in enumerate(([200, 77, 64], [130, 1, 255])):
        inp = forward_inputs(WORKLOADS[1], lengths=lens, H=2, seed=100 + call)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        ref_out, ref_sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                                      d["cu_seqlens"])
        out = torch.full_like(ref_out, float("nan"))
        sf = torch.full_like(ref_sf, float("nan"))
        T, H, Dk = d["q"].shape
        p = kda.Params(len(lens), T, H, Dk, d["v"].shape[-1], 64, 1, 1, 0)
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())
        rc = fn(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]), ptr(d["beta"]),
                ptr(d["S0"]), ptr(d["cu_seqlens"]), ptr(out), ptr(sf), ctypes.byref(p), stream)
        assert rc == 0, f"kda_forward_noalloc returned {rc}"
        torch.cuda.synchronize()
        assert _rel(out, ref_out) <= TOL_BF16
        assert _rel(sf, ref_sf) <= TOL_BF16


def _status_fn():
    lib = kda.load_library()
    fn = lib.kda_forward_noalloc_status
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p]
    return fn


def test_noalloc_status_reports_what_the_device_saw():
    """The status word of the library's scratch array reads back through
    kda_forward_noalloc_status: OK after a well-formed call, KDA_ERR_SEQLENS
    after one with malformed offsets, OK again after the next good call."""
    fn, st_fn = _noalloc_fn(), _status_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    inp = forward_inputs(WORKLOADS[1], lengths=[100, 60], H=2, seed=7)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    T, H, Dk = d["q"].shape
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((2, H, Dk, 128), dtype=torch.float32, device="cuda")
    p = kda.Params(2, T, H, Dk, 128, 64, 1, 1, 0)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    bad_cu = torch.tensor([0, 120, 100], dtype=torch.int32, device="cuda")   # ends short of T
    for cu, want in ((d["cu_seqlens"], 0), (bad_cu, 7), (d["cu_seqlens"], 0)):
        rc = fn(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]), ptr(d["beta"]),
                ptr(d["S0"]), ptr(cu), ptr(out), ptr(sf), ctypes.byref(p), stream)
        assert rc == 0
        st = ctypes.c_int32(-1)
        assert st_fn(ptr(cu), ctypes.byref(st), stream) == 0
        assert st.value == want


def test_noalloc_rejects_too_many_sequences():
    fn = _noalloc_fn()
    p = kda.Params(16385, 16385, 1, 128, 128, 64, 1, 1, 0)
    fake = ctypes.c_void_p(0x10000)
    rc = fn(*([fake] * 9), ctypes.byref(p), None)
    assert rc == KDA_ERR_UNSUPPORTED
