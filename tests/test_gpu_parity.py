"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Small cases compare every element; full-size workloads
compare every output of sampled (sequence, head) chains, which the oracle
computes exactly as it would inside the full problem (chains are
independent)."""
import ctypes
import math

import numpy as np
import pytest
import torch

import gated_delta_rule_113_b200 as kda
import oracle
from gated_delta_rule_113_b200.inputs import WORKLOADS, decode_inputs, forward_inputs
from helpers import as_np, err, head_slice, rel_fro, to_dev, tol

pytestmark = pytest.mark.gpu


PATHS = ["two_pass", "fused_tc", "simt"]


def _run(inp, force_simt=False, path=None, **kw):
    d = to_dev(inp)
    if path is not None:
        kw["fused_tc"] = path == "fused_tc"
        force_simt = path == "simt"
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], force_simt=force_simt, **kw)
    torch.cuda.synchronize()
    return out, sf


def _oracle(inp):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                          inp["S0"], inp["cu_seqlens"].numpy())


def _check(inp, out, sf, io_dtype, heads=None):
    ref = head_slice(inp, heads) if heads is not None else inp
    ro, rs = _oracle(ref)
    go, gs = as_np(out), as_np(sf)
    if heads is not None:
        go, gs = go[:, list(heads)], gs[:, list(heads)]
    e_o, e_s = err(go, ro, io_dtype), err(gs, rs, io_dtype)
    assert e_o <= tol(io_dtype), f"out error {e_o:.3e}"
    assert e_s <= tol(io_dtype), f"S_final error {e_s:.3e}"
    return e_o, e_s


# ---------------------------------------------------------------- small cases
def test_workload0_fp32_full():
    w = WORKLOADS[0]
    inp = forward_inputs(w)
    out, sf = _run(inp)
    _check(inp, out, sf, torch.float32)


@pytest.mark.parametrize("path", PATHS)
def test_bf16_ragged_multi_chunk(path):
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[300, 201], H=4)
    out, sf = _run(inp, path=path)
    _check(inp, out, sf, torch.bfloat16)


@pytest.mark.parametrize("dtype_idx,path", [(0, None), (1, "two_pass"), (1, "fused_tc"),
                                            (1, "simt")])
def test_varlen_edge_lengths(dtype_idx, path):
    w = WORKLOADS[dtype_idx]
    lens = [1, 63, 64, 65, 0, 130, 128, 2]
    inp = forward_inputs(w, lengths=lens, H=2, s0=True)
    out, sf = _run(inp, path=path)
    _check(inp, out, sf, w.torch_dtype)
    # zero-length sequence: S_final == S0 exactly
    assert torch.equal(sf[4].cpu(), inp["S0"][4])


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_mixed_widths(dk, dv):
    import dataclasses
    w = dataclasses.replace(WORKLOADS[1], Dk=dk, Dv=dv)
    inp = forward_inputs(w, lengths=[190, 64], H=3)
    out, sf = _run(inp)
    _check(inp, out, sf, torch.bfloat16)


def test_fp32_io_bf16_gates_and_no_initial_state():
    w = WORKLOADS[0]
    inp = forward_inputs(w, lengths=[150], H=2, s0=False)
    inp["log_alpha"] = inp["log_alpha"].to(torch.bfloat16)
    inp["beta"] = inp["beta"].to(torch.bfloat16)
    out, sf = _run(inp)
    _check(inp, out, sf, torch.float32)


def test_split_chain_gpu():
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[384], H=2)
    d = to_dev(inp)
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"])
    t0 = 192  # chunk-aligned split
    sl = lambda x, a, b: x[a:b].contiguous()
    o1, s1 = kda.forward(*(sl(d[n], 0, t0) for n in ("q", "k", "v", "log_alpha", "beta")), d["S0"])
    o2, s2 = kda.forward(*(sl(d[n], t0, 384) for n in ("q", "k", "v", "log_alpha", "beta")), s1)
    assert rel_fro(as_np(torch.cat([o1, o2])), as_np(out)) < 1e-2
    assert rel_fro(as_np(s2), as_np(sf)) < 1e-2


def test_in_place_state_continuation():
    """S_final may be the same buffer as S0."""
    w = WORKLOADS[0]
    inp = forward_inputs(w, lengths=[100, 37], H=2, s0=True)
    d = to_dev(inp)
    ref_o, ref_s = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                               d["cu_seqlens"])
    S = d["S0"].clone()
    o, s = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S, d["cu_seqlens"],
                       S_final=S)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(S, ref_s)


def test_exact_write_invariant_gpu():
    """beta = 1, q = k = unit coordinate axis: the output reproduces v (any decay)."""
    T, H, D = 200, 2, 128
    g = torch.Generator().manual_seed(5)
    idx = torch.randint(0, D, (T, H), generator=g)
    k = torch.nn.functional.one_hot(idx, D).to(torch.bfloat16)
    v = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    la = (torch.rand(T, H, D, generator=g) * math.log(0.9)).to(torch.bfloat16)
    beta = torch.ones(T, H, dtype=torch.bfloat16)
    S0 = 0.02 * torch.randn(1, H, D, D, generator=g)
    inp = dict(q=k.clone(), k=k, v=v, log_alpha=la, beta=beta, S0=S0,
               cu_seqlens=torch.tensor([0, T], dtype=torch.int32))
    out, _ = _run(inp)
    assert rel_fro(as_np(out), as_np(v)) < 1e-2


def test_value_channel_permutation():
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[130], H=2)
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(1))
    out, sf = _run(inp)
    inp2 = dict(inp, v=inp["v"][..., perm].contiguous(), S0=inp["S0"][..., perm].contiguous())
    out2, sf2 = _run(inp2)
    assert rel_fro(as_np(out2), as_np(out[..., perm.cuda()])) < 1e-3
    assert rel_fro(as_np(sf2), as_np(sf[..., perm.cuda()])) < 1e-3


@pytest.mark.parametrize("path", ["two_pass", "fused_tc"])
def test_deterministic_reruns(path):
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[257, 64], H=4)
    a = _run(inp, path=path)
    b = _run(inp, path=path)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_tensor_core_paths_agree():
    """The two-pass and the single-kernel tensor-core prefills round at
    different points (the two-pass one folds P into Qe = Qg - P W and
    PT = P Tb before the chain), so they are not bit-identical; each carries
    a bf16 operand error of a few 1e-3 against the oracle, and the two agree
    to within twice that."""
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[640, 129, 1], H=3)
    a = _run(inp, path="two_pass")
    b = _run(inp, path="fused_tc")
    assert rel_fro(as_np(a[0]), as_np(b[0])) < 1e-2
    assert rel_fro(as_np(a[1]), as_np(b[1])) < 1e-2


def test_many_heads_spread_over_the_grid():
    """More (chunk, head) items than SMs: the persistent key-side pass strides
    items over its CTAs."""
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[1000, 777, 64], H=24)
    out, sf = _run(inp)
    _check(inp, out, sf, torch.bfloat16)


def test_full_width_chain():
    """More chains than half the SMs: the chain pass runs one transposed CTA
    per (sequence, head) over all 128 value columns; ragged and empty
    sequences, with an initial state."""
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[300, 1, 64, 129, 0, 200], H=20, s0=True)
    out, sf = _run(inp)
    _check(inp, out, sf, torch.bfloat16)


def test_malformed_seqlens_reported_not_faulting():
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[64, 64], H=2)
    d = to_dev(inp)
    bad = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")  # decreasing, wrong end
    ws = torch.empty(kda.forward_workspace_size(2, 128, 2, 128, 128), dtype=torch.uint8,
                     device="cuda")
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], bad, workspace=ws)
    assert kda.workspace_status(ws) == 7
    good = d["cu_seqlens"]
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"], good, workspace=ws)
    assert kda.workspace_status(ws) == 0


def test_overlapping_seqlens_stay_inside_the_workspace():
    """Offsets that describe overlapping sequences need more chunks than the
    workspace was sized for: the kernels must flag them and write nothing out
    of bounds (the guard bytes after the workspace stay untouched)."""
    w = WORKLOADS[1]
    T, H = 256, 2
    inp = forward_inputs(w, lengths=[T], H=H)
    d = to_dev(inp)
    cu = torch.tensor([0, T, 0, T, 0, T, 0, T, 0, T], dtype=torch.int32, device="cuda")
    N = cu.numel() - 1
    n_ws = kda.forward_workspace_size(N, T, H, 128, 128)
    buf = torch.zeros(n_ws + (1 << 20), dtype=torch.uint8, device="cuda")
    ws = buf[:n_ws]
    out = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
    kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, cu, out=out,
                S_final=sf, workspace=ws)
    assert kda.workspace_status(ws) == 7
    assert int(buf[n_ws:].count_nonzero()) == 0


# ------------------------------------------------------------------- decode
def test_decode_small_all_elements():
    w = WORKLOADS[4]
    inp = decode_inputs(w, steps=6, N=8, H=4)
    S = inp["S"].cuda()
    S_ref = inp["S"].double().numpy()
    for t in range(6):
        args = [inp[n][t].cuda() for n in ("q", "k", "v", "log_alpha", "beta")]
        out = kda.decode_step(*args, S)
        ro, S_ref = oracle.decode_step(*(inp[n][t] for n in ("q", "k", "v", "log_alpha", "beta")),
                                       S_ref)
        assert rel_fro(as_np(out), ro) < 2e-2
    assert rel_fro(as_np(S), S_ref) < 2e-2


def test_decode_fp32_all_elements():
    import dataclasses
    w = dataclasses.replace(WORKLOADS[4], io_dtype="f32", Dk=64, Dv=128)
    inp = decode_inputs(w, steps=4, N=3, H=2)
    S = inp["S"].cuda()
    S_ref = inp["S"].double().numpy()
    for t in range(4):
        out = kda.decode_step(*(inp[n][t].cuda() for n in ("q", "k", "v", "log_alpha", "beta")), S)
        ro, S_ref = oracle.decode_step(*(inp[n][t] for n in ("q", "k", "v", "log_alpha", "beta")),
                                       S_ref)
        assert np.max(np.abs(as_np(out) - ro)) / np.max(np.abs(ro)) < 1e-4
    assert np.max(np.abs(as_np(S) - S_ref)) / np.max(np.abs(S_ref)) < 1e-4


def test_decode_equals_prefill():
    """64 decode steps from S equal one prefill over those 64 tokens from S0 = S."""
    w = WORKLOADS[4]
    steps, N, H = 64, 4, 2
    inp = decode_inputs(w, steps=steps, N=N, H=H)
    S = inp["S"].cuda()
    outs = []
    for t in range(steps):
        outs.append(kda.decode_step(*(inp[n][t].cuda() for n in ("q", "k", "v", "log_alpha",
                                                                  "beta")), S))
    dec_out = torch.stack(outs, 1)  # [N, steps, H, Dv]
    pk = lambda n: inp[n].transpose(0, 1).reshape(N * steps, *inp[n].shape[2:]).contiguous().cuda()
    cu = torch.arange(0, N * steps + 1, steps, dtype=torch.int32, device="cuda")
    p_out, p_s = kda.forward(pk("q"), pk("k"), pk("v"), pk("log_alpha"), pk("beta"),
                             inp["S"].cuda(), cu)
    torch.cuda.synchronize()
    assert rel_fro(as_np(dec_out.reshape(N * steps, H, -1)), as_np(p_out)) < 1e-2
    assert rel_fro(as_np(S), as_np(p_s)) < 1e-2


@pytest.mark.parametrize("H", [2, 40])   # 40 heads: the transposed full-width chain
def test_bounded_wait_times_out_and_the_context_stays_usable(H):
    """KDA_FLAG_TEST_STALL makes the chain pass wait on a barrier nothing
    arrives on: the wait gives up after its 2 s bound, the call records
    KDA_ERR_TIMEOUT, and the next call on the same context is correct."""
    import time
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[300, 129], H=H)
    d = to_dev(inp)
    ws = torch.empty(kda.forward_workspace_size(2, 429, H, 128, 128), dtype=torch.uint8,
                     device="cuda")
    lib = kda.load_library()
    out = torch.empty((429, H, 128), dtype=torch.bfloat16, device="cuda")
    sf = torch.empty((2, H, 128, 128), dtype=torch.float32, device="cuda")
    p = kda.Params(2, 429, H, 128, 128, 64, 1, 1, 4)   # KDA_FLAG_TEST_STALL
    t0 = time.time()
    rc = lib.kda_forward(*(kda._ptr(x) for x in (d["q"], d["k"], d["v"], d["log_alpha"],
                                                 d["beta"], d["S0"], d["cu_seqlens"], out, sf)),
                         ctypes.byref(p), kda._ptr(ws), ws.numel(), kda._stream(out.device))
    assert rc == 0
    assert kda.workspace_status(ws) == 6             # KDA_ERR_TIMEOUT
    assert time.time() - t0 < 20
    out2, sf2 = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                            d["cu_seqlens"], workspace=ws)
    assert kda.workspace_status(ws) == 0
    _check(inp, out2, sf2, torch.bfloat16)


# ------------------------------------------------- decay outside the chunk range
KDA_ERR_DECAY = 9


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("bad", ["too_steep", "positive", "nan"])
def test_decay_out_of_range_is_reported_and_other_chains_stay_exact(path, bad):
    """The chunked kernels need log_alpha <= 0 and an in-chunk cumulative
    log-decay above -80.  A chunk that breaks this records KDA_ERR_DECAY in the
    workspace status word; the other (sequence, head) chains still match the
    oracle (only the offending chain's results are unspecified)."""
    w = WORKLOADS[1]
    lens = [200, 150, 70]
    inp = forward_inputs(w, lengths=lens, H=2, s0=True)
    la = inp["log_alpha"].clone()
    r0 = lens[0] + 64            # second chunk of sequence 1, head 1
    if bad == "too_steep":       # -2 per token: cumulative -128 over the chunk
        la[r0:r0 + 64, 1, :] = -2.0
    elif bad == "positive":
        la[r0 + 5, 1, 7] = 0.25
    else:
        la[r0 + 9, 1, 3] = float("nan")
    inp["log_alpha"] = la
    d = to_dev(inp)
    n_ws = kda.forward_workspace_size(len(lens), sum(lens), 2, 128, 128)
    ws = torch.empty(max(n_ws, 1 << 16), dtype=torch.uint8, device="cuda")
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], workspace=ws, force_simt=path == "simt",
                          fused_tc=path == "fused_tc")
    assert kda.workspace_status(ws) == KDA_ERR_DECAY
    # every chain except (sequence 1, head 1) against the oracle
    cu = inp["cu_seqlens"].numpy()
    for n in range(len(lens)):
        for h in range(2):
            if (n, h) == (1, 1):
                continue
            sl = slice(int(cu[n]), int(cu[n + 1]))
            one = {k: inp[k][sl, h:h + 1].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
            one["S0"] = inp["S0"][n:n + 1, h:h + 1].contiguous()
            one["cu_seqlens"] = torch.tensor([0, lens[n]], dtype=torch.int32)
            ro, rs = _oracle(one)
            go = as_np(out[sl, h:h + 1])
            gs = as_np(sf[n:n + 1, h:h + 1])
            assert err(go, ro, torch.bfloat16) <= tol(torch.bfloat16), (n, h)
            assert err(gs, rs, torch.bfloat16) <= tol(torch.bfloat16), (n, h)


def test_in_range_decay_leaves_the_status_ok():
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[64, 64], H=1)
    inp["log_alpha"] = torch.full_like(inp["log_alpha"], -1.2)   # cumulative -76.8 per chunk
    d = to_dev(inp)
    n_ws = kda.forward_workspace_size(2, 128, 1, 128, 128)
    ws = torch.empty(n_ws, dtype=torch.uint8, device="cuda")
    out, sf = kda.forward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["S0"],
                          d["cu_seqlens"], workspace=ws)
    assert kda.workspace_status(ws) == 0
    _check(inp, out, sf, torch.bfloat16)


# ------------------------------------------------- the caller's current device
def _driver():
    lib = ctypes.CDLL("libcuda.so.1")
    lib.cuCtxGetCurrent.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
    return lib


def _current_ctx(drv):
    c = ctypes.c_void_p()
    assert drv.cuCtxGetCurrent(ctypes.byref(c)) == 0
    return c.value


def test_entry_points_leave_the_callers_device_and_context_current():
    """Called straight through the C ABI (no Python device guard around it),
    every entry point returns with the caller's device and CUDA context still
    current.  On a machine with two GPUs the call also runs with the caller on
    another device than the tensors'."""
    lib = kda.load_library()
    drv = _driver()
    w = WORKLOADS[1]
    inp = forward_inputs(w, lengths=[100, 40], H=2, s0=True)
    n_gpus = torch.cuda.device_count()
    for tensor_dev, caller_dev in [(0, 0)] + ([(1, 0), (0, 1)] if n_gpus > 1 else []):
        dev = torch.device("cuda", tensor_dev)
        d = to_dev(inp, dev)
        T, H, Dk = d["q"].shape
        out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
        sf = torch.empty((2, H, Dk, 128), dtype=torch.float32, device=dev)
        p = kda.Params(2, T, H, Dk, 128, 64, 1, 1, 0)
        n_ws = lib.kda_forward_workspace_size(ctypes.byref(p))
        ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())
        torch.cuda.set_device(caller_dev)
        torch.cuda.synchronize(caller_dev)
        ctx0 = _current_ctx(drv)
        stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        rc = lib.kda_forward(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]),
                             ptr(d["beta"]), ptr(d["S0"]), ptr(d["cu_seqlens"]), ptr(out),
                             ptr(sf), ctypes.byref(p), ptr(ws), n_ws, stream)
        assert rc == 0
        assert torch.cuda.current_device() == caller_dev
        assert _current_ctx(drv) == ctx0
        st = ctypes.c_int32(-1)
        assert lib.kda_workspace_status(ptr(ws), ctypes.byref(st), stream) == 0 and st.value == 0
        assert torch.cuda.current_device() == caller_dev
        assert _current_ctx(drv) == ctx0
        # an error return (misaligned workspace) restores it too
        bad_ws = ctypes.c_void_p(ws.data_ptr() + 16)
        rc = lib.kda_forward(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["log_alpha"]),
                             ptr(d["beta"]), ptr(d["S0"]), ptr(d["cu_seqlens"]), ptr(out),
                             ptr(sf), ctypes.byref(p), bad_ws, n_ws - 16, stream)
        assert rc == 4
        assert torch.cuda.current_device() == caller_dev
        assert _current_ctx(drv) == ctx0
        torch.cuda.set_device(0)
        ro, rs = _oracle(inp)
        assert err(as_np(out), ro, torch.bfloat16) <= tol(torch.bfloat16)
