"""Host-only checks of the C ABI (no GPU): the library loads, exports every
function ``include/kda.h`` declares, and rejects malformed calls with the
documented status codes before touching the device."""
import ctypes
import os
import re

import numpy as np

import pytest

import gated_delta_rule_113_b200 as kda

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def _declared_functions():
    names = set()
    for fn in os.listdir(HEADER):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_loads_and_exports_every_declared_symbol():
    lib = kda.load_library()
    declared = _declared_functions()
    assert declared, "no declarations parsed from include/*.h"
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(kda.EXPORTED_SYMBOLS) <= set(declared)
    text = open(os.path.join(HEADER, "kda.h")).read()
    assert lib.kda_abi_version() == int(re.search(r"#define KDA_ABI_VERSION (\d+)", text).group(1))
    assert lib.kda_abi_version() == 4


def test_status_strings():
    lib = kda.load_library()
    for code in range(0, 11):
        assert lib.kda_status_string(code).startswith(b"KDA_")
    assert lib.kda_status_string(1234) == b"KDA_ERR_UNKNOWN"


def _params(**kw):
    base = dict(num_seqs=2, total_tokens=128, H=4, Dk=128, Dv=128, chunk=64,
                io_dtype=1, gate_dtype=1, flags=0)
    base.update(kw)
    return kda.Params(**base)


def test_workspace_size():
    lib = kda.load_library()
    p = _params(num_seqs=1000)
    assert lib.kda_forward_workspace_size(ctypes.byref(p)) >= 256 + 4 * 1000
    assert lib.kda_forward_workspace_size(None) == 0
    assert lib.kda_forward_workspace_size(ctypes.byref(_params(Dk=96))) == 0


FAKE = 0x10000  # 16-byte aligned non-null address; never dereferenced on these paths


def _fwd(lib, p, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=FAKE, out=FAKE,
                Sf=None, ws=0x20000, ws_bytes=1 << 20)
    args.update(over)
    vp = ctypes.c_void_p
    return lib.kda_forward(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["la"]),
                           vp(args["beta"]), vp(args["S0"]), vp(args["cu"]), vp(args["out"]),
                           vp(args["Sf"]), ctypes.byref(p), vp(args["ws"]), args["ws_bytes"], None)


@pytest.mark.parametrize("over,params,code", [
    (dict(q=None), {}, 1),
    (dict(cu=None), {}, 1),
    (dict(out=None), {}, 1),
    ({}, dict(H=0), 1),
    ({}, dict(num_seqs=-1), 1),
    ({}, dict(flags=8), 1),
    ({}, dict(Dk=96), 2),
    ({}, dict(Dv=256), 2),
    ({}, dict(chunk=32), 2),
    ({}, dict(io_dtype=5), 2),
    (dict(q=FAKE + 4), {}, 3),
    (dict(S0=FAKE + 8), {}, 3),
    (dict(ws=None), {}, 4),
    (dict(ws=0x20010), {}, 4),
    (dict(ws_bytes=16), {}, 4),
])
def test_forward_host_validation(over, params, code):
    lib = kda.load_library()
    assert _fwd(lib, _params(**params), **over) == code


def test_forward_empty_problem_is_noop():
    lib = kda.load_library()
    assert _fwd(lib, _params(num_seqs=0, total_tokens=0), q=None, cu=None, out=None, ws=None) == 0
    assert _fwd(lib, _params(num_seqs=0, total_tokens=5)) == 1


def test_decode_host_validation():
    lib = kda.load_library()
    vp = ctypes.c_void_p
    call = lambda p, **o: lib.kda_decode_step(*(vp(o.get(n, FAKE)) for n in
                                                ("q", "k", "v", "la", "b", "S", "out")),
                                              ctypes.byref(p), None)
    assert call(_params(Dk=32)) == 2
    assert call(_params(), S=None) == 1
    assert call(_params(), out=FAKE + 2) == 3
    assert call(_params(num_seqs=0)) == 0


def test_workspace_status_null_args():
    lib = kda.load_library()
    st = ctypes.c_int32(0)
    assert lib.kda_workspace_status(None, ctypes.byref(st), None) == 1


def _fwd_snap(lib, p, every=512, pool=FAKE, base=FAKE, s0=None, n_slots=8, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=FAKE, out=FAKE,
                Sf=None, ws=0x20000, ws_bytes=1 << 20)
    args.update(over)
    vp = ctypes.c_void_p
    snap = kda.Snapshots(vp(pool) if pool else None, vp(base) if base else None,
                         vp(s0) if s0 else None, n_slots, every)
    return lib.kda_forward_snapshots(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["la"]),
                                     vp(args["beta"]), vp(args["S0"]), vp(args["cu"]),
                                     vp(args["out"]), vp(args["Sf"]), ctypes.byref(p),
                                     ctypes.byref(snap), vp(args["ws"]), args["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(every=100), 1),            # not a multiple of the chunk
    (dict(every=-64), 1),
    (dict(pool=None), 1),
    (dict(base=None), 1),            # snapshots requested without slot bases
    (dict(n_slots=0), 1),
    (dict(every=0, s0=FAKE, pool=None), 1),
    (dict(pool=FAKE + 4), 3),        # pool not 16-byte aligned
    (dict(q=None), 1),               # the forward's own checks still apply
])
def test_forward_snapshots_host_validation(kw, code):
    lib = kda.load_library()
    assert _fwd_snap(lib, _params(), **kw) == code


def test_decode_multi_host_validation():
    lib = kda.load_library()
    vp = ctypes.c_void_p
    call = lambda p, n=4, **o: lib.kda_decode_multi(*(vp(o.get(x, FAKE)) for x in
                                                      ("q", "k", "v", "la", "b", "S", "St", "out")),
                                                    ctypes.byref(p), n, None)
    assert call(_params(), n=0) == 1
    assert call(_params(), St=None) == 1
    assert call(_params(), S=None) == 1
    assert call(_params(), St=FAKE + 4) == 3
    assert call(_params(Dk=32)) == 2
    assert call(_params(num_seqs=0)) == 0


def _bwd(lib, p, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=FAKE, do=FAKE, dSf=None,
                dq=FAKE, dk=FAKE, dv=FAKE, dla=FAKE, db=FAKE, dS0=None, ws=0x20000,
                ws_bytes=1 << 40)
    args.update(over)
    vp = ctypes.c_void_p
    names = ("q", "k", "v", "la", "beta", "S0", "cu", "do", "dSf", "dq", "dk", "dv", "dla", "db",
             "dS0")
    return lib.kda_backward(*(vp(args[n]) for n in names), ctypes.byref(p), vp(args["ws"]),
                            args["ws_bytes"], None)


@pytest.mark.parametrize("over,params,code", [
    (dict(q=None), {}, 1),
    (dict(do=None), {}, 1),
    (dict(db=None), {}, 1),
    (dict(cu=None), {}, 1),
    ({}, dict(Dk=96), 2),
    ({}, dict(chunk=32), 2),
    (dict(dq=FAKE + 4), {}, 3),
    (dict(dS0=FAKE + 8), {}, 3),
    (dict(ws=None), {}, 4),
    (dict(ws=0x20010), {}, 4),
    (dict(ws_bytes=16), {}, 4),
])
def test_backward_host_validation(over, params, code):
    lib = kda.load_library()
    assert _bwd(lib, _params(**params), **over) == code


def test_backward_workspace_size():
    lib = kda.load_library()
    p = _params(flags=1)   # the fp32 CUDA-core backward
    n = lib.kda_backward_workspace_size(ctypes.byref(p))
    # the kept states, the per-CTA scratch and the per-slice partial sums
    T, N, H, Dk, Dv = p.total_tokens, p.num_seqs, p.H, p.Dk, p.Dv
    states = 2 * ((T + 63) // 64 + N) * H * Dk * Dv * 4          # one every 32 tokens
    scratch = N * H * (Dv // 32) * (32 * Dk * 32 + 32 * 32) * 4
    part = (Dv // 32) * T * H * (3 * Dk + 1) * 4
    assert states + scratch + part <= n <= states + scratch + part + 4096 + 8 * N + 256 * Dv
    assert lib.kda_backward_workspace_size(ctypes.byref(_params(Dk=96))) == 0
    assert lib.kda_backward_workspace_size(None) == 0


def test_chunk_offset_scan_saturates_instead_of_wrapping():
    """The varlen index counts the chunks of every well-formed (start, end)
    pair of cu_seqlens.  With overlapping (malformed) offsets the pairs need
    not tile the token axis, so the count can pass 2^31: 32768 pairs, every
    other one spanning [0, 2^24), give 2^14 * 2^18 = 2^32 chunks.  A 32-bit
    running sum wraps there (to 0 here, negative on the way), which the chain
    kernel's bound check of g0 + nchunks against the packet count would not
    catch; the kernel's 64-bit sum stored saturated at INT32_MAX always fails
    that check.  This restates the kernel's scan in numpy at that size."""
    T = 1 << 24
    cu = np.tile(np.array([0, T], dtype=np.int64), 1 << 14)
    cu = np.append(cu, 0)                         # 32768 pairs, every other one [0, T)
    a, b = cu[:-1], cu[1:]
    ok = (a >= 0) & (b >= a) & (b <= T)
    chunks = np.where(ok, (b - a + 63) // 64, 0)
    run64 = np.concatenate([[0], np.cumsum(chunks)])
    assert run64[-1] == 1 << 32
    wrapped = run64.astype(np.uint64).astype(np.uint32).astype(np.int32)
    assert (wrapped < 0).any() and wrapped[-1] == 0   # what an int32 scan would store
    stored = np.minimum(run64, 2**31 - 1).astype(np.int32)
    H, slots = 1, ((T + 63) // 64 + len(a)) * 1     # packets the workspace holds
    n_chunks = chunks
    g0 = stored[:-1]
    rejected = (g0 < 0) | ((g0.astype(np.int64) + n_chunks) * H > slots)
    # every sequence whose offset passed the workspace is rejected, none wraps back in
    assert rejected[ok & (run64[:-1] + n_chunks > slots)].all()
    assert (stored >= 0).all()


def test_chunked_backward_workspace_size():
    """bf16 with d_k = d_v = 128: the chunked tensor-core backward keeps the
    forward's operand packets and two fp32 states (the state entering the
    chunk and the gradient reaching it) per (chunk, head)."""
    lib = kda.load_library()
    p = _params()
    n = lib.kda_backward_workspace_size(ctypes.byref(p))
    T, N, H = p.total_tokens, p.num_seqs, p.H
    slots = ((T + 63) // 64 + N) * H
    need = slots * (66048 + 2 * 128 * 128 * 4)
    assert need <= n <= need + 4096 + 8 * N
