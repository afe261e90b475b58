"""fp64 CPU oracle for Kimi Delta Attention (KDA) -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library and never imports it; both sides receive the same arrays from the
seeded input generator and nothing else.

Contents
  * ``forward`` / ``decode_step`` -- the token-by-token recurrence in plain C
    (``kda_oracle.c``), fp64, no FMA contraction, threaded over independent
    (sequence, head) chains.
  * ``backward`` -- the gradients of a loss through that recurrence, the
    forward steps differentiated in reverse order (``kda_oracle_bwd.c``).
  * ``chunked.forward_chunked`` -- an fp64 numpy restatement of the same
    recurrence in chunk form, used only to pin the chunk algebra that the
    GPU kernels rely on (tests compare it with ``forward``);
    ``chunked.backward_chunked`` takes reverse mode through that chunk
    algebra (tests compare it with ``backward``).
  * ``exact.unrolled_product`` -- the recurrence written as an explicit
    product of transition matrices in exact rational arithmetic, for tiny
    inputs (pins ``forward`` to the definition itself).

The recurrence (page "Kimi K3: Open Frontier Intelligence and Implementation
Framework", section "Hybrid Attention Mechanism", KDA bullet: a delta-rule
recurrence with a channel-wise, lower-bounded forget gate):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t,          alpha_t = exp(log_alpha_t)  (per channel)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_SRC_BWD = os.path.join(_HERE, "kda_oracle_bwd.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

# Plain C, IEEE double: no contraction into FMA, no fast-math.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
          "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` and ``kda_oracle_bwd.c`` with gcc into one
    library under ``oracle/_build``; return its path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                                  os.path.getmtime(_SRC_BWD)))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, _SRC_BWD, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load a compiled oracle library from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.kda_oracle_forward.restype = ctypes.c_int
    lib.kda_oracle_forward.argtypes = [
        i64, ctypes.POINTER(i64), i64, i64, i64,
        dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
    lib.kda_oracle_forward_snapshots.restype = ctypes.c_int
    lib.kda_oracle_forward_snapshots.argtypes = [
        i64, ctypes.POINTER(i64), i64, i64, i64,
        dp, dp, dp, dp, dp, dp, dp, dp, i64, ctypes.POINTER(i64), dp, ctypes.c_int]
    lib.kda_oracle_decode_step.restype = ctypes.c_int
    lib.kda_oracle_decode_step.argtypes = [
        i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
    if hasattr(lib, "kda_oracle_backward"):   # builds of the forward source alone lack it
        bind_backward(lib)
    return lib


def bind_backward(lib):
    """Declare the backward entry point on a loaded library (ctypes.CDLL or path)."""
    if isinstance(lib, str):
        lib = ctypes.CDLL(lib)
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.kda_oracle_backward.restype = ctypes.c_int
    lib.kda_oracle_backward.argtypes = [
        i64, ctypes.POINTER(i64), i64, i64, i64,
        dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(build())
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _f64(x) -> np.ndarray:
    """Contiguous float64 copy/view of an array-like (torch tensors included)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, threads=None, lib=None,
            snapshot_every=None):
    """Token-by-token fp64 KDA over packed sequences.

    Shapes: q, k, log_alpha [T_tot, H, Dk]; v [T_tot, H, Dv]; beta [T_tot, H];
    S0 [N, H, Dk, Dv] or None (zero); cu_seqlens int [N+1] or None (one
    sequence of length T_tot).  Returns (out [T_tot, H, Dv], S_final
    [N, H, Dk, Dv]) as float64 arrays.  ``lib`` (tests only) substitutes
    another build of the same C source.

    With ``snapshot_every`` = E > 0 it returns (out, S_final, snaps, snap_off):
    snaps [M, H, Dk, Dv] holds the state of every chain right after each
    E-th token of its sequence (page "Kimi K3: Open Frontier Intelligence and
    Implementation Framework", section "Inference Serving", KDA-aware prefix
    caching), sequence n's m-th one (m = 0, 1, ...) at index snap_off[n] + m,
    with snap_off the exclusive prefix sum of floor(len_n / E).
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    if k.shape != (T, H, Dk) or la.shape != (T, H, Dk):
        raise ValueError("q, k, log_alpha must share the shape [T, H, Dk]")
    if v.shape[:2] != (T, H) or b.shape != (T, H):
        raise ValueError("v must be [T, H, Dv] and beta [T, H]")
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if N < 0 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T")
    s0 = None
    if S0 is not None:
        s0 = _f64(S0)
        if s0.shape != (N, H, Dk, Dv):
            raise ValueError("S0 must be [N, H, Dk, Dv]")
    out = np.zeros((T, H, Dv), dtype=np.float64)
    sf = np.zeros((N, H, Dk, Dv), dtype=np.float64)
    if snapshot_every is None:
        rc = (lib or _load()).kda_oracle_forward(
            N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, Dk, Dv,
            _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(out),
            _ptr(sf), int(threads or default_threads()))
        if rc != 0:
            raise RuntimeError(f"kda_oracle_forward failed with code {rc}")
        return out, sf
    E = int(snapshot_every)
    if E <= 0:
        raise ValueError("snapshot_every must be positive")
    counts = np.diff(cu) // E
    snap_off = np.ascontiguousarray(np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int64)
                                    if N > 0 else np.zeros(0, dtype=np.int64))
    # Guard slots past the end: the mutation tests run deliberately broken
    # builds of this C source in-process, and a snapshot written one slot too
    # far must land in memory this array owns.
    M = int(counts.sum())
    snaps_buf = np.zeros((M + 4, H, Dk, Dv), dtype=np.float64)
    snaps = snaps_buf[:M]
    rc = (lib or _load()).kda_oracle_forward_snapshots(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, Dk, Dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(out),
        _ptr(sf), E, snap_off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(snaps_buf) if M else None, int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_forward_snapshots failed with code {rc}")
    return out, sf, snaps, snap_off


def decode_step(q, k, v, log_alpha, beta, S, threads=None):
    """One recurrent step for N sequences: returns (out [N,H,Dv], S_new)."""
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    s = _f64(S).copy()
    N, H, Dk = q.shape
    Dv = v.shape[2]
    if s.shape != (N, H, Dk, Dv):
        raise ValueError("S must be [N, H, Dk, Dv]")
    out = np.zeros((N, H, Dv), dtype=np.float64)
    rc = _load().kda_oracle_decode_step(
        N, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s),
        _ptr(out), int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_decode_step failed with code {rc}")
    return out, s


def backward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, d_out=None, dS_final=None,
             threads=None, lib=None):
    """fp64 gradients of a loss L through the recurrence (``kda_oracle_bwd.c``).

    Inputs as ``forward``; d_out [T_tot, H, Dv] = dL/d out; dS_final
    [N, H, Dk, Dv] = dL/dS_final or None (zero).  Returns a dict with dq, dk,
    dlog_alpha [T_tot, H, Dk], dv [T_tot, H, Dv], dbeta [T_tot, H] and dS0
    [N, H, Dk, Dv], all float64.  ``lib`` (tests only) substitutes another
    build of the backward source.
    """
    q, k, v, la, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_out))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    if k.shape != (T, H, Dk) or la.shape != (T, H, Dk):
        raise ValueError("q, k, log_alpha must share the shape [T, H, Dk]")
    if v.shape[:2] != (T, H) or b.shape != (T, H) or do.shape != (T, H, Dv):
        raise ValueError("v and d_out must be [T, H, Dv] and beta [T, H]")
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if N < 0 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T")
    s0 = None if S0 is None else _f64(S0)
    dsf = None if dS_final is None else _f64(dS_final)
    for name, x in (("S0", s0), ("dS_final", dsf)):
        if x is not None and x.shape != (N, H, Dk, Dv):
            raise ValueError(f"{name} must be [N, H, Dk, Dv]")
    g = {"dq": np.zeros((T, H, Dk)), "dk": np.zeros((T, H, Dk)), "dv": np.zeros((T, H, Dv)),
         "dlog_alpha": np.zeros((T, H, Dk)), "dbeta": np.zeros((T, H)),
         "dS0": np.zeros((N, H, Dk, Dv))}
    rc = (lib or _load()).kda_oracle_backward(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, Dk, Dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(do), _ptr(dsf),
        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]),
        _ptr(g["dS0"]), int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_backward failed with code {rc}")
    return g
