"""Kimi Delta Attention (KDA) on B200 (sm_100a): Python binding of libkda.so.

The library's C ABI is declared in ``include/kda.h``; this module only
marshals torch tensors into device pointers and the current CUDA stream.
Every step of the computation runs in the library's CUDA kernels; there is
no CPU or PyTorch fallback, and calls raise if the library cannot be
loaded.

    out, S_final = forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None)
    out = decode_step(q, k, v, log_alpha, beta, S)      # S updated in place
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["backward", "backward_workspace_size", "decode_multi", "forward", "decode_step", "forward_workspace_size", "workspace_status",
           "KDAError", "load_library", "LIB_PATH", "EXPORTED_SYMBOLS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")
EXPORTED_SYMBOLS = ("kda_forward_workspace_size", "kda_forward", "kda_forward_snapshots",
                    "kda_forward_noalloc", "kda_forward_noalloc_status", "kda_decode_step", "kda_decode_multi",
                    "kda_backward_workspace_size", "kda_backward", "kda_workspace_status",
                    "kda_status_string", "kda_abi_version")

KDA_F32, KDA_BF16 = 0, 1
FLAG_FORCE_SIMT = 1
FLAG_FUSED_TC = 2
CHUNK = 64

_lock = threading.Lock()
_lib = None


class KDAError(RuntimeError):
    pass


class Snapshots(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("slot_base", ctypes.c_void_p),
                ("s0_slot", ctypes.c_void_p), ("n_slots", ctypes.c_int64),
                ("every", ctypes.c_int32)]


class Params(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("H", ctypes.c_int32), ("Dk", ctypes.c_int32), ("Dv", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("io_dtype", ctypes.c_int32),
                ("gate_dtype", ctypes.c_int32), ("flags", ctypes.c_int32)]


def load_library(path: str = LIB_PATH):
    """Load libkda.so (building it with nvcc if it is absent) and declare signatures."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            from . import build as _build
            _build.build()
        if not os.path.exists(path):
            raise KDAError(f"KDA CUDA library not found at {path}")
        lib = ctypes.CDLL(path)
        vp, sz, pp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Params)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.kda_forward_workspace_size.restype = sz
        lib.kda_forward_workspace_size.argtypes = [pp]
        lib.kda_forward.restype = ctypes.c_int
        lib.kda_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
        lib.kda_forward_snapshots.restype = ctypes.c_int
        lib.kda_forward_snapshots.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, pp,
                                              ctypes.POINTER(Snapshots), vp, sz, vp]
        lib.kda_decode_step.restype = ctypes.c_int
        lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, pp, vp]
        lib.kda_decode_multi.restype = ctypes.c_int
        lib.kda_decode_multi.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, pp, ctypes.c_int32, vp]
        lib.kda_backward_workspace_size.restype = sz
        lib.kda_backward_workspace_size.argtypes = [pp]
        lib.kda_backward.restype = ctypes.c_int
        lib.kda_backward.argtypes = [vp] * 15 + [pp, vp, sz, vp]
        lib.kda_workspace_status.restype = ctypes.c_int
        lib.kda_workspace_status.argtypes = [vp, i32p, vp]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_abi_version.restype = ctypes.c_int32
        lib.kda_abi_version.argtypes = []
        if path == LIB_PATH:
            _lib = lib
        return lib


def _check(rc: int):
    if rc != 0:
        raise KDAError(load_library().kda_status_string(rc).decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KDA_F32
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    raise KDAError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require(tensors, device):
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda or t.device != device:
            raise KDAError(f"{name} must be a CUDA tensor on {device}")
        if not t.is_contiguous():
            raise KDAError(f"{name} must be contiguous")


def forward_workspace_size(N: int, T: int, H: int, Dk: int, Dv: int,
                           io_dtype=torch.bfloat16, gate_dtype=None) -> int:
    gd = io_dtype if gate_dtype is None else gate_dtype
    p = Params(N, T, H, Dk, Dv, CHUNK, KDA_F32 if io_dtype == torch.float32 else KDA_BF16,
               KDA_F32 if gd == torch.float32 else KDA_BF16, 0)
    return int(load_library().kda_forward_workspace_size(ctypes.byref(p)))


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, out=None, S_final=None,
            workspace=None, output_final_state=True, force_simt=False, fused_tc=False,
            snapshot_pool=None, snapshot_slot_base=None, snapshot_every=0, s0_slots=None):
    """Chunked KDA prefill through ``kda_forward`` (``kda_forward_snapshots``
    when a snapshot pool is given).

    q, k, log_alpha [T, H, Dk]; v [T, H, Dv]; beta [T, H]; S0 [N, H, Dk, Dv]
    fp32 or None; cu_seqlens int32 [N+1] on the device (None: one sequence).
    Returns (out [T, H, Dv] in q's dtype, S_final [N, H, Dk, Dv] fp32 or None).
    ``force_simt`` / ``fused_tc`` select the CUDA-core or the single-kernel
    tensor-core prefill instead of the default (for cross-checks).

    Prefix-cache snapshots: ``snapshot_pool`` fp32 [n_slots, H, Dk, Dv];
    every ``snapshot_every`` tokens of sequence n the state goes to slot
    ``snapshot_slot_base[n]`` + m (int32 [N]); ``s0_slots`` (int32 [N]) starts
    sequences from pool slots (negative: from S0).
    """
    lib = load_library()
    dev = q.device
    T, H, Dk = q.shape
    Dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=dev)
    if cu_seqlens.dtype != torch.int32:
        raise KDAError("cu_seqlens must be int32")
    N = cu_seqlens.numel() - 1
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != (T, H) \
            or beta.shape != (T, H):
        raise KDAError("shape mismatch among q, k, v, log_alpha, beta")
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != log_alpha.dtype:
        raise KDAError("q, k, v must share a dtype; log_alpha and beta must share a dtype")
    if S0 is not None and (S0.dtype != torch.float32 or S0.shape != (N, H, Dk, Dv)):
        raise KDAError("S0 must be float32 [N, H, Dk, Dv]")
    if out is None:
        out = torch.empty((T, H, Dv), dtype=q.dtype, device=dev)
    if S_final is None and output_final_state:
        S_final = torch.empty((N, H, Dk, Dv), dtype=torch.float32, device=dev)
    p = Params(N, T, H, Dk, Dv, CHUNK, _dt(q), _dt(log_alpha),
               (FLAG_FORCE_SIMT if force_simt else 0) | (FLAG_FUSED_TC if fused_tc else 0))
    ws_bytes = int(lib.kda_forward_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    _require(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0, cu_seqlens=cu_seqlens,
                  out=out, S_final=S_final, workspace=workspace, snapshot_pool=snapshot_pool,
                  snapshot_slot_base=snapshot_slot_base, s0_slots=s0_slots), dev)
    if snapshot_pool is None:
        with torch.cuda.device(dev):
            _check(lib.kda_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                   _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_final),
                                   ctypes.byref(p), _ptr(workspace), workspace.numel(),
                                   _stream(dev)))
        return out, S_final
    if snapshot_pool.dtype != torch.float32 or tuple(snapshot_pool.shape[1:]) != (H, Dk, Dv):
        raise KDAError("snapshot_pool must be float32 [n_slots, H, Dk, Dv]")
    for name, t in (("snapshot_slot_base", snapshot_slot_base), ("s0_slots", s0_slots)):
        if t is not None and (t.dtype != torch.int32 or t.numel() != N):
            raise KDAError(f"{name} must be int32 [N]")
    snap = Snapshots(_ptr(snapshot_pool), _ptr(snapshot_slot_base), _ptr(s0_slots),
                     int(snapshot_pool.shape[0]), int(snapshot_every))
    with torch.cuda.device(dev):
        _check(lib.kda_forward_snapshots(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                         _ptr(S0), _ptr(cu_seqlens), _ptr(out), _ptr(S_final),
                                         ctypes.byref(p), ctypes.byref(snap), _ptr(workspace),
                                         workspace.numel(), _stream(dev)))
    return out, S_final


def workspace_status(workspace) -> int:
    """Synchronise the current stream and return the workspace's device status code."""
    lib = load_library()
    st = ctypes.c_int32(-1)
    _check(lib.kda_workspace_status(_ptr(workspace), ctypes.byref(st), _stream(workspace.device)))
    return int(st.value)


def decode_step(q, k, v, log_alpha, beta, S, *, out=None):
    """One recurrent KDA token through ``kda_decode_step``; S is updated in place.

    q, k, log_alpha [N, H, Dk]; v [N, H, Dv]; beta [N, H]; S [N, H, Dk, Dv] fp32.
    Returns out [N, H, Dv] in q's dtype.
    """
    lib = load_library()
    dev = q.device
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    if S.dtype != torch.float32 or S.shape != (N, H, Dk, Dv):
        raise KDAError("S must be float32 [N, H, Dk, Dv]")
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != (N, H) \
            or beta.shape != (N, H):
        raise KDAError("shape mismatch among q, k, v, log_alpha, beta")
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != log_alpha.dtype:
        raise KDAError("q, k, v must share a dtype; log_alpha and beta must share a dtype")
    if out is None:
        out = torch.empty((N, H, Dv), dtype=q.dtype, device=dev)
    _require(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S=S, out=out), dev)
    p = Params(N, 0, H, Dk, Dv, CHUNK, _dt(q), _dt(log_alpha), 0)
    with torch.cuda.device(dev):
        _check(lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                   _ptr(S), _ptr(out), ctypes.byref(p), _stream(dev)))
    return out


def decode_multi(q, k, v, log_alpha, beta, S, *, S_tokens=None, out=None):
    """Several consecutive KDA tokens per sequence through ``kda_decode_multi``.

    q, k, log_alpha [N, n, H, Dk]; v [N, n, H, Dv]; beta [N, n, H];
    S [N, H, Dk, Dv] fp32 (read only).  Returns (out [N, n, H, Dv] in q's
    dtype, S_tokens [N, n, H, Dk, Dv] fp32: the state after every token).
    """
    lib = load_library()
    dev = q.device
    N, n, H, Dk = q.shape
    Dv = v.shape[-1]
    if S.dtype != torch.float32 or S.shape != (N, H, Dk, Dv):
        raise KDAError("S must be float32 [N, H, Dk, Dv]")
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:3] != (N, n, H) \
            or beta.shape != (N, n, H):
        raise KDAError("shape mismatch among q, k, v, log_alpha, beta")
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != log_alpha.dtype:
        raise KDAError("q, k, v must share a dtype; log_alpha and beta must share a dtype")
    if out is None:
        out = torch.empty((N, n, H, Dv), dtype=q.dtype, device=dev)
    if S_tokens is None:
        S_tokens = torch.empty((N, n, H, Dk, Dv), dtype=torch.float32, device=dev)
    _require(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S=S, S_tokens=S_tokens,
                  out=out), dev)
    p = Params(N, 0, H, Dk, Dv, CHUNK, _dt(q), _dt(log_alpha), 0)
    with torch.cuda.device(dev):
        _check(lib.kda_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                    _ptr(S), _ptr(S_tokens), _ptr(out), ctypes.byref(p), int(n),
                                    _stream(dev)))
    return out, S_tokens


def backward_workspace_size(N: int, T: int, H: int, Dk: int, Dv: int,
                            dtype=torch.bfloat16, force_simt=False) -> int:
    """Bytes of device workspace ``kda_backward`` needs for this problem (the
    chunked tensor-core path for bf16 with Dk = Dv = 128, unless ``force_simt``)."""
    d = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    p = Params(N, T, H, Dk, Dv, CHUNK, d, d, FLAG_FORCE_SIMT if force_simt else 0)
    return int(load_library().kda_backward_workspace_size(ctypes.byref(p)))


def backward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, d_out, dS_final=None,
             need_dS0=True, workspace=None, force_simt=False):
    """Gradients through ``kda_backward`` of a loss with dL/d out = ``d_out``
    (and dL/dS_final = ``dS_final``, None: zero).

    Inputs as ``forward``.  Returns a dict of fp32 tensors: dq, dk, dlog_alpha
    [T, H, Dk], dv [T, H, Dv], dbeta [T, H] and dS0 [N, H, Dk, Dv] (None when
    ``need_dS0`` is false).  bf16 inputs with Dk = Dv = 128 take the chunked
    tensor-core backward; ``force_simt`` selects the fp32 CUDA-core one.
    """
    lib = load_library()
    dev = q.device
    T, H, Dk = q.shape
    Dv = v.shape[-1]
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=dev)
    if cu_seqlens.dtype != torch.int32:
        raise KDAError("cu_seqlens must be int32")
    N = cu_seqlens.numel() - 1
    if k.shape != q.shape or log_alpha.shape != q.shape or v.shape[:2] != (T, H) \
            or beta.shape != (T, H) or d_out.shape != v.shape:
        raise KDAError("shape mismatch among q, k, v, log_alpha, beta, d_out")
    if k.dtype != q.dtype or v.dtype != q.dtype or d_out.dtype != q.dtype \
            or beta.dtype != log_alpha.dtype:
        raise KDAError("q, k, v, d_out must share a dtype; log_alpha and beta must share a dtype")
    for name, x in (("S0", S0), ("dS_final", dS_final)):
        if x is not None and (x.dtype != torch.float32 or x.shape != (N, H, Dk, Dv)):
            raise KDAError(f"{name} must be float32 [N, H, Dk, Dv]")
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"dq": torch.empty((T, H, Dk), **f32), "dk": torch.empty((T, H, Dk), **f32),
         "dv": torch.empty((T, H, Dv), **f32), "dlog_alpha": torch.empty((T, H, Dk), **f32),
         "dbeta": torch.empty((T, H), **f32),
         "dS0": torch.empty((N, H, Dk, Dv), **f32) if need_dS0 else None}
    p = Params(N, T, H, Dk, Dv, CHUNK, _dt(q), _dt(log_alpha),
               FLAG_FORCE_SIMT if force_simt else 0)
    ws_bytes = int(lib.kda_backward_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    _require(dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0, cu_seqlens=cu_seqlens,
                  d_out=d_out, dS_final=dS_final, workspace=workspace, **g), dev)
    with torch.cuda.device(dev):
        _check(lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                _ptr(S0), _ptr(cu_seqlens), _ptr(d_out), _ptr(dS_final),
                                _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dS0"]),
                                ctypes.byref(p), _ptr(workspace), workspace.numel(),
                                _stream(dev)))
    return g
