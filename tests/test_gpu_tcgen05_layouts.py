"""GPU check of the tcgen05.mma operand layouts and descriptors (the
building blocks of the tensor-core prefill): a one-CTA probe stages bf16
A and B in each shared-memory layout the prefill uses, runs the MMAs into
TMEM and the result is compared with a float64 matmul of the same values."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = tmp_path_factory.mktemp("probe") / "libumma_probe.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC",
                    f"-I{ROOT}/gated_delta_rule_113_b200/csrc", f"-I{ROOT}/include",
                    "-o", str(out), os.path.join(HERE, "cuda", "umma_probe.cu")], check=True)
    lib = ctypes.CDLL(str(out))
    lib.umma_probe.restype = ctypes.c_int
    return lib


def _bf16(x):
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().astype(np.uint16), t.float().double().numpy()


def _run(lib, M, N, K, a_mn, b_mn, b_swz, neg_a=0, seed=0, a_tmem=0):
    rng = np.random.default_rng(seed)
    A_bits, A = _bf16(rng.standard_normal((M, K)))
    B_bits, B = _bf16(rng.standard_normal((K, N)))
    D = np.zeros((128, N), dtype=np.float32)
    p16 = ctypes.POINTER(ctypes.c_uint16)
    rc = lib.umma_probe(M, N, K, a_mn, b_mn, b_swz, neg_a, a_tmem,
                        np.ascontiguousarray(A_bits).ctypes.data_as(p16),
                        np.ascontiguousarray(B_bits).ctypes.data_as(p16),
                        D.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    assert rc == 0, f"probe returned {rc}"
    ref = (-1.0 if neg_a else 1.0) * (A @ B)
    if a_tmem:   # also the product with each column pair of A swapped
        Asw = A.reshape(M, K // 2, 2)[:, :, ::-1].reshape(M, K)
        return D.astype(np.float64), ref, Asw @ B
    return D.astype(np.float64), ref


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,b_swz,neg_a", [
    (128, 64, 128, 0, 0, 128, 0),    # [Kg;Qg] x Ki^T     (A, B K-major)
    (128, 128, 64, 0, 1, 128, 0),    # [Tb;0] x Kg        (B MN-major, two N blocks)
    (128, 32, 64, 0, 1, 64, 0),      # [Tb;0] x V  (32-wide value slice, 64B swizzle)
    (128, 64, 64, 0, 1, 128, 0),     # [Tb;0] x V  (64-wide value slice)
    (128, 32, 128, 0, 1, 64, 0),     # [-W;Qg] x S (32-wide slice)
    (128, 64, 128, 0, 1, 128, 1),    # negated A, 64-wide slice
    (128, 32, 64, 1, 1, 64, 0),      # Ki^T x U    (A MN-major)
    (128, 64, 64, 1, 1, 128, 0),     # Ki^T x U    (A MN-major, 64-wide slice)
])
def test_umma_layouts_m128(probe, M, N, K, a_mn, b_mn, b_swz, neg_a):
    D, ref = _run(probe, M, N, K, a_mn, b_mn, b_swz, neg_a)
    err = np.max(np.abs(D[:M] - ref)) / np.max(np.abs(ref))
    assert err < 1e-5, f"max rel err {err:.3e}"


def test_umma_m64_lane_layout(probe):
    """Where an M=64 result lands in TMEM (lanes 0-63, or 16 lanes per quarter)."""
    D, ref = _run(probe, 64, 64, 64, 0, 1, 128)
    dense = np.max(np.abs(D[:64] - ref)) / np.max(np.abs(ref))
    rows = np.concatenate([np.arange(32 * q, 32 * q + 16) for q in range(4)])
    split = np.max(np.abs(D[rows] - ref)) / np.max(np.abs(ref))
    print(f"M=64 layout: dense lanes 0-63 err {dense:.3e}; 16-per-quarter err {split:.3e}")
    assert min(dense, split) < 1e-5


@pytest.mark.parametrize("N,K,b_mn,b_swz", [
    (128, 128, 0, 128),   # S^T x [-W;Qe]^T  (B K-major, two K atoms)
    (128, 64, 1, 128),    # U^T x Ki          (B MN-major, two N blocks)
    (64, 64, 1, 128),
])
def test_umma_a_from_tensor_memory(probe, N, K, b_mn, b_swz):
    """A staged in tensor memory as packed bf16 pairs (lane = row, column j =
    elements 2j and 2j+1, the even one in the low half) for M = 128."""
    D, ref, ref_swapped = _run(probe, 128, N, K, 0, b_mn, b_swz, a_tmem=1)
    err = np.max(np.abs(D - ref)) / np.max(np.abs(ref))
    err_sw = np.max(np.abs(D - ref_swapped)) / np.max(np.abs(ref_swapped))
    print(f"A in TMEM: even-low err {err:.3e}, odd-low err {err_sw:.3e}")
    assert err < 1e-5, f"max rel err {err:.3e} (swapped pairs: {err_sw:.3e})"
