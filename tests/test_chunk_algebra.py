"""The operand algebra of the two-pass prefill, checked in fp64 on the CPU
against the token-by-token oracle.

Pass 1 turns each chunk of 64 tokens (any L rows here) into a packet that
does not depend on the state; pass 2 walks the chunks of a chain in order.
Writing Gam_r for the in-chunk running decay, Qg = Q Gam, Kg = K Gam,
Ki = K / Gam, A = strict_lower(diag(b) Kg Ki^T), T = (I + A)^{-1},
Tb = T diag(b), W = Tb Kg, P = lower_incl(Qg Ki^T):

  packet   [-W; Qe] with Qe = Qg - P W,   Ki,   [Tb; PT] with PT = P Tb,   Gam_L
  chain    [U; O] = [Tb; PT] V + [-W; Qe] S      (U = Tb V - W S, O = Qg S + P U)
           S' = Diag(Gam_L) (S + Ki^T U)

This is a restatement of the chunk form for the recurrence of the page
"Kimi K3: Open Frontier Intelligence and Implementation Framework" (section
"Hybrid Attention Mechanism", KDA bullet); the test holds the kernels'
rearrangement to the definition, independently of any GPU.
"""
import math

import numpy as np
import pytest
from scipy.linalg import solve_triangular

import oracle


def _packet(Q, K, LA, b):
    L = Q.shape[0]
    g = np.cumsum(LA, axis=0)
    Gam = np.exp(g)
    Qg, Kg, Ki = Q * Gam, K * Gam, K / Gam
    A = np.tril(b[:, None] * (Kg @ Ki.T), k=-1)
    T = solve_triangular(np.eye(L) + A, np.eye(L), lower=True, unit_diagonal=True)
    Tb = T * b[None, :]
    W = Tb @ Kg
    P = np.tril(Qg @ Ki.T)
    return dict(mW=-W, Qe=Qg - P @ W, Ki=Ki, Tb=Tb, PT=P @ Tb, GL=Gam[-1])


def _chain_step(pk, S, V):
    top = np.vstack([pk["Tb"], pk["PT"]]) @ V + np.vstack([pk["mW"], pk["Qe"]]) @ S
    L = V.shape[0]
    U, O = top[:L], top[L:]
    S_next = pk["GL"][:, None] * (S + pk["Ki"].T @ U)
    return O, S_next


def _two_pass(q, k, v, la, beta, S0, cu, C):
    T, H, Dk = q.shape
    Dv = v.shape[2]
    out = np.zeros((T, H, Dv))
    Sf = np.zeros((len(cu) - 1, H, Dk, Dv))
    for n in range(len(cu) - 1):
        for h in range(H):
            S = S0[n, h].copy()
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(c0 + C, cu[n + 1])
                sl = slice(c0, c1)
                pk = _packet(q[sl, h], k[sl, h], la[sl, h], beta[sl, h])
                out[sl, h], S = _chain_step(pk, S, v[sl, h])
            Sf[n, h] = S
    return out, Sf


@pytest.mark.parametrize("C,alpha_min,seed", [(64, 0.9, 0), (16, 0.5, 1), (7, 0.95, 2)])
def test_two_pass_algebra_matches_the_recurrence(C, alpha_min, seed):
    rng = np.random.default_rng(seed)
    lens = [150, 64, 1, 0, 97]
    T, H, Dk, Dv = sum(lens), 2, 8, 6
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    la = rng.uniform(math.log(alpha_min), 0.0, size=(T, H, Dk))
    S0 = 0.1 * rng.standard_normal((len(lens), H, Dk, Dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o_ref, s_ref = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu)
    o, s = _two_pass(q, k, v, la, beta, S0, cu, C)
    scale_o, scale_s = np.max(np.abs(o_ref)), np.max(np.abs(s_ref))
    assert np.max(np.abs(o - o_ref)) <= 1e-10 * scale_o
    assert np.max(np.abs(s - s_ref)) <= 1e-10 * scale_s


def test_packet_terms_have_their_defining_products():
    """PT is P Tb and Qe folds -P W into Qg, so O needs no product after U."""
    rng = np.random.default_rng(5)
    L, Dk, Dv = 12, 5, 4
    Q, K, V = rng.standard_normal((L, Dk)), rng.standard_normal((L, Dk)), rng.standard_normal((L, Dv))
    LA = rng.uniform(math.log(0.6), 0.0, size=(L, Dk))
    b = rng.uniform(0.1, 1.0, size=L)
    S = rng.standard_normal((Dk, Dv))
    pk = _packet(Q, K, LA, b)
    g = np.cumsum(LA, axis=0)
    Qg, Ki = Q * np.exp(g), K * np.exp(-g)
    P = np.tril(Qg @ Ki.T)
    U = pk["Tb"] @ V + pk["mW"] @ S
    O_direct = Qg @ S + P @ U
    O_packet, _ = _chain_step(pk, S, V)
    assert np.allclose(O_packet, O_direct, rtol=1e-12, atol=1e-12)
