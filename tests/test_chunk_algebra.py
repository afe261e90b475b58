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

The backward through the same packets (reverse chain on the transposed
packet operands, then chunk-parallel gradient assembly) is checked against
the backward oracle at the end of this file.

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


# ------------------------------------------------------------------ backward
# The gradients through the same packets.  With dS' = dL/dS_next and
# dS_pre = Diag(Gam_L) dS', the reverse chain needs only the forward packet,
# transposed:
#   dU_s = Ki dS_pre                              (state-dependent part of dU)
#   dS   = dS_pre + Qe^T dO + (-W)^T dU_s          (dL/d entering state)
# and the rest is chunk-parallel once dU_s and the entering state S are
# known:  dU = dU_s + P^T dO,  U = Tb V - W S,  then dQ, dK, dV, dbeta,
# dlog_alpha as in the chunk-form reverse mode.

def _assemble(S, U, dU, dSn, Q, K, V, LA, b, dO):
    """Chunk-parallel gradients given the entering state S, U, the full dU and
    dS' (reverse mode of the chunk form below the chain's two products)."""
    L = Q.shape[0]
    g = np.cumsum(LA, axis=0)
    eg, emg = np.exp(g), np.exp(-g)
    Kg, Ki, Qg = K * eg, K * emg, Q * eg
    M = Kg @ Ki.T
    A = np.tril(b[:, None] * M, k=-1)
    T = solve_triangular(np.eye(L) + A, np.eye(L), lower=True, unit_diagonal=True)
    bKg, bV = b[:, None] * Kg, b[:, None] * V
    W = T @ bKg
    gl = g[-1]
    ed = np.exp(gl[None, :] - g)
    dgl = np.sum(dSn * S, axis=1) * np.exp(gl)
    dKd = U @ dSn.T
    dK = dKd * ed
    d_ed = dKd * K * ed
    dgl = dgl + np.sum(d_ed, axis=0)
    dg = -d_ed
    dQg = dO @ S.T
    dP = np.tril(dO @ U.T)
    dQg = dQg + dP @ Ki
    dKi = dP.T @ Qg
    dW = -dU @ S.T
    dbV, dbKg = T.T @ dU, T.T @ dW
    dT = dU @ bV.T + dW @ bKg.T
    dV = b[:, None] * dbV
    db = np.sum(dbV * V, axis=1) + np.sum(dbKg * Kg, axis=1)
    dKg = b[:, None] * dbKg
    dA = np.tril(-T.T @ dT @ T.T, k=-1)
    db = db + np.sum(dA * M, axis=1)
    dM = b[:, None] * dA
    dKg = dKg + dM @ Ki
    dKi = dKi + dM.T @ Kg
    dQ = dQg * eg
    dK = dK + dKg * eg + dKi * emg
    dg = dg + dQg * Q * eg + dKg * K * eg - dKi * K * emg
    dg[-1] = dg[-1] + dgl
    dLA = np.cumsum(dg[::-1], axis=0)[::-1]
    return dQ, dK, dV, dLA, db


def _two_pass_backward(q, k, v, la, beta, S0, cu, dout, dSf, C):
    T, H, Dk = q.shape
    Dv = v.shape[2]
    grads = {n: np.zeros(s) for n, s in (("dq", (T, H, Dk)), ("dk", (T, H, Dk)),
                                         ("dv", (T, H, Dv)), ("dlog_alpha", (T, H, Dk)),
                                         ("dbeta", (T, H)))}
    dS0 = np.zeros((len(cu) - 1, H, Dk, Dv))
    for n in range(len(cu) - 1):
        for h in range(H):
            starts = list(range(cu[n], cu[n + 1], C))
            packets, entering, S = [], [], S0[n, h].copy()
            for c0 in starts:                         # forward: packets, entering states
                sl = slice(c0, min(c0 + C, cu[n + 1]))
                pk = _packet(q[sl, h], k[sl, h], la[sl, h], beta[sl, h])
                packets.append(pk)
                entering.append(S)
                _, S = _chain_step(pk, S, v[sl, h])
            dS = dSf[n, h].copy()
            for c0, pk, Sc in zip(reversed(starts), reversed(packets), reversed(entering)):
                sl = slice(c0, min(c0 + C, cu[n + 1]))
                dO = dout[sl, h]
                # reverse chain: the packet's operands, transposed
                dS_pre = pk["GL"][:, None] * dS
                dU_s = pk["Ki"] @ dS_pre
                dS_in = dS_pre + pk["Qe"].T @ dO + pk["mW"].T @ dU_s
                # chunk-parallel: U, the full dU, then the row gradients
                L = sl.stop - sl.start
                g = np.cumsum(la[sl, h], axis=0)
                P = np.tril((q[sl, h] * np.exp(g)) @ (k[sl, h] * np.exp(-g)).T)
                U = pk["Tb"] @ v[sl, h] + pk["mW"] @ Sc
                dU = dU_s + P.T @ dO
                dQ, dK, dV, dLA, db = _assemble(Sc, U, dU, dS, q[sl, h], k[sl, h], v[sl, h],
                                                la[sl, h], beta[sl, h], dO)
                grads["dq"][sl, h], grads["dk"][sl, h], grads["dv"][sl, h] = dQ, dK, dV
                grads["dlog_alpha"][sl, h], grads["dbeta"][sl, h] = dLA, db
                dS = dS_in
            dS0[n, h] = dS
    grads["dS0"] = dS0
    return grads


@pytest.mark.parametrize("C,alpha_min,seed", [(64, 0.9, 0), (16, 0.5, 1), (7, 0.95, 2)])
def test_backward_through_the_packets_matches_the_oracle(C, alpha_min, seed):
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
    dout = rng.standard_normal((T, H, Dv))
    dSf = rng.standard_normal((len(lens), H, Dk, Dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    ref = oracle.backward(q, k, v, la, beta, S0, cu, dout, dSf)
    got = _two_pass_backward(q, k, v, la, beta, S0, cu, dout, dSf, C)
    for name, r in ref.items():
        assert np.max(np.abs(got[name] - r)) <= 1e-9 * max(np.max(np.abs(r)), 1.0), name


# ------------------------------------------------------------ transfer form
# A re-association of the chain that leaves one short product per chunk on the
# path from one chunk to the next.  With Ks_j = Ki_j Diag(Gam_L,j) (keys decayed
# to the chunk's end) and X_{j+1} = W_{j+1} Ks_j^T (64 x 64):
#   U_{j+1} = U0_{j+1} - W_{j+1} (Diag(Gam_L,j) S_j) - X_{j+1} U_j
#   S_{j+1} = Diag(Gam_L,j) S_j + Ks_j^T U_j
# U_{j+1} needs S_j (one chunk old) and U_j through X_{j+1} only.

def _transfer_form(q, k, v, la, beta, S0, cu, C, rescaled_w=False):
    T, H, Dk = q.shape
    Dv = v.shape[2]
    out = np.zeros((T, H, Dv))
    Sf = np.zeros((len(cu) - 1, H, Dk, Dv))
    for n in range(len(cu) - 1):
        for h in range(H):
            starts = list(range(cu[n], cu[n + 1], C))
            S = S0[n, h].copy()
            pks, U = [], None
            for c0 in starts:
                sl = slice(c0, min(c0 + C, cu[n + 1]))
                pk = _packet(q[sl, h], k[sl, h], la[sl, h], beta[sl, h])
                pk["U0"], pk["V"] = pk["Tb"] @ v[sl, h], v[sl, h]
                pk["Ks"] = pk["Ki"] * pk["GL"][None, :]
                pks.append((sl, pk))
            for j, (sl, pk) in enumerate(pks):
                if j == 0:
                    U = pk["U0"] + pk["mW"] @ S
                out[sl, h] = pk["Qe"] @ S + pk["PT"] @ pk["V"]
                S_next = pk["GL"][:, None] * S + pk["Ks"].T @ U
                if j + 1 < len(pks):
                    nx = pks[j + 1][1]
                    if rescaled_w:
                        # the next packet's -W rescaled by this chunk's decay, per channel
                        mWp = nx["mW"] * pk["GL"][None, :]
                        U = nx["U0"] + mWp @ S + (mWp @ pk["Ki"].T) @ U
                    else:
                        X = -nx["mW"] @ pk["Ks"].T
                        U = nx["U0"] + nx["mW"] @ (pk["GL"][:, None] * S) - X @ U
                S = S_next
            Sf[n, h] = S
    return out, Sf


@pytest.mark.parametrize("rescaled_w", [False, True])
@pytest.mark.parametrize("C,alpha_min,seed", [(64, 0.9, 3), (16, 0.5, 4), (7, 0.95, 5)])
def test_transfer_form_matches_the_recurrence(C, alpha_min, seed, rescaled_w):
    """Both ways of writing it: with Ks, or with the next packet's W rescaled by
    this chunk's decay, W' = W Diag(Gam_L,j), so that X_{j+1} = W'_{j+1} Ki_j^T,
    U_{j+1} = U0_{j+1} - W'_{j+1} S_j - X_{j+1} U_j and the state update keeps
    its present form S_{j+1} = Diag(Gam_L,j) (S_j + Ki_j^T U_j)."""
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
    o, s = _transfer_form(q, k, v, la, beta, S0, cu, C, rescaled_w)
    assert np.max(np.abs(o - o_ref)) <= 1e-10 * np.max(np.abs(o_ref))
    assert np.max(np.abs(s - s_ref)) <= 1e-10 * np.max(np.abs(s_ref))
