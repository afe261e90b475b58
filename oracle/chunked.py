"""fp64 chunk-form restatement of the KDA recurrence -- TEST INFRASTRUCTURE.

This module exists to pin the chunk algebra that a chunkwise-parallel
implementation relies on: the tests check that it reproduces the
token-by-token oracle (``oracle.forward``) for many chunk sizes, including
chunk sizes that do not divide the sequence length.  It is plain numpy in
float64 with one library triangular solve per chunk; nothing is fused or
reordered beyond the algebra below.

Derivation (from the recurrence of the page "Kimi K3: Open Frontier
Intelligence and Implementation Framework", section "Hybrid Attention
Mechanism", KDA bullet: delta rule with a channel-wise forget gate).

Per token, with D_r = Diag(alpha_r):
    S_r = D_r S_{r-1} + k_r u_r^T,   u_r = beta_r (v_r - (D_r S_{r-1})^T k_r).
Inside one chunk of rows r = 1..L that starts from state S, let
g_r = sum_{s<=r} log alpha_s (inclusive, per channel), Gam_r = exp(g_r).
Unrolling gives  D_r S_{r-1} = Diag(Gam_r) S + sum_{s<r} Diag(Gam_r/Gam_s) k_s u_s^T,
so with Kg = K*Gam, Ki = K/Gam, Qg = Q*Gam (row-wise, per channel):
    (I + A) U = diag(b) (V - Kg S),   A = strict_lower(diag(b) Kg Ki^T)
    T = (I + A)^{-1},  W = T diag(b) Kg,  U0 = T diag(b) V,  U = U0 - W S
    O = Qg S + lower_incl(Qg Ki^T) U
    S_next = Diag(Gam_L) S + (K * Gam_L/Gam)^T U
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _chunk(S, Q, K, V, LA, b):
    """One chunk of L rows starting from state S (Dk x Dv); returns (O, S_next)."""
    L = Q.shape[0]
    g = np.cumsum(LA, axis=0)                   # inclusive in-chunk log decay
    Kg = K * np.exp(g)
    Ki = K * np.exp(-g)
    Qg = Q * np.exp(g)
    A = np.tril(b[:, None] * (Kg @ Ki.T), k=-1)
    I = np.eye(L)
    # T = (I + A)^{-1} applied to diag(b) Kg and diag(b) V (unit lower triangular)
    W = solve_triangular(I + A, b[:, None] * Kg, lower=True, unit_diagonal=True)
    U0 = solve_triangular(I + A, b[:, None] * V, lower=True, unit_diagonal=True)
    U = U0 - W @ S
    P = np.tril(Qg @ Ki.T)
    O = Qg @ S + P @ U
    Kd = K * np.exp(g[-1][None, :] - g)
    S_next = np.exp(g[-1])[:, None] * S + Kd.T @ U
    return O, S_next


def forward_chunked(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, chunk=64):
    """Same contract as ``oracle.forward`` (float64 arrays), computed chunk-wise."""
    q, k, v, la, b = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    out = np.zeros((T, H, Dv))
    Sf = np.zeros((N, H, Dk, Dv))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            S = np.zeros((Dk, Dv)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                O, S = _chunk(S, q[c0:c1, h], k[c0:c1, h], v[c0:c1, h],
                              la[c0:c1, h], b[c0:c1, h])
                out[c0:c1, h] = O
            Sf[n, h] = S
    return out, Sf


def _chunk_backward(S, Q, K, V, LA, b, dO, dSn):
    """Gradients through one chunk of ``_chunk``: given dL/dO and dL/dS_next,
    returns (dQ, dK, dV, dLA, db, dS) with dS = dL/d(entering state).

    Reverse mode through the forward steps above, last step first; T is formed
    explicitly (one unit-lower-triangular solve) because its gradient is
    dA = -T^T dT T^T restricted to the strictly lower entries A depends on."""
    L = Q.shape[0]
    g = np.cumsum(LA, axis=0)
    eg, emg = np.exp(g), np.exp(-g)
    Kg, Ki, Qg = K * eg, K * emg, Q * eg
    M = Kg @ Ki.T
    A = np.tril(b[:, None] * M, k=-1)
    I = np.eye(L)
    T = solve_triangular(I + A, I, lower=True, unit_diagonal=True)
    bKg, bV = b[:, None] * Kg, b[:, None] * V
    W, U0 = T @ bKg, T @ bV
    U = U0 - W @ S
    P = np.tril(Qg @ Ki.T)
    gl = g[-1]
    ed = np.exp(gl[None, :] - g)
    Kd = K * ed

    # S_next = Diag(exp(gl)) S + Kd^T U
    dS = np.exp(gl)[:, None] * dSn
    dgl = np.sum(dSn * S, axis=1) * np.exp(gl)
    dKd = U @ dSn.T
    dU = Kd @ dSn
    # Kd = K * exp(gl - g)
    dK = dKd * ed
    d_ed = dKd * K * ed
    dgl = dgl + np.sum(d_ed, axis=0)
    dg = -d_ed
    # O = Qg S + P U,  P = lower_incl(Qg Ki^T)
    dQg = dO @ S.T
    dS = dS + Qg.T @ dO
    dP = np.tril(dO @ U.T)
    dU = dU + P.T @ dO
    dQg = dQg + dP @ Ki
    dKi = dP.T @ Qg
    # U = U0 - W S
    dU0 = dU
    dW = -dU @ S.T
    dS = dS - W.T @ dU
    # U0 = T (b V),  W = T (b Kg)
    dbV, dbKg = T.T @ dU0, T.T @ dW
    dT = dU0 @ bV.T + dW @ bKg.T
    dV = b[:, None] * dbV
    db = np.sum(dbV * V, axis=1) + np.sum(dbKg * Kg, axis=1)
    dKg = b[:, None] * dbKg
    # T = (I + A)^{-1},  A = strict_lower(diag(b) M),  M = Kg Ki^T
    dA = np.tril(-T.T @ dT @ T.T, k=-1)
    db = db + np.sum(dA * M, axis=1)
    dM = b[:, None] * dA
    dKg = dKg + dM @ Ki
    dKi = dKi + dM.T @ Kg
    # Qg = Q e^g,  Kg = K e^g,  Ki = K e^-g
    dQ = dQg * eg
    dK = dK + dKg * eg + dKi * emg
    dg = dg + dQg * Q * eg + dKg * K * eg - dKi * K * emg
    dg[-1] = dg[-1] + dgl
    # g = inclusive cumsum of LA: each row's gradient collects the rows at or after it
    dLA = np.cumsum(dg[::-1], axis=0)[::-1]
    return dQ, dK, dV, dLA, db, dS


def backward_chunked(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, d_out=None,
                     dS_final=None, chunk=64):
    """Same contract as ``oracle.backward`` (float64 dict), computed chunk-wise:
    the forward keeps each chunk's entering state, then the chunks are walked
    backward with ``_chunk_backward``, dL/dS flowing from chunk to chunk."""
    q, k, v, la, b, do = (np.asarray(x, dtype=np.float64)
                          for x in (q, k, v, log_alpha, beta, d_out))
    T, H, Dk = q.shape
    Dv = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    g = {"dq": np.zeros((T, H, Dk)), "dk": np.zeros((T, H, Dk)), "dv": np.zeros((T, H, Dv)),
         "dlog_alpha": np.zeros((T, H, Dk)), "dbeta": np.zeros((T, H)),
         "dS0": np.zeros((N, H, Dk, Dv))}
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        starts = list(range(t0, t1, chunk))
        for h in range(H):
            S = np.zeros((Dk, Dv)) if S0 is None else np.array(S0[n, h], dtype=np.float64)
            entering = []
            for c0 in starts:
                c1 = min(c0 + chunk, t1)
                entering.append(S)
                _, S = _chunk(S, q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], la[c0:c1, h],
                              b[c0:c1, h])
            dS = np.zeros((Dk, Dv)) if dS_final is None else np.array(dS_final[n, h], dtype=np.float64)
            for c0, Sc in zip(reversed(starts), reversed(entering)):
                c1 = min(c0 + chunk, t1)
                dQ, dK, dV, dLA, db, dS = _chunk_backward(
                    Sc, q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], la[c0:c1, h], b[c0:c1, h],
                    do[c0:c1, h], dS)
                g["dq"][c0:c1, h], g["dk"][c0:c1, h], g["dv"][c0:c1, h] = dQ, dK, dV
                g["dlog_alpha"][c0:c1, h], g["dbeta"][c0:c1, h] = dLA, db
            g["dS0"][n, h] = dS
    return g
