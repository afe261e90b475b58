"""Exact rational form of the KDA recurrence -- TEST INFRASTRUCTURE.

For tiny inputs this writes the recurrence of the page "Kimi K3: Open
Frontier Intelligence and Implementation Framework" (section "Hybrid
Attention Mechanism", KDA bullet) as an explicit product of transition
matrices, in ``fractions.Fraction`` arithmetic:

    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)
    S_t = M_t ... M_1 S_0 + sum_{s<=t} M_t ... M_{s+1} beta_s k_s v_s^T
    o_t = S_t^T q_t

Every S_t is formed from the closed sum above (not by stepping a running
state), so it is an independent statement of the definition against which
the fp64 oracle is pinned.  Cost is O(T^2 D^3): keep T and D tiny.
"""
from __future__ import annotations

from fractions import Fraction


def _eye(n):
    return [[Fraction(int(i == j)) for j in range(n)] for i in range(n)]


def _matmul(A, B):
    n, m, p = len(A), len(B), len(B[0])
    return [[sum((A[i][r] * B[r][j] for r in range(m)), Fraction(0)) for j in range(p)]
            for i in range(n)]


def _add(A, B):
    return [[a + b for a, b in zip(ra, rb)] for ra, rb in zip(A, B)]


def transition(k, alpha, beta):
    """M = (I - beta k k^T) Diag(alpha), exact."""
    n = len(k)
    return [[(Fraction(int(i == j)) - beta * k[i] * k[j]) * alpha[j] for j in range(n)]
            for i in range(n)]


def unrolled_product(q, k, v, alpha, beta, S0):
    """Exact outputs and states for one chain.

    q, k, alpha: T lists of Dk Fractions; v: T lists of Dv Fractions;
    beta: T Fractions; S0: Dk x Dv Fractions.
    Returns (o, S) with o[t] a list of Dv Fractions and S[t] the state after
    token t (S[0] is the state after the first token).
    """
    T = len(q)
    Dk = len(S0)
    M = [transition(k[t], alpha[t], beta[t]) for t in range(T)]

    def prod(hi, lo):
        """M_hi M_{hi-1} ... M_lo (1-based, inclusive); identity when hi < lo."""
        P = _eye(Dk)
        for s in range(lo, hi + 1):
            P = _matmul(M[s - 1], P)
        return P

    outs, states = [], []
    for t in range(1, T + 1):
        S = _matmul(prod(t, 1), S0)
        for s in range(1, t + 1):
            write = [[beta[s - 1] * k[s - 1][i] * v[s - 1][j] for j in range(len(v[0]))]
                     for i in range(Dk)]
            S = _add(S, _matmul(prod(t, s + 1), write))
        o = [sum((S[i][j] * q[t - 1][i] for i in range(Dk)), Fraction(0))
             for j in range(len(v[0]))]
        outs.append(o)
        states.append(S)
    return outs, states
