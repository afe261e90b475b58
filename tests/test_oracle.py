"""Pins for the fp64 CPU oracle (no GPU).

The oracle (``oracle.forward``) is trusted only because these tests tie it to
facts that do not come from the oracle itself:
  * the definition written as an exact rational product of transition
    matrices (``oracle.exact``) on tiny inputs;
  * closed forms: no writes (beta = 0) leave a pure per-channel decay of S0;
    a unit key written with beta = 1 is read back exactly (exact-write);
  * the no-decay case equals the textbook DeltaNet update;
  * an independent chunk-form restatement agrees for many chunk sizes;
  * structural invariants: linearity in (V, S0), v-channel separability,
    split-chain consistency, varlen isolation, a norm bound.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact
from oracle.chunked import forward_chunked


def _rand_chain(rng, T, H, Dk, Dv, alpha_min=0.5, unit_k=True, N=1):
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    la = rng.uniform(math.log(alpha_min), 0.0, size=(T, H, Dk))
    S0 = 0.1 * rng.standard_normal((N, H, Dk, Dv))
    return q, k, v, la, beta, S0


def _rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------------------
# exact rational definition
# --------------------------------------------------------------------------
@pytest.mark.parametrize("Dk,Dv,T,seed", [(2, 2, 4, 0), (3, 2, 3, 1), (2, 3, 4, 2), (3, 3, 2, 3)])
def test_exact_unrolled(Dk, Dv, T, seed):
    rng = np.random.default_rng(seed)
    fr = lambda: Fraction(int(rng.integers(-8, 9)), 8)
    alphas = [Fraction(1), Fraction(1, 2), Fraction(3, 4)]
    betas = [Fraction(0), Fraction(1, 2), Fraction(1)]
    q = [[fr() for _ in range(Dk)] for _ in range(T)]
    k = [[fr() for _ in range(Dk)] for _ in range(T)]
    v = [[fr() for _ in range(Dv)] for _ in range(T)]
    al = [[alphas[int(rng.integers(0, 3))] for _ in range(Dk)] for _ in range(T)]
    be = [betas[int(rng.integers(0, 3))] for _ in range(T)]
    S0 = [[fr() for _ in range(Dv)] for _ in range(Dk)]
    o_ex, S_ex = exact.unrolled_product(q, k, v, al, be, S0)

    f = lambda x: np.array(x, dtype=np.float64)
    out, Sf = oracle.forward(
        f(q)[:, None, :], f(k)[:, None, :], f(v)[:, None, :],
        np.log(f(al))[:, None, :], f(be)[:, None], S0=f(S0)[None, None])
    o_ref = f([[float(x) for x in row] for row in o_ex])
    S_ref = f([[float(x) for x in row] for row in S_ex[-1]])
    assert np.allclose(out[:, 0, :], o_ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(Sf[0, 0], S_ref, rtol=1e-13, atol=1e-13)


def test_exact_unrolled_two_heads_two_seqs():
    """Head and sequence indexing: each (seq, head) chain equals its own exact product."""
    rng = np.random.default_rng(7)
    T, H, Dk, Dv = 5, 2, 2, 3
    fr = lambda: Fraction(int(rng.integers(-4, 5)), 4)
    q = [[[fr() for _ in range(Dk)] for _ in range(H)] for _ in range(T)]
    k = [[[fr() for _ in range(Dk)] for _ in range(H)] for _ in range(T)]
    v = [[[fr() for _ in range(Dv)] for _ in range(H)] for _ in range(T)]
    al = [[[Fraction(1, 2) if (t + h + c) % 2 else Fraction(3, 4) for c in range(Dk)]
           for h in range(H)] for t in range(T)]
    be = [[Fraction(1, 2) if (t + h) % 3 else Fraction(1) for h in range(H)] for t in range(T)]
    S0 = [[[[fr() for _ in range(Dv)] for _ in range(Dk)] for _ in range(H)] for _ in range(2)]
    cu = [0, 2, 5]
    f = lambda x: np.array(x, dtype=np.float64)
    out, Sf = oracle.forward(f(q), f(k), f(v), np.log(f(al)), f(be), S0=f(S0), cu_seqlens=cu)
    for n in range(2):
        for h in range(H):
            ts = range(cu[n], cu[n + 1])
            o_ex, S_ex = exact.unrolled_product(
                [q[t][h] for t in ts], [k[t][h] for t in ts], [v[t][h] for t in ts],
                [al[t][h] for t in ts], [be[t][h] for t in ts], S0[n][h])
            for i, t in enumerate(ts):
                assert np.allclose(out[t, h], [float(x) for x in o_ex[i]], rtol=1e-13, atol=1e-13)
            assert np.allclose(Sf[n, h], f([[float(x) for x in r] for r in S_ex[-1]]),
                               rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# closed forms and special cases
# --------------------------------------------------------------------------
def test_beta_zero_pure_decay():
    """beta = 0: no erase and no write; S_t = Diag(exp(sum log alpha)) S0, o_t = S_t^T q_t."""
    rng = np.random.default_rng(3)
    T, H, Dk, Dv = 37, 2, 8, 5
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    beta[:] = 0.0
    out, Sf = oracle.forward(q, k, v, la, beta, S0=S0)
    G = np.cumsum(la, axis=0)                       # [T, H, Dk]
    for h in range(H):
        for t in range(T):
            St = np.exp(G[t, h])[:, None] * S0[0, h]
            assert np.allclose(out[t, h], St.T @ q[t, h], rtol=1e-12, atol=1e-14)
        assert np.allclose(Sf[0, h], np.exp(G[-1, h])[:, None] * S0[0, h], rtol=1e-12)


def test_exact_write_any_decay():
    """beta = 1 and ||k|| = 1 store v exactly along k: S_t^T k_t = v_t for any alpha.

    With q_t = k_t the oracle's output must equal v_t.  Keys are exact unit
    vectors (coordinate axes and (3/5, 4/5) rotations) so the fp64 identity
    holds to rounding.
    """
    rng = np.random.default_rng(4)
    T, H, Dk, Dv = 40, 3, 4, 6
    k = np.zeros((T, H, Dk))
    for t in range(T):
        for h in range(H):
            i, j = rng.choice(Dk, 2, replace=False)
            s = 1.0 if rng.random() < 0.5 else -1.0
            k[t, h, i], k[t, h, j] = 0.6 * s, 0.8
    v = rng.standard_normal((T, H, Dv))
    la = rng.uniform(math.log(0.3), 0.0, size=(T, H, Dk))
    beta = np.ones((T, H))
    S0 = rng.standard_normal((1, H, Dk, Dv))
    out, _ = oracle.forward(k.copy(), k, v, la, beta, S0=S0)
    assert np.allclose(out, v, rtol=0, atol=1e-12)


def test_deltanet_reduction():
    """alpha = 1: the textbook DeltaNet update S <- S + beta k (v^T - k^T S)."""
    rng = np.random.default_rng(5)
    T, H, Dk, Dv = 50, 2, 6, 4
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    la[:] = 0.0
    out, Sf = oracle.forward(q, k, v, la, beta, S0=S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kt = k[t, h][:, None]
            S = S + beta[t, h] * kt @ (v[t, h][None, :] - kt.T @ S)
            assert np.allclose(out[t, h], S.T @ q[t, h], rtol=1e-12, atol=1e-13)
        assert np.allclose(Sf[0, h], S, rtol=1e-12, atol=1e-13)


def test_single_token_closed_form():
    """One token from S0: S_1 = (I - b k k^T) D S0 + b k v^T, o = S_1^T q (matrix form)."""
    rng = np.random.default_rng(6)
    Dk, Dv = 5, 7
    q, k, v, la, beta, S0 = _rand_chain(rng, 1, 1, Dk, Dv, unit_k=False)
    out, Sf = oracle.forward(q, k, v, la, beta, S0=S0)
    kk = k[0, 0][:, None]
    M = (np.eye(Dk) - beta[0, 0] * kk @ kk.T) @ np.diag(np.exp(la[0, 0]))
    S1 = M @ S0[0, 0] + beta[0, 0] * kk @ v[0, 0][None, :]
    assert np.allclose(Sf[0, 0], S1, rtol=1e-13, atol=1e-14)
    assert np.allclose(out[0, 0], S1.T @ q[0, 0], rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# chunk form (pins the algebra used by chunked kernels)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("C", [1, 7, 16, 64, 200])
def test_chunk_equivalence(C):
    rng = np.random.default_rng(10 + C)
    T, H, Dk, Dv = 200, 2, 16, 8
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv, alpha_min=0.6)
    ref_o, ref_s = oracle.forward(q, k, v, la, beta, S0=S0)
    o, s = forward_chunked(q, k, v, la, beta, S0=S0, chunk=C)
    assert _rel(o, ref_o) < 1e-11
    assert _rel(s, ref_s) < 1e-11


def test_chunk_equivalence_varlen_partial_chunks():
    rng = np.random.default_rng(21)
    lens = [1, 63, 64, 65, 0, 130]
    T, H, Dk, Dv = sum(lens), 2, 8, 8
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv, N=len(lens))
    cu = np.concatenate([[0], np.cumsum(lens)])
    ref_o, ref_s = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu)
    o, s = forward_chunked(q, k, v, la, beta, S0=S0, cu_seqlens=cu, chunk=64)
    assert _rel(o, ref_o) < 1e-11
    assert _rel(s, ref_s) < 1e-11


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
def test_split_chain():
    rng = np.random.default_rng(11)
    T, H, Dk, Dv = 90, 2, 8, 6
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    o, s = oracle.forward(q, k, v, la, beta, S0=S0)
    t0 = 37
    o1, s1 = oracle.forward(q[:t0], k[:t0], v[:t0], la[:t0], beta[:t0], S0=S0)
    o2, s2 = oracle.forward(q[t0:], k[t0:], v[t0:], la[t0:], beta[t0:], S0=s1)
    assert np.allclose(np.concatenate([o1, o2]), o, rtol=1e-13, atol=1e-14)
    assert np.allclose(s2, s, rtol=1e-13, atol=1e-14)


def test_linearity_in_v_and_state():
    rng = np.random.default_rng(12)
    T, H, Dk, Dv = 40, 2, 6, 5
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    o1, s1 = oracle.forward(q, k, v, la, beta, S0=S0)
    o2, s2 = oracle.forward(q, k, v2, la, beta, S0=S02)
    o3, s3 = oracle.forward(q, k, 2.5 * v - v2, la, beta, S0=2.5 * S0 - S02)
    assert np.allclose(o3, 2.5 * o1 - o2, rtol=1e-11, atol=1e-12)
    assert np.allclose(s3, 2.5 * s1 - s2, rtol=1e-11, atol=1e-12)


def test_value_channel_separability():
    rng = np.random.default_rng(13)
    T, H, Dk, Dv = 30, 2, 6, 7
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    perm = rng.permutation(Dv)
    o, s = oracle.forward(q, k, v, la, beta, S0=S0)
    op, sp = oracle.forward(q, k, v[..., perm], la, beta, S0=S0[..., perm])
    assert np.array_equal(op, o[..., perm])
    assert np.array_equal(sp, s[..., perm])


def test_varlen_isolation_and_empty_sequence():
    rng = np.random.default_rng(14)
    lens = [3, 0, 17, 1]
    T, H, Dk, Dv = sum(lens), 2, 5, 4
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv, N=len(lens))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, s = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        a, b = cu[n], cu[n + 1]
        if L == 0:
            assert np.array_equal(s[n], S0[n])
            continue
        on, sn = oracle.forward(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], S0=S0[n:n + 1])
        assert np.array_equal(o[a:b], on)
        assert np.array_equal(s[n], sn[0])


def test_state_norm_bound():
    """||k|| = 1, beta in [0,1], alpha in (0,1]: ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||."""
    rng = np.random.default_rng(15)
    T, H, Dk, Dv = 60, 1, 8, 8
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv)
    S = S0
    for t in range(T):
        _, Sn = oracle.forward(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1],
                               beta[t:t + 1], S0=S)
        lhs = np.linalg.norm(Sn[0, 0], 2)
        rhs = np.linalg.norm(S[0, 0], 2) + beta[t, 0] * np.linalg.norm(v[t, 0])
        assert lhs <= rhs * (1 + 1e-12)
        S = Sn


def test_thread_count_invariance():
    rng = np.random.default_rng(16)
    lens = [20, 33, 5]
    T, H, Dk, Dv = sum(lens), 3, 8, 8
    q, k, v, la, beta, S0 = _rand_chain(rng, T, H, Dk, Dv, N=3)
    cu = np.concatenate([[0], np.cumsum(lens)])
    a = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, threads=1)
    b = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, threads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_decode_step_equals_one_token_forward():
    rng = np.random.default_rng(17)
    N, H, Dk, Dv = 5, 2, 6, 4
    q, k, v, la, beta, S0 = _rand_chain(rng, N, H, Dk, Dv, N=N)
    o_d, S_d = oracle.decode_step(q, k, v, la, beta, S0)
    o_f, S_f = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=np.arange(N + 1))
    assert np.array_equal(o_d, o_f) and np.array_equal(S_d, S_f)


def test_bad_seqlens_rejected():
    rng = np.random.default_rng(18)
    q, k, v, la, beta, S0 = _rand_chain(rng, 4, 1, 2, 2)
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, beta, cu_seqlens=[0, 3, 2, 4])
    with pytest.raises(ValueError):
        oracle.forward(q, k, v, la, beta, cu_seqlens=[0, 3])


# --------------------------------------------------------------------------
# state snapshots (prefix caching at fixed token boundaries)
# --------------------------------------------------------------------------
def _snapshot_case(seed=21, E=16):
    rng = np.random.default_rng(seed)
    lens = [50, 7, 32, 0, 65]   # partial, shorter than E, exact multiple, empty, one past
    T, H, Dk, Dv = sum(lens), 2, 6, 5
    q, k, v, la, beta, _ = _rand_chain(rng, T, H, Dk, Dv)
    S0 = 0.1 * rng.standard_normal((len(lens), H, Dk, Dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    return lens, cu, E, (q, k, v, la, beta, S0)


def test_snapshot_counts_and_offsets():
    lens, cu, E, (q, k, v, la, beta, S0) = _snapshot_case()
    o, s, snaps, off = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, snapshot_every=E)
    counts = [n // E for n in lens]
    assert snaps.shape[0] == sum(counts)
    assert list(off) == list(np.concatenate([[0], np.cumsum(counts)[:-1]]))
    # the plain call returns the same outputs and final states
    o2, s2 = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu)
    assert np.array_equal(o, o2) and np.array_equal(s, s2)


def test_snapshot_equals_final_state_of_the_prefix():
    """Snapshot m of sequence n is the final state of the same chain run on the
    first (m + 1) E tokens only, through the plain entry point."""
    lens, cu, E, (q, k, v, la, beta, S0) = _snapshot_case()
    _, _, snaps, off = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, snapshot_every=E)
    checked = 0
    for n, L in enumerate(lens):
        for m in range(L // E):
            a, b = cu[n], cu[n] + (m + 1) * E
            _, sp = oracle.forward(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], S0=S0[n:n + 1])
            assert np.allclose(snaps[off[n] + m], sp[0], rtol=1e-13, atol=1e-14)
            checked += 1
    assert checked == sum(L // E for L in lens)


def test_resume_from_snapshot_reproduces_the_tail():
    """A prefill started from snapshot m (as S0) on the rest of the sequence gives
    the same outputs and final state as the uninterrupted run."""
    lens, cu, E, (q, k, v, la, beta, S0) = _snapshot_case()
    o, s, snaps, off = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, snapshot_every=E)
    n, m = 4, 3                      # sequence of 65 tokens, resume after token 64
    a = cu[n] + (m + 1) * E
    b = cu[n + 1]
    o2, s2 = oracle.forward(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b],
                            S0=snaps[off[n] + m][None])
    assert np.allclose(o2, o[a:b], rtol=1e-13, atol=1e-14)
    assert np.allclose(s2[0], s[n], rtol=1e-13, atol=1e-14)


def test_snapshot_at_sequence_end_is_the_final_state():
    lens, cu, E, (q, k, v, la, beta, S0) = _snapshot_case()
    _, s, snaps, off = oracle.forward(q, k, v, la, beta, S0=S0, cu_seqlens=cu, snapshot_every=E)
    n = 2                            # 32 tokens = 2 E: its last snapshot is its final state
    assert np.array_equal(snaps[off[n] + 1], s[n])


# --------------------------------------------------------------------------
# stored exact values (tests/golden/exact_chain.json, written by
# tests/golden/make_exact_chain.py from oracle.exact only)
# --------------------------------------------------------------------------
def test_oracle_reproduces_the_stored_exact_chain():
    import json
    import os
    from fractions import Fraction
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "exact_chain.json")
    doc = json.load(open(path))
    f = lambda M: np.array([[float(Fraction(x)) for x in row] for row in M])
    inp = doc["inputs"]
    T = len(inp["q"])
    q, k, v, alpha = (f(inp[n])[:, None, :] for n in ("q", "k", "v", "alpha"))
    beta = np.array([float(Fraction(x)) for x in inp["beta"]])[:, None]
    S0 = f(inp["S0"])[None, None]
    out, sf = oracle.forward(q, k, v, np.log(alpha), beta, S0=S0)
    assert np.allclose(out[:, 0], f(doc["out"]), rtol=1e-13, atol=1e-14)
    assert np.allclose(sf[0, 0], f(doc["states"][T - 1]), rtol=1e-13, atol=1e-14)
    # and every intermediate state, through the snapshot entry point
    _, _, snaps, _ = oracle.forward(q, k, v, np.log(alpha), beta, S0=S0, snapshot_every=1)
    for t in range(T):
        assert np.allclose(snaps[t, 0], f(doc["states"][t]), rtol=1e-13, atol=1e-14)
