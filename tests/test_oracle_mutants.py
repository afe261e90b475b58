"""The oracle's pins must be sharp: plant plausible mistakes in a copy of the
oracle's C source (on the CPU, in a temporary directory), rebuild it, and
check that the pins reject every mutant while accepting the real source.
"""
import math
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

# (name, original line fragment, mutated fragment)
MUTANTS = [
    ("error_sign", "e[j] = vt[j] - e[j];", "e[j] = e[j] - vt[j];"),
    ("decay_dropped", "for (int64_t j = 0; j < Dv; ++j) row[j] = a * row[j];",
     "for (int64_t j = 0; j < Dv; ++j) row[j] = row[j];"),
    ("decay_inverted", "const double a = exp(lat[c]);", "const double a = exp(-lat[c]);"),
    ("beta_dropped", "const double w = bt * kt[c];", "const double w = kt[c];"),
    ("readout_uses_key", "const double qc = qt[c];", "const double qc = kt[c];"),
    ("readout_transposed", "ot[j] = ot[j] + qc * row[j];", "ot[j] = ot[j] + qc * S[j * Dv + c];"),
    ("erase_uses_query", "const double kc = kt[c];", "const double kc = qt[c];"),
    ("head_index_wrong", "const double *vt = J->v + (t * H + h) * Dv;",
     "const double *vt = J->v + (t * H + 0) * Dv;"),
    ("s0_ignored", "memcpy(S, J->S0 + (n * H + h) * Dk * Dv, sizeof(double) * Dk * Dv);",
     "memset(S, 0, sizeof(double) * Dk * Dv);"),
    ("snapshot_one_token_early", "const int64_t done = t - t0 + 1;", "const int64_t done = t - t0 + 2;"),
    ("snapshot_wrong_slot", "const int64_t m = J->snap_off[n] + done / J->snap_every - 1;",
     "const int64_t m = J->snap_off[n] + done / J->snap_every - 1 + (done > J->snap_every);"),
]


def _build(tmp_path, name, src_text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src_text)
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"], check=True)
    return oracle.bind(str(so))


def _exact_pin(lib) -> bool:
    rng = np.random.default_rng(99)
    T, H, D = 4, 2, 3
    fr = lambda: Fraction(int(rng.integers(-8, 9)), 8)
    ok = True
    q = [[[fr() for _ in range(D)] for _ in range(H)] for _ in range(T)]
    k = [[[fr() for _ in range(D)] for _ in range(H)] for _ in range(T)]
    v = [[[fr() for _ in range(D)] for _ in range(H)] for _ in range(T)]
    al = [[[Fraction(1, 2) if (t + c) % 2 else Fraction(3, 4) for c in range(D)]
           for _ in range(H)] for t in range(T)]
    be = [[Fraction(1, 2) if t % 2 else Fraction(1) for _ in range(H)] for t in range(T)]
    S0 = [[[[fr() for _ in range(D)] for _ in range(D)] for _ in range(H)]]
    f = lambda x: np.array(x, dtype=np.float64)
    out, Sf = oracle.forward(f(q), f(k), f(v), np.log(f(al)), f(be), S0=f(S0), lib=lib)
    for h in range(H):
        o_ex, S_ex = exact.unrolled_product([q[t][h] for t in range(T)], [k[t][h] for t in range(T)],
                                            [v[t][h] for t in range(T)], [al[t][h] for t in range(T)],
                                            [be[t][h] for t in range(T)], S0[0][h])
        ok &= np.allclose(out[:, h], f([[float(x) for x in r] for r in o_ex]), rtol=1e-12, atol=1e-12)
        ok &= np.allclose(Sf[0, h], f([[float(x) for x in r] for r in S_ex[-1]]), rtol=1e-12, atol=1e-12)
    return bool(ok)


def _exact_write_pin(lib) -> bool:
    rng = np.random.default_rng(5)
    T, H, Dk, Dv = 12, 2, 4, 4
    k = np.zeros((T, H, Dk))
    for t in range(T):
        for h in range(H):
            i, j = rng.choice(Dk, 2, replace=False)
            k[t, h, i], k[t, h, j] = 0.6, 0.8
    v = rng.standard_normal((T, H, Dv))
    la = rng.uniform(math.log(0.4), 0.0, size=(T, H, Dk))
    S0 = rng.standard_normal((1, H, Dk, Dv))
    out, _ = oracle.forward(k.copy(), k, v, la, np.ones((T, H)), S0=S0, lib=lib)
    return bool(np.allclose(out, v, atol=1e-12))


def _snapshot_pin(lib) -> bool:
    """Snapshots equal the final states of the prefixes (plain entry point)."""
    rng = np.random.default_rng(3)
    lens, E = [37, 20], 8
    T, H, D = sum(lens), 2, 3
    q, k, v = (rng.standard_normal((T, H, D)) for _ in range(3))
    la = rng.uniform(-0.5, 0.0, size=(T, H, D))
    beta = rng.uniform(0.2, 1.0, size=(T, H))
    cu = np.array([0, lens[0], T])
    _, _, snaps, off = oracle.forward(q, k, v, la, beta, cu_seqlens=cu, lib=lib, snapshot_every=E)
    ok = snaps.shape[0] == sum(L // E for L in lens)
    for n, L in enumerate(lens):
        for m in range(L // E):
            a, b = cu[n], cu[n] + (m + 1) * E
            _, sp = oracle.forward(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], lib=lib)
            ok = ok and np.allclose(snaps[off[n] + m], sp[0], rtol=1e-12, atol=1e-12)
    return bool(ok)


def _pins_pass(lib) -> bool:
    return _exact_pin(lib) and _exact_write_pin(lib) and _snapshot_pin(lib)


def test_real_source_passes(tmp_path):
    assert _pins_pass(_build(tmp_path, "real", open(SRC).read()))


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_rejected(tmp_path, name, orig, mut):
    text = open(SRC).read()
    assert text.count(orig) == 1, f"mutation anchor for {name} not unique in the oracle source"
    lib = _build(tmp_path, name, text.replace(orig, mut))
    assert not _pins_pass(lib), f"pins failed to reject mutant {name}"
