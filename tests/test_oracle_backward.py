"""Pins of the fp64 backward oracle (oracle.backward, kda_oracle_bwd.c).

The gradients are pinned to things other than themselves:
  * central finite differences of the (separately pinned) forward oracle, on
    tiny inputs, for every input element;
  * closed forms when beta = 0 and log_alpha = 0 (the state never changes);
  * PyTorch's fp64 autograd of the recurrence written out with tensor ops;
and plausible mistakes planted in a copy of the backward source must fail the
finite-difference pin.  The recurrence is that of the page "Kimi K3: Open
Frontier Intelligence and Implementation Framework" (section "Hybrid
Attention Mechanism", KDA bullet).
"""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

SRC_BWD = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle_bwd.c")


def _tiny(seed=0, lens=(3, 0, 2), H=2, Dk=3, Dv=2):
    rng = np.random.default_rng(seed)
    T, N = sum(lens), len(lens)
    x = lambda *s: rng.standard_normal(s)
    return dict(q=x(T, H, Dk), k=x(T, H, Dk), v=x(T, H, Dv),
                log_alpha=rng.uniform(math.log(0.3), 0.0, (T, H, Dk)),
                beta=rng.uniform(0.1, 1.0, (T, H)), S0=x(N, H, Dk, Dv),
                cu=np.concatenate([[0], np.cumsum(lens)]).astype(np.int64),
                d_out=x(T, H, Dv), dS_final=x(N, H, Dk, Dv))


def _loss(inp):
    out, sf = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                             inp["S0"], inp["cu"])
    return float(np.sum(out * inp["d_out"]) + np.sum(sf * inp["dS_final"]))


def _grads(inp, lib=None):
    return oracle.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["S0"], inp["cu"], inp["d_out"], inp["dS_final"], lib=lib)


NAMES = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "beta": "dbeta",
         "S0": "dS0"}


def _fd_pin(lib=None, seed=0) -> bool:
    """Every gradient element against a central difference (eps = 1e-6)."""
    inp = _tiny(seed)
    g = _grads(inp, lib)
    eps = 1e-6
    for name, gname in NAMES.items():
        x = inp[name]
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(inp)
            x[idx] = keep - eps
            lm = _loss(inp)
            x[idx] = keep
            fd = (lp - lm) / (2 * eps)
            if abs(fd - g[gname][idx]) > 1e-6 * (1 + abs(fd)):
                return False
    return True


def test_backward_matches_finite_differences():
    assert _fd_pin(seed=0)
    assert _fd_pin(seed=1)


def test_backward_closed_form_without_write_or_decay():
    """beta = 0, log_alpha = 0: S_t = S0 for every t, so o_t = S0^T q_t and
    dq_t = S0 do_t, dS0 = dS_final + sum_t q_t do_t^T, dv = dk = 0,
    dlog_alpha_t[c] = sum_j G_t[c,j] S0[c,j] and dbeta_t = k_t^T G_t e_t with
    G_t = dS_final + sum_{s>=t} q_s do_s^T and e_t = v_t - S0^T k_t."""
    inp = _tiny(2, lens=(5,), H=1, Dk=4, Dv=3)
    inp["beta"][:] = 0.0
    inp["log_alpha"][:] = 0.0
    g = _grads(inp)
    S0, dSf = inp["S0"][0, 0], inp["dS_final"][0, 0]
    q, k, v, do = (inp[n][:, 0] for n in ("q", "k", "v", "d_out"))
    T = q.shape[0]
    np.testing.assert_allclose(g["dq"][:, 0], do @ S0.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dS0"][0, 0], dSf + q.T @ do, rtol=1e-12, atol=1e-12)
    assert np.all(g["dv"] == 0) and np.all(g["dk"] == 0)
    for t in range(T):
        Gt = dSf + q[t:].T @ do[t:]
        np.testing.assert_allclose(g["dlog_alpha"][t, 0], np.sum(Gt * S0, axis=1),
                                   rtol=1e-12, atol=1e-12)
        e = v[t] - S0.T @ k[t]
        np.testing.assert_allclose(g["dbeta"][t, 0], k[t] @ Gt @ e, rtol=1e-12, atol=1e-12)


def test_backward_matches_autograd():
    inp = _tiny(3, lens=(17, 13), H=2, Dk=4, Dv=5)
    t = {n: torch.tensor(inp[n], dtype=torch.float64, requires_grad=True) for n in NAMES}
    outs, finals = [], []
    for n in range(len(inp["cu"]) - 1):
        a, b = int(inp["cu"][n]), int(inp["cu"][n + 1])
        for h in range(2):
            S = t["S0"][n, h]
            for i in range(a, b):
                S = torch.exp(t["log_alpha"][i, h])[:, None] * S
                e = t["v"][i, h] - S.T @ t["k"][i, h]
                S = S + t["beta"][i, h] * torch.outer(t["k"][i, h], e)
                outs.append((i, h, S.T @ t["q"][i, h]))
            finals.append((n, h, S))
    L = sum((o * torch.tensor(inp["d_out"][i, h])).sum() for i, h, o in outs)
    L = L + sum((S * torch.tensor(inp["dS_final"][n, h])).sum() for n, h, S in finals)
    L.backward()
    g = _grads(inp)
    for name, gname in NAMES.items():
        np.testing.assert_allclose(g[gname], t[name].grad.numpy(), rtol=1e-10, atol=1e-10,
                                   err_msg=gname)


# (name, original fragment, mutated fragment) in kda_oracle_bwd.c
MUTANTS = [
    ("dk_misses_P_de", "dkt[c] = dkt[c] - pde;", "dkt[c] = dkt[c];"),
    ("dP_sign", "dP[c * Dv + j] = dP[c * Dv + j] - kt[c] * de[j];",
     "dP[c * Dv + j] = dP[c * Dv + j] + kt[c] * de[j];"),
    ("dlog_alpha_misses_alpha", "dlat[c] = a * acc;", "dlat[c] = acc;"),
    ("state_grad_not_decayed", "G[c * Dv + j] = a * dP[c * Dv + j];",
     "G[c * Dv + j] = dP[c * Dv + j];"),
    ("dq_uses_previous_state", "acc = acc + S[c * Dv + j] * dot[j];",
     "acc = acc + Sp[c * Dv + j] * dot[j];"),
    ("dbeta_misses_key", "db = db + kt[c] * ge;", "db = db + ge;"),
    ("de_misses_beta", "de[j] = de[j] + bt * kt[c] * G[c * Dv + j];",
     "de[j] = de[j] + kt[c] * G[c * Dv + j];"),
    ("dS_final_ignored", "if (J->dSf) memcpy(G, J->dSf + (n * H + h) * KV, sizeof(double) * KV);",
     "if (0) memcpy(G, J->dSf, 0);"),
    ("readout_grad_transposed", "G[c * Dv + j] = G[c * Dv + j] + qt[c] * dot[j];",
     "G[c * Dv + j] = G[c * Dv + j] + qt[j % Dk] * dot[c % Dv];"),
]


def _build_bwd(tmp_path, name, text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(text)
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(so), str(c), "-lm"], check=True)
    return oracle.bind_backward(str(so))


def test_real_backward_source_passes(tmp_path):
    assert _fd_pin(_build_bwd(tmp_path, "real", open(SRC_BWD).read()))


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_backward_mutant_rejected(tmp_path, name, orig, mut):
    text = open(SRC_BWD).read()
    assert text.count(orig) == 1, f"mutation anchor for {name} not unique"
    assert not _fd_pin(_build_bwd(tmp_path, name, text.replace(orig, mut))), name


@pytest.mark.parametrize("C", [1, 7, 16, 64])
def test_chunk_form_backward_matches_token_backward(C):
    """The chunk-form gradients (oracle.chunked.backward_chunked: reverse mode
    through the chunk algebra of the forward, the algebra a chunked backward
    kernel uses) equal the token-level backward, including partial last
    chunks and an empty sequence."""
    from oracle.chunked import backward_chunked
    rng = np.random.default_rng(C)
    lens = [70, 0, 33, 129]
    T, H, Dk, Dv, N = sum(lens), 2, 8, 6, len(lens)
    x = lambda *s: rng.standard_normal(s)
    q, k = x(T, H, Dk), x(T, H, Dk)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v, do = x(T, H, Dv), x(T, H, Dv)
    la = rng.uniform(math.log(0.8), 0.0, (T, H, Dk))
    b = rng.uniform(0.1, 1.0, (T, H))
    S0, dSf = x(N, H, Dk, Dv), x(N, H, Dk, Dv)
    cu = np.concatenate([[0], np.cumsum(lens)])
    ref = oracle.backward(q, k, v, la, b, S0, cu, do, dSf)
    got = backward_chunked(q, k, v, la, b, S0, cu, do, dSf, chunk=C)
    for name in NAMES.values():
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-10, atol=1e-10, err_msg=name)


def test_chunk_form_backward_property():
    """Random small shapes, lengths (empty ones included) and chunk sizes: the
    chunk-form gradients equal the token-level ones."""
    from hypothesis import given, settings, strategies as st
    from oracle.chunked import backward_chunked

    @settings(max_examples=40, deadline=None, derandomize=True)
    @given(lens=st.lists(st.integers(0, 23), min_size=1, max_size=3),
           C=st.integers(1, 9), H=st.integers(1, 2), Dk=st.integers(1, 5), Dv=st.integers(1, 4),
           seed=st.integers(0, 2**16))
    def check(lens, C, H, Dk, Dv, seed):
        rng = np.random.default_rng(seed)
        T, N = sum(lens), len(lens)
        x = lambda *s: rng.standard_normal(s)
        la = rng.uniform(math.log(0.5), 0.0, (T, H, Dk))
        args = (x(T, H, Dk), x(T, H, Dk), x(T, H, Dv), la, rng.uniform(0.0, 1.0, (T, H)),
                x(N, H, Dk, Dv), np.concatenate([[0], np.cumsum(lens)]), x(T, H, Dv),
                x(N, H, Dk, Dv))
        ref = oracle.backward(*args)
        got = backward_chunked(*args, chunk=C)
        for name in NAMES.values():
            np.testing.assert_allclose(got[name], ref[name], rtol=1e-9, atol=1e-9, err_msg=name)

    check()
