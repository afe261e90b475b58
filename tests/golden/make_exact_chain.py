"""Writes exact_chain.json: one tiny KDA chain with rational inputs and its
outputs and states in exact rational arithmetic.

The values come only from ``oracle.exact`` (the recurrence of the page "Kimi
K3: Open Frontier Intelligence and Implementation Framework", section
"Hybrid Attention Mechanism", KDA bullet, written as an explicit product of
transition matrices in fractions.Fraction).  Re-run it only if that
definition's reading changes:  python tests/golden/make_exact_chain.py
"""
import json
import os
import sys
from fractions import Fraction

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import exact  # noqa: E402

F = Fraction
# T = 3 tokens, Dk = 3, Dv = 2; decays are powers of two so exp(log_alpha)
# is exact in binary floating point as well.
q = [[F(1, 2), F(-1, 4), F(3, 4)], [F(0), F(1), F(-1, 2)], [F(1, 8), F(1, 8), F(1, 2)]]
k = [[F(3, 5), F(4, 5), F(0)], [F(0), F(3, 5), F(4, 5)], [F(1), F(0), F(0)]]
v = [[F(1), F(-2)], [F(1, 2), F(3, 4)], [F(-1, 4), F(1)]]
alpha = [[F(1, 2), F(1), F(1, 4)], [F(1), F(1, 2), F(1, 2)], [F(1, 4), F(1, 2), F(1)]]
beta = [F(1, 2), F(1), F(3, 4)]
S0 = [[F(1, 4), F(0)], [F(-1, 2), F(1, 8)], [F(0), F(1)]]

o, S = exact.unrolled_product(q, k, v, alpha, beta, S0)
enc = lambda M: [[str(x) for x in row] for row in M]
doc = {
    "source": "oracle.exact.unrolled_product (make_exact_chain.py)",
    "inputs": {"q": enc(q), "k": enc(k), "v": enc(v), "alpha": enc(alpha),
               "beta": [str(x) for x in beta], "S0": enc(S0)},
    "out": enc(o),
    "states": [enc(St) for St in S],
}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "exact_chain.json"), "w") as f:
    json.dump(doc, f, indent=1)
