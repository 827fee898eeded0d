"""Writes ``brute_tiny.json``: an exact worked example of the KDA recurrence.

The source pages print no worked example, so this fixture is computed from the
definition itself -- the delta-rule update with a channel-wise forget gate,
S <- (I - beta k k^T) Diag(alpha) S + beta k v^T, o = S^T q (KimiLinear KDA/MLA
tutorial (icman.com.cn), sec. 2 and sec. 5; "Kimi Linear" article (jdon.com),
on KDA's fine-grained gates) -- in exact rational arithmetic by
``oracle/brute.py`` (explicit transition-matrix products, no state stepping).

Shape: two packed sequences (lengths 3 and 2, cu_seqlens [0, 3, 5]), two
heads, d_k = 3, d_v = 2 (non-square, so a transposed state or operand shows),
rational unit keys, rational alpha per channel, beta in [0, 1], nonzero S0.
Run from the repository root: ``python tests/golden/make_golden.py``.
"""
from __future__ import annotations

import json
import os
import sys
from fractions import Fraction as F

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "..", ".."))
from oracle import brute  # noqa: E402

CU = [0, 3, 5]
H, DK, DV = 2, 3, 2
# per packed token t and head h
KEYS = [
    [[F(3, 5), F(4, 5), F(0)], [F(2, 3), F(1, 3), F(2, 3)]],
    [[F(0), F(3, 5), F(4, 5)], [F(2, 7), F(3, 7), F(6, 7)]],
    [[F(2, 3), F(2, 3), F(1, 3)], [F(4, 5), F(0), F(-3, 5)]],
    [[F(1), F(0), F(0)], [F(0), F(-4, 5), F(3, 5)]],
    [[F(6, 7), F(2, 7), F(-3, 7)], [F(1, 3), F(2, 3), F(-2, 3)]],
]
ALPHA = [
    [[F(1, 2), F(3, 4), F(1)], [F(7, 8), F(1, 2), F(5, 8)]],
    [[F(9, 10), F(1), F(1, 4)], [F(1), F(3, 4), F(1, 2)]],
    [[F(3, 4), F(5, 8), F(7, 8)], [F(1, 2), F(1), F(9, 10)]],
    [[F(1, 2), F(1, 2), F(1)], [F(3, 4), F(7, 8), F(1, 4)]],
    [[F(1), F(9, 10), F(3, 4)], [F(5, 8), F(1, 2), F(1)]],
]
BETA = [[F(1, 2), F(1)], [F(1, 3), F(0)], [F(3, 4), F(1, 2)], [F(1), F(2, 3)], [F(1, 4), F(3, 4)]]
Q = [
    [[F(1), F(-1, 2), F(2)], [F(1, 3), F(1), F(-1)]],
    [[F(-1), F(2), F(1, 2)], [F(2), F(0), F(1, 4)]],
    [[F(1, 2), F(1, 2), F(-3, 2)], [F(-1), F(-1, 3), F(1)]],
    [[F(3), F(1), F(0)], [F(1, 2), F(-2), F(1)]],
    [[F(0), F(-1), F(1)], [F(1), F(1), F(1)]],
]
V = [
    [[F(1), F(-2)], [F(3, 2), F(1, 2)]],
    [[F(-1, 2), F(1)], [F(2), F(-1)]],
    [[F(2), F(3)], [F(-1), F(1, 4)]],
    [[F(1, 3), F(-1)], [F(1), F(2)]],
    [[F(-2), F(1, 2)], [F(0), F(-3, 4)]],
]
S0 = [  # [n][h] d_k x d_v
    [[[F(1, 2), F(0)], [F(-1), F(1, 4)], [F(0), F(2)]],
     [[F(0), F(1)], [F(1, 3), F(0)], [F(-1, 2), F(1, 2)]]],
    [[[F(1), F(1)], [F(0), F(-1)], [F(1, 4), F(0)]],
     [[F(-2), F(0)], [F(0), F(1, 2)], [F(1), F(-1, 3)]]],
]


def fr(x: F) -> str:
    return "%d/%d" % (x.numerator, x.denominator)


def main():
    out = [[None] * H for _ in range(CU[-1])]
    S_final = [[None] * H for _ in range(len(CU) - 1)]
    for n in range(len(CU) - 1):
        t0, t1 = CU[n], CU[n + 1]
        for h in range(H):
            outs, S = brute.sequence([Q[t][h] for t in range(t0, t1)],
                                     [KEYS[t][h] for t in range(t0, t1)],
                                     [V[t][h] for t in range(t0, t1)],
                                     [ALPHA[t][h] for t in range(t0, t1)],
                                     [BETA[t][h] for t in range(t0, t1)], S0[n][h])
            for i, t in enumerate(range(t0, t1)):
                out[t][h] = [fr(x) for x in outs[i]]
            S_final[n][h] = [[fr(x) for x in r] for r in S]
    rec = lambda a: [rec(x) for x in a] if isinstance(a, list) else fr(a)  # noqa: E731
    doc = {
        "about": "Exact KDA recurrence, computed in rational arithmetic from the definition "
                 "(delta rule with channel-wise forget gate: KimiLinear KDA/MLA tutorial "
                 "(icman.com.cn) sec. 2 and 5; 'Kimi Linear' article (jdon.com)). "
                 "Layouts: tokens packed [T][H][d], cu_seqlens offsets, S0/S_final [N][H][dk][dv].",
        "cu_seqlens": CU, "H": H, "dk": DK, "dv": DV,
        "k": rec(KEYS), "alpha": rec(ALPHA), "beta": rec(BETA), "q": rec(Q), "v": rec(V),
        "S0": rec(S0), "out": out, "S_final": S_final,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "brute_tiny.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
