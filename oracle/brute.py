"""Exact rational brute force of the KDA recurrence (test infrastructure only).

Instead of stepping the state, this forms every transition matrix
``A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)`` explicitly and evaluates the
unrolled product

    S_t = A_t ... A_1 S0 + sum_{i<=t} (A_t ... A_{i+1}) beta_i k_i v_i^T ,   o_t = S_t^T q_t

in ``fractions.Fraction`` arithmetic, so the result is exact. Inputs are
rationals (alpha given directly, not its logarithm). Keys with rational unit
norm (Pythagorean tuples such as (3/5, 4/5, 0)) keep the erase term exactly
norm-preserving, as the unit-norm precondition of the delta erase term asks
(KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 5).

Pure Python; intended for d <= 4 and a handful of tokens.
"""
from __future__ import annotations

from fractions import Fraction as F
from typing import List, Sequence

Mat = List[List[F]]


def _eye(n: int) -> Mat:
    return [[F(int(i == j)) for j in range(n)] for i in range(n)]


def _mm(a: Mat, b: Mat) -> Mat:
    n, m, p = len(a), len(b), len(b[0])
    return [[sum((a[i][l] * b[l][j] for l in range(m)), F(0)) for j in range(p)] for i in range(n)]


def _add(a: Mat, b: Mat) -> Mat:
    return [[x + y for x, y in zip(ra, rb)] for ra, rb in zip(a, b)]


def _outer(x: Sequence[F], y: Sequence[F]) -> Mat:
    return [[xi * yj for yj in y] for xi in x]


def _scale(s: F, a: Mat) -> Mat:
    return [[s * x for x in r] for r in a]


def transition(k: Sequence[F], alpha: Sequence[F], beta: F) -> Mat:
    """A = (I - beta k k^T) Diag(alpha), formed entry by entry."""
    d = len(k)
    erase = _add(_eye(d), _scale(-beta, _outer(k, k)))
    diag = [[alpha[i] if i == j else F(0) for j in range(d)] for i in range(d)]
    return _mm(erase, diag)


def sequence(q, k, v, alpha, beta, S0):
    """One (sequence, head): lists over tokens of d_k / d_v vectors, alpha per channel,
    scalar beta; S0 a d_k x d_v list of lists. Returns (outputs per token, final state)."""
    Tn = len(k)
    dk, dv = len(S0), len(S0[0])
    As = [transition(k[t], alpha[t], beta[t]) for t in range(Tn)]
    outs = []
    S_t = S0
    for t in range(Tn):
        # product A_t ... A_1 applied to S0
        P = _eye(dk)
        for i in range(t, -1, -1):
            P = _mm(P, As[i])
        S_t = _mm(P, S0)
        # writes of tokens i <= t, carried forward by A_t ... A_{i+1}
        for i in range(t + 1):
            R = _eye(dk)
            for j in range(t, i, -1):
                R = _mm(R, As[j])
            S_t = _add(S_t, _mm(R, _scale(beta[i], _outer(k[i], v[i]))))
        outs.append([sum((S_t[r][c] * q[t][r] for r in range(dk)), F(0)) for c in range(dv)])
    return outs, S_t
