"""Exact rational arithmetic of the gated delta rule on tiny inputs -- TEST INFRASTRUCTURE.

It follows the expanded one-step recurrence printed on the page "ARCHITECTURE
PREVIEW / FIELD NOTES" (section 03, the equation under "GATED DELTANET"):
    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
    y_t = S_t^T q_t,
with every quantity a ``fractions.Fraction``, so the result carries no rounding
at all.  It serves only to write ``tests/golden/`` fixtures against which the fp64
oracle (which uses the four-equation form) is pinned.
"""
from __future__ import annotations

from fractions import Fraction


def _mat(rows, cols, val=Fraction(0)):
    return [[Fraction(val) for _ in range(cols)] for _ in range(rows)]


def one_step_exact(S0, ks, vs, qs, alphas, betas):
    """S0 [dk][dv]; ks, qs: lists of dk-vectors; vs: list of dv-vectors; scalars per step.

    Returns (ys, S_T) with ys a list of dv-vectors.  All entries are Fractions.
    """
    dk, dv = len(S0), len(S0[0])
    S = [[Fraction(x) for x in row] for row in S0]
    ys = []
    for k, v, q, a, b in zip(ks, vs, qs, alphas, betas):
        k = [Fraction(x) for x in k]
        v = [Fraction(x) for x in v]
        q = [Fraction(x) for x in q]
        a, b = Fraction(a), Fraction(b)
        # transition matrix alpha (I - beta k k^T), d_k x d_k
        M = _mat(dk, dk)
        for i in range(dk):
            for j in range(dk):
                M[i][j] = a * ((1 if i == j else 0) - b * k[i] * k[j])
        new = _mat(dk, dv)
        for i in range(dk):
            for j in range(dv):
                acc = sum((M[i][m] * S[m][j] for m in range(dk)), Fraction(0))
                new[i][j] = acc + b * k[i] * v[j]
        S = new
        ys.append([sum((S[i][j] * q[i] for i in range(dk)), Fraction(0)) for j in range(dv)])
    return ys, S
