"""fp64 oracle of the span-state combination of a context-parallel prefill -- TEST
INFRASTRUCTURE ONLY (only tests/, the package's smoke check and bench.py's CPU legs may use it).

Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (GATED DELTANET equations): each token
maps the state affinely, S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, so a
span of tokens maps it affinely too, S_out = M S_in + B.  Given the maps of consecutive spans,
the state entering span p is S_in[0] = S0, S_in[p+1] = M[p] S_in[p] + B[p]; this module writes
that recurrence out, one span after another, in float64 (numpy's matmul as the step).
Pinned in tests/test_context_parallel_cpu.py: with the oracle's own span maps, the combined
states re-run span by span reproduce the oracle over the whole sequence.
"""
from __future__ import annotations

import numpy as np


def affine_prefix(M, B, S0=None):
    """States entering each span and the state after the last one.

    M, B: [P, Hv, dk, dk] and [P, Hv, dk, dv]; S0: [Hv, dk, dv] or None (zero).
    Returns [P + 1, Hv, dk, dv] float64.
    """
    M = np.asarray(M, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    P = M.shape[0]
    S = np.zeros(B.shape[1:]) if S0 is None else np.asarray(S0, dtype=np.float64)
    out = [S]
    for p in range(P):
        S = np.matmul(M[p], S) + B[p]
        out.append(S)
    return np.stack(out)
