"""fp64 reference of the GDN output tail -- TEST INFRASTRUCTURE ONLY.

Page "ARCHITECTURE PREVIEW / FIELD NOTES", section 03 (figure caption): the state readout y
passes a normalisation and an output gate before the output projection; the page gives no
formula.  Plainest reading, written out here from its definition: per (token, V head) the
128 values of y are RMS-normalised, scaled by a per-channel weight w shared by the heads,
and gated by SiLU of the gate input z of that token and head:

    o = y / sqrt(mean(y^2) + eps) * w * z * sigmoid(z)

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU leg may use it.
"""
from __future__ import annotations

import numpy as np


def output_gate(y, z, w, eps: float = 1e-6):
    """y, z [..., 128] (any float dtype, widened to fp64), w [128] -> o [..., 128] fp64."""
    y = np.asarray(y, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ms = np.mean(y * y, axis=-1, keepdims=True)
    gate = z / (1.0 + np.exp(-z))          # SiLU(z) = z sigmoid(z)
    return y / np.sqrt(ms + eps) * w * gate
