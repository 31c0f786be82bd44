"""fp64 oracle of the mixer's output epilogue -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the bench's CPU legs may use it; the CUDA
library shares no code with it.

Source: page "GLM-5.3-Flash Internals -- a measured profile", section
"Findings" (the site catalog: the KDA input projections, among them
``g_b_proj``, sit before the mixer, and ``o_norm`` / ``o_proj`` after it).  The
pages name these modules only; the plain reading taken here is

    y[t, h, :] = o[t, h, :] / sqrt(mean_c o[t, h, c]^2 + eps) * w * sigmoid(z[t, h, :])

an RMS normalisation over each head's 128 value channels with a learnt
per-channel weight w (shared by the heads), gated channel-wise by the sigmoid
of the ``g_b_proj`` output z of the same token and head.  ``o_proj`` is the
dense projection that follows and is not part of this function.

Pinned (``tests/test_epilogue_oracle.py``) by: the library RMS normalisation
(``torch.nn.functional.rms_norm``) at a saturated gate; scale invariance per
(token, head) at eps = 0; unit RMS of y / (w sigmoid(z)) at eps = 0; the
gate's closed forms (sigmoid(0) = 1/2, sigmoid(-z) = 1 - sigmoid(z), and the
library logistic function); a hand-worked two-channel case.
"""
from __future__ import annotations

import numpy as np


def sigmoid(z: np.ndarray) -> np.ndarray:
    """The logistic function 1 / (1 + e^-z), fp64, without overflow for |z| large."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gated_rmsnorm(o: np.ndarray, z: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """o, z [..., d] (any leading shape), w [d] -> y [..., d] in fp64.

    The mean of squares runs over the last axis (one head's value channels)."""
    o = np.asarray(o, dtype=np.float64)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + float(eps)) * np.asarray(w, dtype=np.float64) * sigmoid(z)
