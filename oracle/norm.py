"""Per-head RMS normalisation (QK-norm), fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Not described on the pages (they name the models -- SD3, Flux.1 -- whose attention uses it);
the plain definition is used: for every head vector x of length d,
    y = x / sqrt(mean(x^2) + eps) * gain.
"""
from __future__ import annotations

import numpy as np


def rms_normalize(x: np.ndarray, gain=None, eps: float = 1e-6) -> np.ndarray:
    """x: [..., d] -> same shape, float64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if gain is not None:
        y = y * np.asarray(gain, dtype=np.float64)
    return y
