"""Classifier-free-guidance combine and rel-MAE_t, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* The two guidance paths (conditional eps_c, unconditional eps_u) are those of
  "조건부 가이드 스케줄링 기반 하이브리드 데이터-파이프라인 병렬 처리를 통한 디퓨전 모델 가속화",
  first block 단락 1 and second block 단락 1.  The pages do not print the combine; the
  plain reading used here is the standard guided prediction eps_u + w (eps_c - eps_u).
* rel-MAE_t -- same page, second block 단락 2-3: the L1 norm of the difference of the two
  noise predictions divided by the L1 norm of the unconditional prediction.  It is taken
  per sample (each image has its own switching schedule).  Zero denominator: 0 when the
  numerator is 0 too, else +inf.
"""
from __future__ import annotations

import math

import numpy as np


def cfg_combine(eps_c: np.ndarray, eps_u: np.ndarray, w: float) -> np.ndarray:
    """Guided prediction eps_u + w * (eps_c - eps_u), in float64."""
    c = np.asarray(eps_c, dtype=np.float64)
    u = np.asarray(eps_u, dtype=np.float64)
    return u + w * (c - u)


def _l1(x: np.ndarray) -> float:
    # exactly rounded sum of |x| (math.fsum), so the oracle carries no summation-order error
    return math.fsum(np.abs(x).ravel().tolist()) if x.size < 1 << 16 else _l1_blocked(x)


def _l1_blocked(x: np.ndarray) -> float:
    # fsum over fp64 block partials: each partial is a pairwise numpy sum of <= 4096 terms
    a = np.abs(x).ravel()
    parts = [float(np.sum(a[i:i + 4096])) for i in range(0, a.size, 4096)]
    return math.fsum(parts)


def rel_mae(eps_c: np.ndarray, eps_u: np.ndarray):
    """Per-sample (num, den, rel) with num = ||c-u||_1, den = ||u||_1, rel = num / den.

    eps_c, eps_u: [B, ...]; returns three float64 arrays of shape [B].
    """
    c = np.asarray(eps_c, dtype=np.float64)
    u = np.asarray(eps_u, dtype=np.float64)
    B = c.shape[0]
    num = np.array([_l1(c[b] - u[b]) for b in range(B)])
    den = np.array([_l1(u[b]) for b in range(B)])
    rel = np.empty(B)
    for b in range(B):
        if den[b] == 0.0:
            rel[b] = 0.0 if num[b] == 0.0 else math.inf
        else:
            rel[b] = num[b] / den[b]
    return num, den, rel


def cfg_combine_relmae(eps_c, eps_u, w):
    """(guided eps, rel-MAE per sample), both float64."""
    return cfg_combine(eps_c, eps_u, w), rel_mae(eps_c, eps_u)[2]
