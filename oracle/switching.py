"""Hybrid-CFG adaptive switching, restated as a plain function of the rel-MAE_t series.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"조건부 가이드 스케줄링 기반 하이브리드 데이터-파이프라인 병렬 처리를 통한 디퓨전 모델 가속화",
second block 단락 2-3: the denoising steps are split into Warm-Up, Parallelism and
Fully-Connecting; the switch points tau1, tau2 are set by rel-MAE_t, and parallelism is used
while rel-MAE_t has settled below a threshold.  The pages give no thresholds; the reading
used here takes them as parameters:
  tau1 = first step t+1 such that rel-MAE_s <= enter_below for the `enter_patience` steps
         s = t-enter_patience+1 .. t (all observed in Warm-Up);
  tau2 = first step t+1 >= tau1 + 1 such that, for the step t run in Parallelism,
         rel-MAE_t >= exit_above, or t+1 - tau1 >= max_parallel_steps (if > 0).
The phase that applies to step t is Warm-Up for t < tau1, Parallelism for tau1 <= t < tau2,
Fully-Connecting for t >= tau2.
"""
from __future__ import annotations

import math
from typing import List, Tuple

WARMUP, PARALLEL, FULL = 0, 1, 2


def switch_points(relmae: List[float], enter_below: float, enter_patience: int = 1,
                  exit_above: float = math.inf, max_parallel_steps: int = 0) -> Tuple[int, int]:
    """(tau1, tau2), -1 where the switch never happens within the series."""
    tau1 = -1
    for t in range(len(relmae)):
        lo = t - enter_patience + 1
        if lo >= 0 and all(r <= enter_below for r in relmae[lo:t + 1]):
            tau1 = t + 1
            break
    if tau1 < 0:
        return -1, -1
    tau2 = -1
    for t in range(tau1, len(relmae)):
        n_parallel = t + 1 - tau1
        if relmae[t] >= exit_above or (max_parallel_steps > 0 and n_parallel >= max_parallel_steps):
            tau2 = t + 1
            break
    return tau1, tau2


def phases(relmae: List[float], *args, **kw) -> List[int]:
    """Phase that applies to each step t = 0 .. len(relmae) (one more than observed)."""
    tau1, tau2 = switch_points(relmae, *args, **kw)
    out = []
    for t in range(len(relmae) + 1):
        if tau1 < 0 or t < tau1:
            out.append(WARMUP)
        elif tau2 < 0 or t < tau2:
            out.append(PARALLEL)
        else:
            out.append(FULL)
    return out
