"""Hybrid-CFG switching controller: the oracle pinned by hand-worked sequences, and the C
controller (pf_switch_init / pf_switch_update, host only) equal to the oracle."""
import math

import numpy as np
import pytest

import patch_attention_b200 as pa
from oracle import switching as sw


def test_oracle_hand_worked_sequences():
    # rel-MAE 0.9, 0.6, 0.4, 0.3, 0.2, 0.5 with enter_below 0.45, patience 2:
    # steps 2 and 3 are the first two consecutive values <= 0.45 -> tau1 = 4;
    # exit_above 0.45: step 5 (value 0.5) run in Parallelism -> tau2 = 6
    r = [0.9, 0.6, 0.4, 0.3, 0.2, 0.5]
    assert sw.switch_points(r, 0.45, 2, 0.45) == (4, 6)
    assert sw.phases(r, 0.45, 2, 0.45) == [0, 0, 0, 0, 1, 1, 2]
    # patience 1 enters right after the first low value
    assert sw.switch_points(r, 0.45, 1) == (3, -1)
    # parallel step budget: 2 steps of Parallelism then Fully-Connecting
    assert sw.switch_points(r, 0.45, 1, math.inf, 2) == (3, 5)
    # a dip that does not last resets the patience counter
    assert sw.switch_points([0.4, 0.9, 0.4, 0.4], 0.45, 2) == (4, -1)
    # never below the threshold: Warm-Up throughout
    assert sw.switch_points([0.9, 0.8], 0.1) == (-1, -1)
    assert sw.phases([0.9, 0.8], 0.1) == [0, 0, 0]


def _run_c(r, *args):
    s = pa.HybridCfgSwitch(*args)
    out = [s.phase]
    for x in r:
        out.append(s.update(x))
    return out, s.tau


@pytest.mark.parametrize("seed", range(20))
def test_c_controller_equals_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    # a decaying series with noise and occasional rebounds, like rel-MAE over a sweep
    r = list(np.clip(np.linspace(1.0, 0.05, n) + rng.normal(0, 0.1, n), 0, None).astype(np.float32))
    r = [float(x) for x in r]
    enter = float(np.float32(rng.uniform(0.1, 0.8)))
    patience = int(rng.integers(1, 4))
    exit_above = float(np.float32(rng.uniform(0.2, 1.5))) if seed % 3 else math.inf
    budget = int(rng.integers(0, 20))
    got, tau = _run_c(r, enter, patience, exit_above, budget)
    assert got == sw.phases(r, enter, patience, exit_above, budget)
    assert tau == sw.switch_points(r, enter, patience, exit_above, budget)


def test_sweep_from_the_guidance_schedule():
    # rel-MAE_t follows s_t (1.0 -> 0.05 over 50 steps): with enter_below 0.5 and patience 1
    # the switch happens right after the first step with s_t <= 0.5
    s = [1.0 - 0.95 * t / 49 for t in range(50)]
    first = next(t for t, v in enumerate(s) if v <= 0.5)
    got, tau = _run_c(s, 0.5, 1, math.inf, 0)
    assert tau == (first + 1, -1)
    assert got[first] == pa.PF_PHASE_WARMUP and got[first + 1] == pa.PF_PHASE_PARALLEL


def test_controller_argument_checks():
    with pytest.raises(pa.PatchAttnError):
        pa.HybridCfgSwitch(float("nan"))
    with pytest.raises(pa.PatchAttnError):
        pa.HybridCfgSwitch(0.5, enter_patience=0)
    s = pa.HybridCfgSwitch(0.5)
    with pytest.raises(pa.PatchAttnError):
        s.update(float("nan"))
    assert s.state.step == 0
