"""Pins for the fp64 guidance-combine / rel-MAE oracle (CPU only)."""
import json
import math
import os

import numpy as np

import oracle
from patch_attention_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_case():
    g = json.load(open(os.path.join(GOLDEN, "cfg_case.json")))
    c, u = np.array(g["eps_c"]), np.array(g["eps_u"])
    np.testing.assert_array_equal(oracle.cfg_combine(c, u, g["w"]), np.array(g["out"]))
    num, den, rel = oracle.rel_mae(c, u)
    np.testing.assert_array_equal(num, g["num"])
    np.testing.assert_array_equal(den, g["den"])
    assert rel[0] == g["rel_mae_num"] / g["rel_mae_den"]


def test_equal_paths_give_zero_rel_mae_and_u():
    rng = np.random.default_rng(0)
    u = rng.standard_normal((3, 1000))
    out, rel = oracle.cfg_combine_relmae(u.copy(), u, 7.0)
    np.testing.assert_array_equal(rel, 0.0)
    np.testing.assert_array_equal(out, u)


def test_w0_gives_u_and_w1_gives_c():
    rng = np.random.default_rng(1)
    c, u = rng.standard_normal((2, 500)), rng.standard_normal((2, 500))
    np.testing.assert_array_equal(oracle.cfg_combine(c, u, 0.0), u)
    np.testing.assert_allclose(oracle.cfg_combine(c, u, 1.0), c, rtol=0, atol=1e-15)


def test_linear_in_w():
    rng = np.random.default_rng(2)
    c, u = rng.standard_normal((1, 64)), rng.standard_normal((1, 64))
    for w in (-2.0, 0.5, 3.0, 7.0):
        np.testing.assert_allclose(oracle.cfg_combine(c, u, w) - u, w * (c - u), rtol=1e-14, atol=1e-14)


def test_rel_mae_per_sample_not_pooled():
    u = np.array([[1.0, 1.0], [4.0, 4.0]])
    c = np.array([[2.0, 1.0], [4.0, 4.0]])
    num, den, rel = oracle.rel_mae(c, u)
    np.testing.assert_array_equal(rel, [0.5, 0.0])


def test_zero_denominator():
    u = np.zeros((2, 4))
    c = np.array([[0.0, 0.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]])
    _, _, rel = oracle.rel_mae(c, u)
    assert rel[0] == 0.0 and math.isinf(rel[1])


def test_statistical_closed_form_over_sweep():
    """c = u + s z with u, z iid N(0,1): E|c-u| = s E|z| = s E|u|, so rel-MAE -> s."""
    wl = synth.CfgWorkload("cfg", batch=2, channels=4, height=64, width=64, n_steps=50)
    gen = synth.CfgInputs(wl, seed=5)
    n = wl.n_per_sample
    for t in range(0, 50, 7):
        c, u = gen.step_tensors(t)
        _, _, rel = oracle.rel_mae(c.double().numpy(), u.double().numpy())
        s = wl.s_t(t)
        assert np.all(np.abs(rel - s) <= 5.0 / math.sqrt(n) * max(s, 1.0)), (t, rel, s)


def test_large_sum_accuracy():
    # blocked path (numpy partials + fsum) vs an exact rational reference
    x = np.full((1, 300000), 0.1)
    x[0, ::2] = -0.3
    _, den, _ = oracle.rel_mae(x, x)
    exact = 150000 * 0.1 + 150000 * 0.3  # in exact arithmetic of the fp64 inputs
    from fractions import Fraction
    ref = 150000 * Fraction(0.1) + 150000 * Fraction(0.3)
    assert abs(den[0] - float(ref)) <= 1e-14 * exact
