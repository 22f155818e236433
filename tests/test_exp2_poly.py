"""Pin of the attention kernel's FMA-pipe 2^x (exp2_poly2 in csrc/attn_fwd.cu), on the CPU.

The kernel's four polynomial constants are read from its source, and its fp32 steps are
replayed here with numpy: the clamp at -125, the 1.5 * 2^23 shifter that rounds x to the
nearest integer n, the exact remainder f = x - n, the cubic in Horner form with fused
multiply-adds, and the integer add of n into the exponent field.  Checked against
math.exp2: the stated maximum relative error (7.5e-5) on [-1/2, 1/2], the same bound after
the exponent add over [-125, 8], and that inputs below -125 (including -inf) give a tiny
positive normal number rather than a wrapped exponent.  The constants themselves are
re-derived by the Lawson fit in tests/golden/fit_exp2_poly.py.
"""
import math
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "patch_attention_b200", "csrc", "attn_fwd.cu")
sys.path.insert(0, os.path.join(ROOT, "tests", "golden"))

from fit_exp2_poly import lawson_fit  # noqa: E402

SHIFTER = np.float32(12582912.0)  # 1.5 * 2^23
BOUND = 7.5e-5


def kernel_constants():
    """(c3, c2, c1, c0) of the Horner chain, in the order the kernel applies them."""
    src = open(SRC).read()
    body = re.search(r"float2 exp2_poly2\(float2 x\) \{(.*?)\n\}", src, re.S).group(1)
    # constants below 1 in the order they appear: c3, c2 (first Horner step), c1, c0; the
    # shifter 1.5 * 2^23 is excluded
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    vals = [v for v in vals if v < 1.0]
    assert len(vals) == 4, vals
    return [np.float32(v) for v in vals]


def fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in fp64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_replay(x):
    c3, c2, c1, c0 = kernel_constants()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + SHIFTER).astype(np.float32)
    r = (t - SHIFTER).astype(np.float32)
    f = fma32(r, np.full_like(r, -1.0), x)
    p = fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = fma32(p, f, np.full_like(f, c1))
    p = fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32), f


def test_polynomial_error_on_the_reduced_interval():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    y, fr = exp2_poly_replay(f)
    assert np.array_equal(fr, f)  # |f| <= 1/2 rounds to n = 0
    ref = np.exp2(f.astype(np.float64))
    rel = np.abs(y.astype(np.float64) / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # the bound is tight: the fit equioscillates, so the maximum is close to it
    assert rel.max() >= 0.9 * BOUND


def test_exponent_add_over_the_used_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-125.0, 8.0, 200000),
                        np.arange(-125, 9) + 0.5, np.arange(-125, 9) - 0.5, np.arange(-125, 9)]).astype(np.float32)
    x = x[x >= -125.0]
    y, _ = exp2_poly_replay(x)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    ref = np.array([math.exp2(float(v)) for v in x[:2000]] , dtype=np.float64)
    rel0 = np.abs(y[:2000].astype(np.float64) / ref - 1.0)
    assert rel0.max() <= BOUND
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, (rel.max(), x[np.argmax(rel)])
    # results stay normal fp32 numbers down to the clamp
    assert y.min() >= np.finfo(np.float32).tiny


def test_inputs_below_the_clamp_give_a_tiny_positive_number():
    x = np.array([-125.0, -125.5, -126.0, -150.0, -1e6, -np.inf], dtype=np.float32)
    y, _ = exp2_poly_replay(x)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124)
    assert np.all(y == y[0])


def test_constants_match_the_lawson_fit():
    c, err = lawson_fit()
    assert err <= BOUND
    c3, c2, c1, c0 = [float(v) for v in kernel_constants()]
    for got, want in zip((c0, c1, c2, c3), c):
        assert abs(got - want) <= 2e-6 * max(1.0, abs(want)) + 1e-6, (got, want)
