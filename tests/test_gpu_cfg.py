"""GPU parity of the fused guidance combine + rel-MAE kernel against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from patch_attention_b200 import synth

pytestmark = pytest.mark.gpu

REL_TOL = 1e-5


def _check(c, u, w, out_f, out_b, rel):
    cn, un = c.double().cpu().numpy(), u.double().cpu().numpy()
    B = c.shape[0]
    ref = oracle.cfg_combine(cn, un, w)
    _, _, rref = oracle.rel_mae(cn.reshape(B, -1), un.reshape(B, -1))
    # fp32 output: one rounding of c-u, one fused multiply-add
    if out_f is not None:
        got = out_f.double().cpu().numpy()
        bound = 2.0 ** -22 * (np.abs(un) + abs(w) * np.abs(cn - un)) + 1e-30
        assert np.all(np.abs(got - ref) <= bound)
    if out_b is not None:
        got_b = out_b.double().cpu().numpy()
        # within one bf16 ulp of the exact value
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
        assert np.all(np.abs(got_b - ref) <= ulp * 1.0001)
    r = rel.double().cpu().numpy()
    assert np.all(np.abs(r - rref) <= REL_TOL * np.abs(rref) + 1e-30), (r, rref)


@pytest.mark.parametrize("shape", synth.CFG_SHAPES)
@pytest.mark.parametrize("batch", [1, 2, 3, 4])
def test_cfg_sweep_sizes(shape, batch):
    wl = synth.CfgWorkload("cfg", batch, *shape)
    gen = synth.CfgInputs(wl, device="cuda")
    for t in (0, 25, 49):
        c, u = gen.step_tensors(t)
        out_f, out_b, rel = pa.cfg_combine_relmae(c, u, wl.w)
        _check(c, u, wl.w, out_f, out_b, rel)


def test_cfg_full_sweep_50_steps_largest():
    wl = synth.CfgWorkload("cfg", 1, 16, 512, 512)
    gen = synth.CfgInputs(wl, device="cuda")
    series = []
    for t in range(wl.n_steps):
        c, u = gen.step_tensors(t)
        _, out_b, rel = pa.cfg_combine_relmae(c, u, wl.w, want_f32=False)
        cn, un = c.double().cpu().numpy(), u.double().cpu().numpy()
        _, _, rref = oracle.rel_mae(cn.reshape(1, -1), un.reshape(1, -1))
        assert abs(rel.item() - rref[0]) <= REL_TOL * rref[0]
        series.append(rel.item())
    # rel-MAE tracks s_t (eps_c = eps_u + s_t z): monotone decreasing over the sweep
    assert all(a > b for a, b in zip(series, series[1:]))


def test_cfg_outputs_optional_and_identities():
    g = torch.Generator(device="cuda").manual_seed(0)
    u = torch.randn(2, 4096, device="cuda", generator=g)
    c = torch.randn(2, 4096, device="cuda", generator=g)
    f, b, rel = pa.cfg_combine_relmae(u.clone(), u, 7.0)
    assert torch.equal(f, u) and torch.all(rel == 0)
    f, _, _ = pa.cfg_combine_relmae(c, u, 0.0, want_bf16=False)
    assert torch.equal(f, u)
    _, b, rel = pa.cfg_combine_relmae(c, u, 1.0, want_f32=False)
    _check(c, u, 1.0, None, b, rel)


def test_cfg_deterministic():
    g = torch.Generator(device="cuda").manual_seed(1)
    u = torch.randn(3, 16 * 256 * 256, device="cuda", generator=g)
    c = u + 0.3 * torch.randn(3, 16 * 256 * 256, device="cuda", generator=g)
    r1 = pa.cfg_combine_relmae(c, u, 7.0)
    r2 = pa.cfg_combine_relmae(c, u, 7.0)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)


def test_cfg_zero_denominator():
    u = torch.zeros(2, 64, device="cuda")
    c = torch.zeros(2, 64, device="cuda")
    c[1, 3] = 1.0
    _, _, rel = pa.cfg_combine_relmae(c, u, 7.0)
    assert rel[0].item() == 0.0 and math.isinf(rel[1].item())
