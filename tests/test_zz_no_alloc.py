"""The no-allocation guidance entry point (pf_cfg_combine_relmae_static) against the
workspace entry point (pf_cfg_combine_relmae) and the fp64 oracle, through the C ABI.

Some callers cannot allocate device memory at the moment they run the guidance step: the
device allocator belongs to another framework that must account for every allocation, or
the loop cannot afford the synchronisation an allocation may imply.  For them the library
keeps the kernel's partial sums in a fixed array of its own.  This file is collected last
so that a run stopping at its first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from patch_attention_b200 import synth

pytestmark = pytest.mark.gpu

REL_TOL = 1e-5  # rel-MAE, as in the other guidance tests


def _reference(c, u, w):
    return pa.cfg_combine_relmae(c, u, w)


def _static(c, u, w):
    B = c.shape[0]
    out_f = torch.empty_like(c)
    out_b = torch.empty(c.shape, dtype=torch.bfloat16, device=c.device)
    rel = torch.full((B,), float("nan"), dtype=torch.float32, device=c.device)
    pa.pf_cfg_combine_relmae_static(c, u, w, out_f, out_b, rel)
    return out_f, out_b, rel


def _compare(got, ref, c, u, w):
    gf, gb, gr = got
    rf, rb, rr = ref
    cn, un = c.double().cpu().numpy(), u.double().cpu().numpy()
    bound = 2.0 ** -22 * (np.abs(un) + abs(w) * np.abs(cn - un)) + 1e-30
    assert np.all(np.abs(gf.double().cpu().numpy() - rf.double().cpu().numpy()) <= bound)
    ref_b = rb.double().cpu().numpy()
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref_b), 1e-30))) - 7)
    assert np.all(np.abs(gb.double().cpu().numpy() - ref_b) <= ulp * 1.0001)
    r, q = gr.double().cpu().numpy(), rr.double().cpu().numpy()
    assert np.all(np.isfinite(r))
    assert np.all(np.abs(r - q) <= REL_TOL * np.abs(q) + 1e-30), (r, q)


def test_static_entry_matches_workspace_entry_two_calls():
    # two calls in a row with different shapes and batches: the second reuses the array the
    # first one left behind
    w = 7.0
    first = synth.CfgInputs(synth.CfgWorkload("cfg", 4, 16, 512, 512), device="cuda").step_tensors(3)
    second = synth.CfgInputs(synth.CfgWorkload("cfg", 2, 4, 128, 128), device="cuda").step_tensors(40)
    for c, u in (first, second):
        got = _static(c, u, w)
        torch.cuda.synchronize()
        _compare(got, _reference(c, u, w), c, u, w)


def _compare_with_oracle(got, c, u, w):
    # same bounds as the workspace entry point's oracle tests: fp32 out within one rounding of
    # c - u and one fused multiply-add, bf16 out within one bf16 ulp, rel-MAE within 1e-5
    gf, gb, gr = got
    B = c.shape[0]
    cn, un = c.double().cpu().numpy(), u.double().cpu().numpy()
    ref = oracle.cfg_combine(cn, un, w)
    _, _, rref = oracle.rel_mae(cn.reshape(B, -1), un.reshape(B, -1))
    bound = 2.0 ** -22 * (np.abs(un) + abs(w) * np.abs(cn - un)) + 1e-30
    assert np.all(np.abs(gf.double().cpu().numpy() - ref) <= bound)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(gb.double().cpu().numpy() - ref) <= ulp * 1.0001)
    r = gr.double().cpu().numpy()
    assert np.all(np.abs(r - rref) <= REL_TOL * np.abs(rref) + 1e-30), (r, rref)


def test_static_entry_matches_the_oracle_two_calls():
    # two calls in a row (the second on a smaller batch, over the array the first one left)
    w = 7.0
    for B, shape, t in ((3, (4, 128, 128), 10), (1, (16, 64, 64), 45)):
        c, u = synth.CfgInputs(synth.CfgWorkload("cfg", B, *shape), device="cuda").step_tensors(t)
        got = _static(c, u, w)
        torch.cuda.synchronize()
        _compare_with_oracle(got, c, u, w)


def test_static_entry_rejects_batches_beyond_the_array():
    c = torch.zeros(4097, 4, device="cuda")
    rel = torch.empty(4097, device="cuda")
    with pytest.raises(pa.PatchAttnError) as e:
        pa.pf_cfg_combine_relmae_static(c, c, 7.0, None, None, rel)
    assert e.value.status == pa.PF_ERR_SHAPE
