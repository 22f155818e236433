"""Rare paths of the online softmax on the GPU, against the oracle.

A key that dominates the logits of every other query row (and not of the rows between them)
appears only after the first key tile, so within every warp some rows must rescale their
running output and some must not: the warp-collective TMEM accesses of the rescale (and, on
the speculative path, of the exact redo) have to stay correct when only part of a warp needs
them.
"""
import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from tests._oracle_util import f64

pytestmark = pytest.mark.gpu


def _spiked_inputs(d, n_img, n_txt, heads, spike_rows, seed=3):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, n_img, heads, d, generator=g) * 0.3
    k = torch.randn(1, n_img, heads, d, generator=g) * 0.3
    v = torch.randn(1, n_img, heads, d, generator=g)
    kt = torch.randn(1, n_txt, heads, d, generator=g) * 0.3
    vt = torch.randn(1, n_txt, heads, d, generator=g)
    # even query rows carry a component along axis 0, odd rows none; the spike keys are
    # large along axis 0: scaled logit 3 * 40 / sqrt(d) >= 10 (natural units) above the rest
    q[:, 0::2, :, 0] = 3.0
    q[:, 1::2, :, 0] = 0.0
    for r in spike_rows:
        k[:, r, :, 0] = 40.0
    return [t.bfloat16().cuda() for t in (q, k, v, kt, vt)]


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("d", [64, 72, 128])
def test_rows_of_a_warp_that_rescale_and_rows_that_do_not(d, split):
    n_img, M, T, H = 1024, 2, 40, 2
    P = n_img // M
    q, k, v, kt, vt = _spiked_inputs(d, n_img, T, H, spike_rows=(300,))
    pat = pa.PatchAttention(1, H, d, n_img, M, T, 1, split=split)
    try:
        pat.init_layer(0, k, v)
        keys = np.concatenate([f64(k[0]), f64(kt[0])])
        vals = np.concatenate([f64(v[0]), f64(vt[0])])
        vmax = float(np.abs(vals).max())
        scale = d ** -0.5
        for p in range(M):
            sl = slice(p * P, (p + 1) * P)
            o = pat.step(0, p, q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), kt, vt)
            got = f64(o[0])
            ref = oracle.attend(f64(q[0, sl]), keys, vals, scale)
            # the spike dominates the even rows: their output is close to the spike's value
            assert np.abs(ref[0::2] - vals[300][None]).max() < 0.05 * vmax
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (p, rel)
            assert np.abs(got - ref).max() <= 2e-2 * vmax, p
        pat.check()
    finally:
        pat.close()
