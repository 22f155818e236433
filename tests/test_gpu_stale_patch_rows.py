"""The buffer rows of patch p are never read by patch p's own call.

When patch p of a step is computed, its rows of the layer buffer still hold the previous
step and are replaced by the call's fresh K_p/V_p ("기술 요약: PipeFusion", 핵심 메커니즘 2:
patch p's own rows are the fresh activations); the same launch writes them.  Here those stale
rows are made non-finite just before the call, with a patch length (200) that is not a
multiple of the 128-row context tile, so the last tile of the rows before the patch reaches
into the patch's rows.  The oracle never uses them, so the output must stay finite and match
it: a kernel that read them (even under a softmax weight of 0, as 0 * inf) would produce NaN.
With two buffer halves the rows of patch p in both halves are made non-finite.
"""
import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from tests._oracle_util import f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("split,schedule", [(True, pa.PF_SCHED_PIPEFUSION), (False, pa.PF_SCHED_PIPEFUSION),
                                            (True, pa.PF_SCHED_PIPEFUSION_2H)])
@pytest.mark.parametrize("d", [64, 72, 128])
def test_stale_rows_of_the_patch_are_never_read(d, split, schedule):
    B, H, N, M, T = 1, 2, 600, 3, 10
    P = N // M
    g = torch.Generator(device="cuda").manual_seed(11)
    mk = lambda *s: torch.randn(*s, device="cuda", generator=g).bfloat16()
    k0, v0 = mk(B, N, H, d), mk(B, N, H, d)               # step 0: the buffer's start
    q1, k1, v1 = mk(B, N, H, d), mk(B, N, H, d), mk(B, N, H, d)  # step 1
    kt, vt = mk(B, T, H, d), mk(B, T, H, d)
    pat = pa.PatchAttention(B, H, d, N, M, T, 1, split=split, schedule=schedule)
    prev_k, prev_v = f64(k0[0]), f64(v0[0])
    try:
        pat.init_layer(0, k0, v0)
        rd = pat.read_half(0)
        kb, vb = pat.buffer_kv(0, rd)
        two = schedule == pa.PF_SCHED_PIPEFUSION_2H
        # with two halves the call writes into the other half; its rows of patch p are stale
        # too (from the step before the previous one, here never written)
        kw, vw = pat.buffer_kv(0, 1 - rd) if two else (kb, vb)
        for p in range(M):
            sl = slice(p * P, (p + 1) * P)
            for t in (kb, vb, kw, vw):
                t[:, sl] = float("inf")
            prev_k[sl] = np.inf
            prev_v[sl] = np.inf
            o = pat.step(0, p, q1[:, sl].contiguous(), k1[:, sl].contiguous(), v1[:, sl].contiguous(),
                         kt, vt)
            got = f64(o[0])
            assert np.all(np.isfinite(got)), f"patch {p}: non-finite output"
            ref = oracle.patch_attention(f64(q1[0]), f64(k1[0]), f64(v1[0]), prev_k, prev_v,
                                         f64(kt[0]), f64(vt[0]), p, M, d ** -0.5)
            assert np.all(np.isfinite(ref))
            vmax = max(float(np.abs(f64(v1[0, :(p + 1) * P])).max()),
                       float(np.abs(prev_v[(p + 1) * P:]).max()) if p + 1 < M else 0.0,
                       float(np.abs(f64(vt[0])).max()))
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (p, rel)
            assert np.abs(got - ref).max() <= 2e-2 * vmax, p
            # the call replaced the patch's rows with the fresh ones, bit for bit (in the half
            # being written)
            assert torch.equal(kw[:, sl].view(torch.int16), k1[:, sl].view(torch.int16))
            assert torch.equal(vw[:, sl].view(torch.int16), v1[:, sl].view(torch.int16))
        pat.check()
    finally:
        pat.close()
