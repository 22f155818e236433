"""Joint-attention text queries and per-head QK RMS normalisation: oracle pins (CPU), host
argument checks (CPU) and GPU parity."""
import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from oracle.norm import rms_normalize
from patch_attention_b200 import synth
from tests._oracle_util import f64

FAKE = 0x7F0000000000


# ---------------------------------------------------------------- oracle pins (CPU)


def test_rms_normalize_closed_forms():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 3, 64)) * 3.0
    y = rms_normalize(x, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)  # unit RMS
    np.testing.assert_allclose(rms_normalize(7.5 * x, eps=0.0), y, rtol=1e-13)      # scale free
    g = rng.standard_normal(64)
    np.testing.assert_allclose(rms_normalize(x, g, eps=0.0), y * g, rtol=1e-14)     # gain
    c = np.full((1, 4), 2.0)                                                        # constant
    np.testing.assert_allclose(rms_normalize(c, eps=0.0), 1.0, rtol=1e-15)
    z = np.zeros((1, 8))
    np.testing.assert_array_equal(rms_normalize(z, eps=1e-6), 0.0)                  # eps guards 0
    # eps enters as mean + eps: x = (1,1,1,1), eps = 3 -> 1 / sqrt(4)
    np.testing.assert_allclose(rms_normalize(np.ones((1, 4)), eps=3.0), 0.5, rtol=1e-15)


# ---------------------------------------------------------------- host checks (CPU)


def test_host_argument_checks():
    L = pa._lib()
    assert L.pf_qk_rmsnorm(None, 4, 64, None, 1e-6, None) == pa.PF_ERR_INVALID_ARG
    assert L.pf_qk_rmsnorm(FAKE, 4, 60, None, 1e-6, None) == pa.PF_ERR_SHAPE
    assert L.pf_qk_rmsnorm(FAKE, 4, 264, None, 1e-6, None) == pa.PF_ERR_SHAPE
    assert L.pf_qk_rmsnorm(FAKE, 4, 64, None, 0.0, None) == pa.PF_ERR_INVALID_ARG
    assert L.pf_qk_rmsnorm(FAKE + 8, 4, 64, None, 1e-6, None) == pa.PF_ERR_ALIGN
    cfg = pa.make_config(1, 2, 64, 256, 4, 0, 1)
    ctx = pa.pf_create(cfg, [FAKE])
    try:
        assert L.pf_text_attn_step(ctx, 0, FAKE, FAKE, FAKE, FAKE, None) == pa.PF_ERR_SHAPE
    finally:
        pa.pf_destroy(ctx)
    cfg = pa.make_config(1, 2, 64, 256, 4, 8, 1)
    ctx = pa.pf_create(cfg, [FAKE])
    try:
        assert L.pf_text_attn_step(ctx, 0, FAKE, FAKE, FAKE, FAKE, None) == pa.PF_ERR_STATE
        assert L.pf_text_attn_step(ctx, 1, FAKE, FAKE, FAKE, FAKE, None) == pa.PF_ERR_INVALID_ARG
        assert L.pf_text_attn_step(ctx, 0, FAKE, None, FAKE, FAKE, None) == pa.PF_ERR_INVALID_ARG
        assert L.pf_text_attn_step(ctx, 0, FAKE, FAKE + 2, FAKE, FAKE, None) == pa.PF_ERR_ALIGN
    finally:
        pa.pf_destroy(ctx)


# ---------------------------------------------------------------- GPU parity


@pytest.mark.gpu
@pytest.mark.parametrize("d,T,B", [(64, 154, 1), (72, 120, 1), (128, 512, 1), (128, 40, 1),
                                   (64, 300, 1), (128, 154, 2)])
@pytest.mark.parametrize("schedule", [pa.PF_SCHED_PIPEFUSION, pa.PF_SCHED_DISTRIFUSION,
                                      pa.PF_SCHED_PIPEFUSION_2H])
def test_text_queries_against_buffer_and_text(d, T, B, schedule):
    wl = synth.AttnWorkload("txt", B, 3, d, 24, 32, 4, T, 1, 2, 0.95, 0.3)
    P = wl.patch_len
    gen = synth.AttnInputs(wl, seed=7, device="cuda")
    pat = pa.PatchAttention(B, 3, d, wl.n_img, 4, T, 1, schedule=schedule)
    g = torch.Generator(device="cuda").manual_seed(11)
    try:
        prev = None
        for s in range(2):
            cur = gen.step_tensors(0)
            if s == 0:
                pat.init_layer(0, cur["k"], cur["v"])
                prev = cur
            q_txt = torch.randn(B, T, 3, d, device="cuda", generator=g).bfloat16()
            for p in range(4):
                sl = slice(p * P, (p + 1) * P)
                pat.step(0, p, cur["q"][:, sl].contiguous(), cur["k"][:, sl].contiguous(),
                         cur["v"][:, sl].contiguous(), cur["k_txt"], cur["v_txt"])
                if p == 1:
                    # mid-step: the buffer holds this step for patches <= 1 under PipeFusion
                    # (either layout), the previous step everywhere under DistriFusion
                    o = pat.text_step(0, q_txt, cur["k_txt"], cur["v_txt"])
                    for bi in range(B):
                        if schedule != pa.PF_SCHED_DISTRIFUSION:
                            kb = oracle.expected_buffer(f64(cur["k"][bi]), f64(prev["k"][bi]), 1, 4)
                            vb = oracle.expected_buffer(f64(cur["v"][bi]), f64(prev["v"][bi]), 1, 4)
                        else:
                            kb, vb = f64(prev["k"][bi]), f64(prev["v"][bi])
                        ref = oracle.attend(f64(q_txt[bi]), np.concatenate([kb, f64(cur["k_txt"][bi])]),
                                            np.concatenate([vb, f64(cur["v_txt"][bi])]), wl.softmax_scale)
                        _close(f64(o[bi]), ref, f64(cur["v"][bi]), f64(prev["v"][bi]),
                               f64(cur["v_txt"][bi]))
            # after the step: the buffer is all this step's K/V
            o = pat.text_step(0, q_txt, cur["k_txt"], cur["v_txt"])
            for bi in range(B):
                ref = oracle.attend(f64(q_txt[bi]),
                                    np.concatenate([f64(cur["k"][bi]), f64(cur["k_txt"][bi])]),
                                    np.concatenate([f64(cur["v"][bi]), f64(cur["v_txt"][bi])]),
                                    wl.softmax_scale)
                _close(f64(o[bi]), ref, f64(cur["v"][bi]), f64(cur["v_txt"][bi]))
            assert pat.next_patch(0) == 0
            prev = cur
        pat.check()
    finally:
        pat.close()


def _close(got, ref, *vs):
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    vmax = max(float(np.abs(v).max()) for v in vs)
    assert rel <= 5e-3, rel
    assert np.max(np.abs(got - ref)) <= 2e-2 * vmax


@pytest.mark.gpu
@pytest.mark.parametrize("d", [8, 64, 72, 128, 256])
@pytest.mark.parametrize("with_gain", [False, True])
def test_qk_rmsnorm_matches_oracle(d, with_gain):
    # d = 8 .. 256 covers every lane-segment width of the kernel (1 .. 32 lanes per vector);
    # 3330 vectors leave a ragged last group for every width
    g = torch.Generator(device="cuda").manual_seed(d)
    x = (torch.randn(2, 333, 5, d, device="cuda", generator=g) * 2.5).bfloat16()
    x0 = f64(x)
    gain = (torch.rand(d, device="cuda", generator=g) + 0.5).bfloat16() if with_gain else None
    pa.pf_qk_rmsnorm(x, gain, 1e-6)
    torch.cuda.synchronize()
    ref = rms_normalize(x0, None if gain is None else f64(gain), 1e-6)
    got = f64(x)
    # within one bf16 ulp of the exact value (fp32 arithmetic, one final rounding)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp * 1.0001)
