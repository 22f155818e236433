"""GPU parity of the fused scatter + patch-attention kernel against the fp64 oracle.

Every call goes through the C ABI.  Buffers are compared bit-exact after every call;
outputs within rel-L2 <= 5e-3 and max-abs <= 2e-2 * max|V_used| (bf16 inputs, fp32
accumulation, P rounded to bf16 before PV, O rounded to bf16).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from patch_attention_b200 import synth
from tests._gpu_harness import f64, run_workload

pytestmark = pytest.mark.gpu

W = synth.ATTN_WORKLOADS


def _wl(base, **kw):
    return dataclasses.replace(base, **kw)


PF, PF2 = pa.PF_SCHED_PIPEFUSION, pa.PF_SCHED_PIPEFUSION_2H


@pytest.mark.parametrize("schedule", [PF, PF2])
def test_tiny_every_call(schedule):
    chk = run_workload(W["tiny"], full_check=lambda s, l, p: True, oracle_buffer=lambda s, l, p: True,
                       schedule=schedule)
    assert chk.n == 3 * 4


@pytest.mark.parametrize("schedule", [PF, PF2])
def test_pixart_all_steps(schedule):
    wl = W["pixart"]
    last = wl.n_steps - 1
    chk = run_workload(wl, full_check=lambda s, l, p: s in (0, 1, 2, last),
                       sample_check=lambda s, l, p: True, n_sample_rows=32,
                       oracle_buffer=lambda s, l, p: s in (1, last), schedule=schedule)
    assert chk.n > 0


@pytest.mark.parametrize("schedule", [PF, PF2])
def test_sd3_full_size_sampled(schedule):
    wl = W["sd3"]
    S = wl.n_steps
    chk = run_workload(wl, steps=S, schedule=schedule,
                       full_check=lambda s, l, p: False,
                       sample_check=lambda s, l, p: (s in (0, 1, S - 1) and l in (0, 3)) or (s == 7 and p == 3),
                       n_sample_rows=8, oracle_buffer=lambda s, l, p: s == 1 and l == 0 and p in (0, 7))
    assert chk.n > 0


@pytest.mark.parametrize("schedule", [PF, PF2])
def test_flux_full_size_sampled(schedule):
    wl = W["flux"]
    S = wl.n_steps
    M = wl.n_patches
    chk = run_workload(wl, steps=S, schedule=schedule,
                       full_check=lambda s, l, p: False,
                       sample_check=lambda s, l, p: s in (0, 1, S - 1) and l in (0, 3) and p in (0, M // 2, M - 1),
                       n_sample_rows=4, oracle_buffer=lambda s, l, p: s == 1 and l == 3 and p == M - 1)
    assert chk.n > 0


@pytest.mark.parametrize("split,schedule", [(True, PF), (False, PF), (True, PF2)])
@pytest.mark.parametrize("d", [64, 72, 128])
def test_ragged_shapes(d, split, schedule):
    # patches that are not multiples of the 128-row tile, a ragged text tail, batch 2;
    # with and without the key-range split across CTAs; one buffer half or two
    wl = synth.AttnWorkload("ragged", batch=2, heads=3, head_dim=d, grid_h=20, grid_w=30,
                            n_patches=3, n_txt=77, n_layers=2, n_steps=3, ar_a=0.95, ar_b=0.3)
    chk = run_workload(wl, full_check=lambda s, l, p: True, oracle_buffer=lambda s, l, p: True,
                       split=split, schedule=schedule)
    assert chk.n == 3 * 2 * 3 * 2


@pytest.mark.parametrize("d", [64, 128])
def test_single_patch_and_tiny_patch(d):
    # M = 1 (the whole image is one patch) and patches of 8 rows
    for n_patches, gh, gw in ((1, 16, 24), (32, 16, 16)):
        wl = synth.AttnWorkload("edge", 1, 2, d, gh, gw, n_patches, 5, 1, 2, 0.95, 0.3)
        run_workload(wl, full_check=lambda s, l, p: True)


def _one_call(d, q, k, v, kt=None, vt=None, n_patches=1):
    B, N, H, _ = k.shape
    T = 0 if kt is None else kt.shape[1]
    pat = pa.PatchAttention(B, H, d, N, n_patches, T, 1)
    try:
        pat.init_layer(0, k, v)
        P = N // n_patches
        outs = []
        for p in range(n_patches):
            sl = slice(p * P, (p + 1) * P)
            outs.append(pat.step(0, p, q[:, sl].contiguous(), k[:, sl].contiguous(),
                                 v[:, sl].contiguous(), kt, vt))
        pat.check()
        return torch.cat(outs, dim=1)
    finally:
        pat.close()


@pytest.mark.parametrize("d", [64, 72, 128])
def test_unit_values_give_unit_output(d):
    g = torch.Generator(device="cuda").manual_seed(1)
    B, N, H = 1, 1024, 2
    q = torch.randn(B, N, H, d, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, N, H, d, device="cuda", generator=g).bfloat16()
    v = torch.ones(B, N, H, d, device="cuda", dtype=torch.bfloat16)
    o = _one_call(d, q, k, v, n_patches=4)
    assert torch.all((o.float() - 1).abs() <= 1e-2)


@pytest.mark.parametrize("d", [64, 72, 128])
def test_zero_query_gives_mean_value(d):
    g = torch.Generator(device="cuda").manual_seed(2)
    B, N, H, T = 1, 640, 2, 40
    q = torch.zeros(B, N, H, d, device="cuda", dtype=torch.bfloat16)
    k = torch.randn(B, N, H, d, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, N, H, d, device="cuda", generator=g).bfloat16()
    kt = torch.randn(B, T, H, d, device="cuda", generator=g).bfloat16()
    vt = torch.randn(B, T, H, d, device="cuda", generator=g).bfloat16()
    o = _one_call(d, q, k, v, kt, vt, n_patches=5)
    ref = oracle.attend(np.zeros((1, H, d)), np.concatenate([f64(k[0]), f64(kt[0])]),
                        np.concatenate([f64(v[0]), f64(vt[0])]), d ** -0.5)
    err = np.abs(f64(o[0]) - ref).max()
    assert err <= 8e-3, err


def test_deterministic_bitwise():
    wl = synth.AttnWorkload("det", 1, 4, 128, 32, 32, 4, 33, 1, 2, 0.95, 0.3)

    def run():
        gen = synth.AttnInputs(wl, seed=5, device="cuda")
        pat = pa.PatchAttention(1, 4, 128, 1024, 4, 33, 1)
        outs = []
        try:
            for s in range(2):
                cur = gen.step_tensors(0)
                if s == 0:
                    pat.init_layer(0, cur["k"], cur["v"])
                for p in range(4):
                    sl = slice(p * 256, (p + 1) * 256)
                    outs.append(pat.step(0, p, cur["q"][:, sl].contiguous(), cur["k"][:, sl].contiguous(),
                                         cur["v"][:, sl].contiguous(), cur["k_txt"], cur["v_txt"]).clone())
            kb, vb = pat.buffer_kv(0)
            return outs, kb.clone(), vb.clone()
        finally:
            pat.close()

    a, b = run(), run()
    for x, y in zip(a[0], b[0]):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))
    assert torch.equal(a[2].view(torch.int16), b[2].view(torch.int16))


def test_output_margins_untouched():
    # outputs and buffers live inside larger allocations filled with a sentinel
    B, H, d, N, M, T = 1, 2, 72, 384, 3, 10
    g = torch.Generator(device="cuda").manual_seed(3)
    mk = lambda *s: torch.randn(*s, device="cuda", generator=g).bfloat16()
    q, k, v, kt, vt = mk(B, N, H, d), mk(B, N, H, d), mk(B, N, H, d), mk(B, T, H, d), mk(B, T, H, d)
    cfg = pa.make_config(B, H, d, N, M, T, 1)
    nbytes = pa.pf_kvbuf_bytes(cfg)
    pad = 4096
    buf_big = torch.full((nbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    ctx = pa.pf_create(cfg, [buf_big.data_ptr() + pad])
    P = N // M
    n_o = B * P * H * d
    o_big = torch.full((n_o + 2 * 2048,), -7.0, dtype=torch.bfloat16, device="cuda")
    try:
        pa.pf_kvbuf_init(ctx, 0, k, v)
        for p in range(M):
            sl = slice(p * P, (p + 1) * P)
            o = o_big[2048:2048 + n_o].view(B, P, H, d)
            pa.pf_patch_attn_step(ctx, 0, p, q[:, sl].contiguous(), k[:, sl].contiguous(),
                                  v[:, sl].contiguous(), kt, vt, o)
            torch.cuda.synchronize()
            assert torch.all(o_big[:2048] == -7.0) and torch.all(o_big[2048 + n_o:] == -7.0)
            assert torch.all(buf_big[:pad] == 0xA5) and torch.all(buf_big[pad + nbytes:] == 0xA5)
        pa.pf_check_device_status(ctx)
    finally:
        pa.pf_destroy(ctx)


def test_order_errors_leave_gpu_state_intact():
    B, H, d, N, M = 1, 2, 64, 256, 4
    g = torch.Generator(device="cuda").manual_seed(4)
    mk = lambda *s: torch.randn(*s, device="cuda", generator=g).bfloat16()
    q, k, v = mk(B, N, H, d), mk(B, N, H, d), mk(B, N, H, d)
    pat = pa.PatchAttention(B, H, d, N, M, 0, 1)
    try:
        with pytest.raises(pa.PatchAttnError) as e:
            pat.step(0, 0, q[:, :64].contiguous(), k[:, :64].contiguous(), v[:, :64].contiguous())
        assert e.value.status == pa.PF_ERR_STATE
        pat.init_layer(0, k, v)
        with pytest.raises(pa.PatchAttnError) as e:
            pat.step(0, 1, q[:, 64:128].contiguous(), k[:, 64:128].contiguous(), v[:, 64:128].contiguous())
        assert e.value.status == pa.PF_ERR_ORDER
        assert pat.next_patch(0) == 0
        pat.step(0, 0, q[:, :64].contiguous(), k[:, :64].contiguous(), v[:, :64].contiguous())
        assert pat.next_patch(0) == 1
        pat.check()
    finally:
        pat.close()


@pytest.mark.parametrize("d", [64, 72, 128])
def test_distrifusion_schedule(d):
    # patches in a random order each step; every other patch is seen at the previous step
    wl = synth.AttnWorkload("distri", batch=1, heads=3, head_dim=d, grid_h=16, grid_w=40,
                            n_patches=5, n_txt=20, n_layers=2, n_steps=3, ar_a=0.95, ar_b=0.3)
    chk = run_workload(wl, full_check=lambda s, l, p: True, schedule=pa.PF_SCHED_DISTRIFUSION)
    assert chk.n == 3 * 2 * 5


def test_pipefusion_closer_to_fresh_than_distrifusion_on_gpu():
    """Quality claim of the pages, measured on the GPU outputs of both schedules."""
    wl = synth.AttnWorkload("claim", 1, 4, 64, 32, 32, 4, 16, 1, 3, 0.95, 0.3)
    P = wl.patch_len
    errs = {}
    for sched in (pa.PF_SCHED_PIPEFUSION, pa.PF_SCHED_DISTRIFUSION):
        gen = synth.AttnInputs(wl, seed=3, device="cuda")
        pat = pa.PatchAttention(1, 4, 64, wl.n_img, 4, 16, 1, schedule=sched)
        e = 0.0
        try:
            for s in range(3):
                cur = gen.step_tensors(0)
                if s == 0:
                    pat.init_layer(0, cur["k"], cur["v"])
                outs = []
                for p in range(4):
                    sl = slice(p * P, (p + 1) * P)
                    outs.append(pat.step(0, p, cur["q"][:, sl].contiguous(), cur["k"][:, sl].contiguous(),
                                         cur["v"][:, sl].contiguous(), cur["k_txt"], cur["v_txt"]))
                if s == 2:
                    o = f64(torch.cat(outs, dim=1)[0])
                    fresh = oracle.attend(f64(cur["q"][0]), np.concatenate([f64(cur["k"][0]), f64(cur["k_txt"][0])]),
                                          np.concatenate([f64(cur["v"][0]), f64(cur["v_txt"][0])]), wl.softmax_scale)
                    e = float(np.sum((o - fresh) ** 2))
            pat.check()
        finally:
            pat.close()
        errs[sched] = e
    assert errs[pa.PF_SCHED_PIPEFUSION] < errs[pa.PF_SCHED_DISTRIFUSION], errs
