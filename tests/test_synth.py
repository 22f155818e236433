"""Statistics and determinism of the seeded input generators (CPU only)."""
import math

import torch

from patch_attention_b200 import synth


def _wl(**kw):
    base = dict(name="tiny", batch=1, heads=4, head_dim=64, grid_h=32, grid_w=32, n_patches=4,
                n_txt=16, n_layers=2, n_steps=3, ar_a=0.95, ar_b=0.3)
    base.update(kw)
    return synth.AttnWorkload(**base)


def test_ar1_moments_and_lag_correlation():
    wl = _wl()
    gen = synth.AttnInputs(wl, seed=3)
    a, b = wl.ar_a, wl.ar_b
    xs = [gen.step_tensors(0)["k"].float() for _ in range(12)]
    n = xs[0].numel()
    tol = 6.0 / math.sqrt(n)
    for s, x in enumerate(xs):
        var_s = a ** (2 * s) + b * b * (1 - a ** (2 * s)) / (1 - a * a)
        assert abs(x.mean().item()) < tol * math.sqrt(var_s)
        assert abs(x.var().item() / var_s - 1) < 0.02, (s, x.var().item(), var_s)
    # lag-1 correlation corr(X_s, X_{s-1}) = a * sqrt(var_{s-1} / var_s)
    for s in range(1, 12):
        v0 = a ** (2 * (s - 1)) + b * b * (1 - a ** (2 * (s - 1))) / (1 - a * a)
        v1 = a ** (2 * s) + b * b * (1 - a ** (2 * s)) / (1 - a * a)
        r = torch.corrcoef(torch.stack([xs[s].flatten(), xs[s - 1].flatten()]))[0, 1].item()
        assert abs(r - a * math.sqrt(v0 / v1)) < 0.01


def test_stationary_variance_limit():
    for a, b in ((0.95, 0.3), (0.97, 0.25)):
        assert abs(b * b / (1 - a * a) - {0.95: 0.923, 0.97: 1.058}[a]) < 1e-3


def test_deterministic_and_order_independent():
    wl = _wl()
    g1 = synth.AttnInputs(wl, seed=9)
    g2 = synth.AttnInputs(wl, seed=9)
    l1 = [g1.step_tensors(1) for _ in range(2)]
    a0 = g1.step_tensors(0)
    b0 = g2.step_tensors(0)                      # other order: layer 0 first
    l2 = [g2.step_tensors(1) for _ in range(2)]
    for k in a0:
        assert torch.equal(a0[k], b0[k])
        assert torch.equal(l1[1][k], l2[1][k])
    assert not torch.equal(a0["q"], a0["k"])
    assert not torch.equal(l1[0]["k"], a0["k"])  # layers differ


def test_rmsnorm_workload_has_unit_rms_queries_keys():
    wl = _wl(qk_rmsnorm=True, head_dim=128)
    t = synth.AttnInputs(wl, seed=1).step_tensors(0)
    for k in ("q", "k", "k_txt"):
        rms = t[k].float().pow(2).mean(-1).sqrt()
        assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)
    assert t["v"].float().pow(2).mean(-1).sqrt().std() > 0.05


def test_shapes_and_dtypes():
    for name, wl in synth.ATTN_WORKLOADS.items():
        assert wl.n_img % wl.n_patches == 0
    wl = _wl()
    t = synth.AttnInputs(wl).step_tensors(0)
    assert t["q"].shape == (1, wl.n_img, wl.heads, wl.head_dim) and t["q"].dtype == torch.bfloat16
    assert t["k_txt"].shape == (1, wl.n_txt, wl.heads, wl.head_dim)


def test_workload_flop_counts():
    w = synth.ATTN_WORKLOADS
    assert abs(w["tiny"].flop_per_layer_step() - 3.36e7) / 3.36e7 < 0.01
    assert abs(w["pixart"].flop_per_layer_step() - 7.96e10) / 7.96e10 < 0.01
    assert abs(4 * w["sd3"].flop_per_layer_step() - 6.66e12) / 6.66e12 < 0.01
    assert abs(4 * w["flux"].flop_per_layer_step() - 2.13e14) / 2.13e14 < 0.01


def test_cfg_schedule_endpoints():
    wl = synth.CfgWorkload("cfg", 1, 4, 8, 8)
    assert wl.s_t(0) == 1.0 and abs(wl.s_t(49) - 0.05) < 1e-12
    c, u = synth.CfgInputs(wl, seed=2).step_tensors(0)
    assert c.dtype == torch.float32 and c.shape == (1, 4, 8, 8)
