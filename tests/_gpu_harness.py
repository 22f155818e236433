"""Shared driver for the GPU parity tests: walks a workload's diffusion steps through the
C ABI (via the Python binding) and compares against the fp64 oracle."""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

import oracle
import patch_attention_b200 as pa
from patch_attention_b200 import synth

REL_L2_TOL = 5e-3      # relative L2 of O over the checked outputs
MAX_ABS_FRAC = 2e-2    # max |O_gpu - O_ref| <= 2e-2 * max |V_used|


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


class Checker:
    """Accumulates error statistics over checked calls; asserts at the end."""

    def __init__(self):
        self.worst_rel_l2 = 0.0
        self.worst_abs_frac = 0.0
        self.n = 0

    def add(self, got: np.ndarray, ref: np.ndarray, vmax: float, what: str):
        err = got - ref
        rel = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30))
        absf = float(np.max(np.abs(err)) / max(vmax, 1e-30))
        self.worst_rel_l2 = max(self.worst_rel_l2, rel)
        self.worst_abs_frac = max(self.worst_abs_frac, absf)
        self.n += 1
        assert rel <= REL_L2_TOL, f"{what}: rel-L2 {rel:.3e} > {REL_L2_TOL}"
        assert absf <= MAX_ABS_FRAC, f"{what}: max-abs/max|V| {absf:.3e} > {MAX_ABS_FRAC}"


PIPEFUSION = (pa.PF_SCHED_PIPEFUSION, pa.PF_SCHED_PIPEFUSION_2H)


def buffer_now(pat: pa.PatchAttention, layer: int):
    """(K, V) of the layer's buffer as the next call sees it: the one half of the single-half
    schedule, else the rows composed from both halves."""
    if pat.cfg.schedule == pa.PF_SCHED_PIPEFUSION:
        return pat.buffer_kv(layer, 0)
    return pat.buffer_as_it_stands(layer)


def device_buffer_check(pat: pa.PatchAttention, layer: int, p: int, cur, prev):
    """Bit-exact: buffer rows of patches <= p hold this step's K/V, the rest the previous step's."""
    kb, vb = buffer_now(pat, layer)
    P = pat.plen
    hi = (p + 1) * P
    for buf, now, old in ((kb, cur["k"], prev["k"]), (vb, cur["v"], prev["v"])):
        assert torch.equal(buf[:, :hi].view(torch.int16), now[:, :hi].view(torch.int16)), "fresh rows"
        assert torch.equal(buf[:, hi:].view(torch.int16), old[:, hi:].view(torch.int16)), "stale rows"


def oracle_buffer_check(pat: pa.PatchAttention, layer: int, p: int, cur, prev):
    kb, vb = buffer_now(pat, layer)
    for buf, now, old in ((kb, cur["k"], prev["k"]), (vb, cur["v"], prev["v"])):
        got = buf.cpu().view(torch.int16).numpy()[0]
        exp = oracle.expected_buffer(now.cpu().view(torch.int16).numpy()[0],
                                     old.cpu().view(torch.int16).numpy()[0], p, pat.cfg.n_patches)
        assert np.array_equal(got, exp), "buffer differs from the oracle's expectation"


def oracle_patch_output(wl, cur_cpu, prev_cpu, p, b=0, rows=None, heads=None):
    """fp64 oracle output of patch p for batch b: [rows, heads, d]."""
    sl = slice(None) if heads is None else heads
    take = lambda t: f64(t[b][:, sl])
    return oracle.patch_attention(
        take(cur_cpu["q"]), take(cur_cpu["k"]), take(cur_cpu["v"]), take(prev_cpu["k"]),
        take(prev_cpu["v"]), take(cur_cpu["k_txt"]), take(cur_cpu["v_txt"]), p, wl.n_patches,
        wl.softmax_scale, rows=rows)


def vmax_used(cur_cpu, prev_cpu, p, n_patches, b=0, heads=None):
    sl = slice(None) if heads is None else heads
    P = cur_cpu["v"].shape[1] // n_patches
    hi = (p + 1) * P
    parts = [cur_cpu["v"][b, :hi, sl], prev_cpu["v"][b, hi:, sl], cur_cpu["v_txt"][b, :, sl]]
    return max(float(x.abs().max()) if x.numel() else 0.0 for x in parts)


def run_workload(wl: synth.AttnWorkload, steps: Optional[int] = None, full_check=lambda s, l, p: True,
                 sample_check=lambda s, l, p: False, n_sample_rows: int = 8, seed: Optional[int] = None,
                 schedule=pa.PF_SCHED_PIPEFUSION, a=None, b=None, oracle_buffer=lambda s, l, p: False,
                 split=True):
    """Run `steps` diffusion steps of `wl` through the library and check against the oracle.

    full_check(s, l, p)   -> compare every output row of that call with the oracle
    sample_check(s, l, p) -> compare n_sample_rows rows (first, last, random) x one random head
    Every call's buffer is checked bit-exact on the device.
    """
    dev = torch.device("cuda")
    S = wl.n_steps if steps is None else steps
    gen = synth.AttnInputs(wl, seed=seed, device=dev, a=a, b=b)
    pat = pa.PatchAttention(wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt,
                            wl.n_layers, schedule=schedule, split=split)
    rng = np.random.default_rng(1234)
    chk = Checker()
    P = wl.patch_len
    prev = [None] * wl.n_layers
    try:
        for s in range(S):
            for layer in range(wl.n_layers):
                cur = gen.step_tensors(layer)
                if s == 0:
                    pat.init_layer(layer, cur["k"], cur["v"])
                    prev[layer] = cur
                pv = prev[layer]
                need_cpu = any(full_check(s, layer, p) or sample_check(s, layer, p)
                               for p in range(wl.n_patches))
                cur_cpu = {k: v.cpu() for k, v in cur.items()} if need_cpu else None
                prev_cpu = {k: v.cpu() for k, v in pv.items()} if need_cpu else None
                order = range(wl.n_patches)
                if schedule == pa.PF_SCHED_DISTRIFUSION:
                    order = list(rng.permutation(wl.n_patches))
                for p in order:
                    sl = slice(p * P, (p + 1) * P)
                    q_p = cur["q"][:, sl].contiguous()
                    k_p = cur["k"][:, sl].contiguous()
                    v_p = cur["v"][:, sl].contiguous()
                    o = pat.step(layer, p, q_p, k_p, v_p, cur["k_txt"], cur["v_txt"])
                    if schedule in PIPEFUSION:
                        device_buffer_check(pat, layer, p, cur, pv)
                        if oracle_buffer(s, layer, p):
                            oracle_buffer_check(pat, layer, p, cur, pv)
                    if full_check(s, layer, p):
                        for bi in range(wl.batch):
                            ref = _ref(wl, cur_cpu, prev_cpu, p, bi, None, None, schedule)
                            vmax = _vmax(cur_cpu, prev_cpu, p, wl.n_patches, bi, None, schedule)
                            chk.add(f64(o[bi]), ref, vmax, f"s{s} l{layer} p{p} b{bi}")
                    elif sample_check(s, layer, p):
                        rows = sorted(set([0, P - 1] + list(rng.integers(0, P, n_sample_rows - 2))))
                        for bi in range(wl.batch):
                            h = int(rng.integers(0, wl.heads))
                            ref = _ref(wl, cur_cpu, prev_cpu, p, bi, rows, slice(h, h + 1), schedule)
                            vmax = _vmax(cur_cpu, prev_cpu, p, wl.n_patches, bi, slice(h, h + 1), schedule)
                            got = f64(o[bi][rows][:, h:h + 1])
                            chk.add(got, ref, vmax, f"s{s} l{layer} p{p} b{bi} h{h} rows")
                if schedule == pa.PF_SCHED_DISTRIFUSION:
                    # after the step, one half of the buffer holds exactly this step's K/V
                    # (the stale context of the next step)
                    halves = [pat.buffer_kv(layer, hf) for hf in (0, 1)]
                    assert any(torch.equal(kb.view(torch.int16), cur["k"].view(torch.int16)) and
                               torch.equal(vb.view(torch.int16), cur["v"].view(torch.int16))
                               for kb, vb in halves), "no buffer half holds the step's K/V"
                prev[layer] = cur
            pat.check()
        torch.cuda.synchronize()
    finally:
        pat.close()
    return chk


def _ref(wl, cur_cpu, prev_cpu, p, b, rows, heads, schedule):
    if schedule in PIPEFUSION:
        return oracle_patch_output(wl, cur_cpu, prev_cpu, p, b, rows, heads)
    sl = slice(None) if heads is None else heads
    take = lambda t: f64(t[b][:, sl])
    return oracle.distrifusion_attention(
        take(cur_cpu["q"]), take(cur_cpu["k"]), take(cur_cpu["v"]), take(prev_cpu["k"]),
        take(prev_cpu["v"]), take(cur_cpu["k_txt"]), take(cur_cpu["v_txt"]), p, wl.n_patches,
        wl.softmax_scale, rows=rows)


def _vmax(cur_cpu, prev_cpu, p, M, b, heads, schedule):
    if schedule in PIPEFUSION:
        return vmax_used(cur_cpu, prev_cpu, p, M, b, heads)
    sl = slice(None) if heads is None else heads
    return max(float(cur_cpu["v"][b, :, sl].abs().max()), float(prev_cpu["v"][b, :, sl].abs().max()),
               float(cur_cpu["v_txt"][b, :, sl].abs().max()) if cur_cpu["v_txt"].numel() else 0.0)
