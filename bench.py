#!/usr/bin/env python
"""Benchmark of the patch-attention hot path on B200.

One step = one diffusion step of the workload: for every patch p = 0..M-1 (in order)
and every layer l, one ``pf_patch_attn_step`` micro-step (fused K/V scatter + attention
against the layer's stale/fresh buffer plus text tokens), followed by one fused
guidance combine + rel-MAE over the workload's latent (``pf_cfg_combine_relmae``).

Printed: one JSON line (rank 0).  ``value`` = algorithmic attention TFLOP/s over all
ranks (4 * N_img * N_kv * head_dim * heads per layer per step, real head_dim) with the
inputs resident in HBM; ``e2e`` = the same metric with the step's inputs copied from
pinned host memory and the outputs copied back inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload flux|sd3|pixart|tiny]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from patch_attention_b200 import synth  # noqa: E402

CFG_SHAPE = {"tiny": (4, 16, 16), "pixart": (4, 128, 128), "sd3": (16, 256, 256), "flux": (16, 512, 512)}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------------- utils


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("attn_fwd.cu", "sm100_ptx.cuh", "pf_internal.h"):
        with open(os.path.join(ROOT, "patch_attention_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu summary, or None
    when the summary is missing or was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "patch_attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent or ent.get("kernel_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------------- oracle


def oracle_inputs(wl: synth.AttnWorkload, seed: int = 7, heads: int = 2):
    """fp64 inputs of one micro-step (step 1) for `heads` heads at full context length."""
    hs = min(heads, wl.heads)
    small = synth.AttnWorkload(wl.name, wl.batch, hs, wl.head_dim, wl.grid_h, wl.grid_w,
                               wl.n_patches, wl.n_txt, 1, 2, wl.ar_a, wl.ar_b, wl.qk_rmsnorm)
    gen = synth.AttnInputs(small, seed=seed, device="cpu")
    prev = gen.step_tensors(0)
    cur = gen.step_tensors(0)
    f = lambda t: t[0].to(torch.float64).numpy()
    return hs, [f(cur["q"]), f(cur["k"]), f(cur["v"]), f(prev["k"]), f(prev["v"]), f(cur["k_txt"]),
                f(cur["v_txt"])]


def oracle_sample(wl: synth.AttnWorkload, hs: int, arrs, rows_per_call: int, seed: int):
    """Time the fp64 oracle on a bounded sample: `rows_per_call` query rows x `hs` heads of
    the middle patch.  Returns (seconds, algorithmic FLOP)."""
    import numpy as np
    import oracle

    p = wl.n_patches // 2
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.patch_len, size=min(rows_per_call, wl.patch_len), replace=False))
    t0 = time.perf_counter()
    oracle.patch_attention(*arrs, p, wl.n_patches, wl.softmax_scale, rows=rows)
    dt = time.perf_counter() - t0
    return dt, 4.0 * len(rows) * wl.n_kv * wl.head_dim * hs


def cpu_rows_for(wl) -> int:
    return {"tiny": 64, "pixart": 512, "sd3": 512, "flux": 512}.get(wl.name, 256)


def cpu_baseline(wl, budget_s: float = 10.0):
    """Oracle throughput on repeated bounded samples until about `budget_s` of CPU work."""
    rows = cpu_rows_for(wl)
    hs, arrs = oracle_inputs(wl)
    tot_t = tot_f = 0.0
    n = 0
    while tot_t < budget_s and n < 64:
        dt, fl = oracle_sample(wl, hs, arrs, rows, seed=11 + n)
        tot_t += dt
        tot_f += fl
        n += 1
    sample = (f"{n} x ({rows} query rows x {hs} heads) of a {wl.name} micro-step at full context "
              f"({wl.n_kv} keys), fp64 oracle incl. key assembly, {tot_t:.1f} s")
    return {"value": tot_f / tot_t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": sample}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    wl = synth.ATTN_WORKLOADS[args.workload]
    rows = cpu_rows_for(wl)
    hs, arrs = oracle_inputs(wl)
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        dt, fl = oracle_sample(wl, hs, arrs, rows, seed=7 + i)
        if i >= args.warmup:
            times.append(dt)
            flops.append(fl)
    tot_t, tot_f = sum(times), sum(flops)
    value = tot_f / tot_t / 1e12
    cores = blas_threads()
    sample = (f"per step: {rows} query rows x 2 heads of one {wl.name} micro-step (step 1, middle "
              f"patch) at full context ({wl.n_kv} keys), fp64 oracle incl. key assembly")
    line = {
        "impl": "reference", "metric": "patch-attn TFLOP/s (algorithmic, per diffusion step)",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------- GPU

L2_BYTES = 126 << 20
NOMINAL_FLOP_PER_CLK_SM = 8192  # dense bf16 tcgen05: one 128x128x16 MMA per 64 cycles per SM


def n_sms(dev) -> int:
    return torch.cuda.get_device_properties(dev).multi_processor_count


# PipeFusion's schedule over one buffer half per layer (the pages' layout) or two (the same
# rows; the step being written goes to the other half, so consecutive calls on a layer overlap)
BUFFER_HALVES = 2


def pipefusion_schedule(pa):
    return pa.PF_SCHED_PIPEFUSION_2H if BUFFER_HALVES == 2 else pa.PF_SCHED_PIPEFUSION


class StepRunner:
    """One attention workload resident in HBM: per-layer buffers, `n_sets` alternating input
    sets (AR(1) steps) and outputs.  A step = every patch in order x every layer through
    pf_patch_attn_step, then one guidance combine over the model's latent."""

    def __init__(self, pa, wl, dev, seed, min_set_bytes=2 * L2_BYTES):
        self.pa, self.wl, self.dev = pa, wl, dev
        B, H, d, N, M, T, L = wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, wl.n_layers
        assert B == 1, "patch slices are passed as views; batch 1 keeps them contiguous"
        set_bytes = L * (3 * N + 2 * T) * H * d * 2
        # enough alternating input sets that consecutive steps' inputs together exceed L2
        self.n_sets = max(2, -(-min_set_bytes // set_bytes))
        gen = synth.AttnInputs(wl, seed=seed, device=dev)
        self.sets = [[gen.step_tensors(l) for l in range(L)] for _ in range(self.n_sets)]
        del gen  # drop the fp32 AR(1) state
        torch.cuda.empty_cache()
        self.set_bytes = set_bytes
        self.pat = pa.PatchAttention(B, H, d, N, M, T, L, schedule=pipefusion_schedule(pa))
        for l in range(L):
            self.pat.init_layer(l, self.sets[0][l]["k"], self.sets[0][l]["v"])
        self.outs = [torch.empty(B, N, H, d, dtype=torch.bfloat16, device=dev) for _ in range(L)]
        self.cshape = CFG_SHAPE[wl.name]
        self.cwl = synth.CfgWorkload("cfg", B, *self.cshape)
        self.c_in, self.u_in = synth.CfgInputs(self.cwl, device=dev).step_tensors(25)
        self.n_cfg = self.c_in.numel() // B
        self.cfg_out = torch.empty(self.c_in.shape, dtype=torch.bfloat16, device=dev)
        self.rel = torch.empty(B, dtype=torch.float32, device=dev)
        self.cws = torch.empty(max(16, pa.pf_cfg_workspace_bytes(B, self.n_cfg)), dtype=torch.uint8, device=dev)
        self.L_ = pa._lib()
        self.row_bytes = H * d * 2
        # precomputed pointers: the timed loop is argument marshalling only
        self.ptrs = []
        for st in range(self.n_sets):
            per = []
            for l in range(L):
                t = self.sets[st][l]
                per.append((t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                            t["k_txt"].data_ptr() if T else None, t["v_txt"].data_ptr() if T else None))
            self.ptrs.append(per)
        self.optrs = [o.data_ptr() for o in self.outs]
        self.launches_per_step = M * L + 2  # attention launches + guidance partial + finalize

    def attn_section(self, set_idx, sh):
        wl, L_, ctx = self.wl, self.L_, self.pat.ctx
        per = self.ptrs[set_idx % self.n_sets]
        for p in range(wl.n_patches):
            off = p * wl.patch_len * self.row_bytes
            for l in range(wl.n_layers):
                q, k, v, kt, vt = per[l]
                st = L_.pf_patch_attn_step(ctx, l, p, q + off, k + off, v + off, kt, vt, self.optrs[l] + off, sh)
                if st != 0:
                    raise self.pa.PatchAttnError(st, "pf_patch_attn_step")

    def cfg_section(self, sh):
        st = self.L_.pf_cfg_combine_relmae(self.c_in.data_ptr(), self.u_in.data_ptr(), self.wl.batch, self.n_cfg,
                                           self.cwl.w, None, self.cfg_out.data_ptr(), self.rel.data_ptr(),
                                           self.cws.data_ptr(), self.cws.numel(), sh)
        if st != 0:
            raise self.pa.PatchAttnError(st, "pf_cfg_combine_relmae")

    def run(self, steps, first_set, world, sample_clocks=True):
        """Time exactly `steps` steps (barrier + synchronize on both sides).  Returns the
        total ms, per-step attention and guidance ms from events on the launching stream,
        and the clock samples taken during the timed region."""
        dev = self.dev
        stream = torch.cuda.current_stream(dev)
        sh = stream.cuda_stream
        ev = lambda: torch.cuda.Event(enable_timing=True)
        a0 = [ev() for _ in range(steps)]
        a1 = [ev() for _ in range(steps)]
        c1 = [ev() for _ in range(steps)]
        start, stop = ev(), ev()
        clocks = ClockSampler(dev.index or 0) if sample_clocks else None
        barrier(world)
        torch.cuda.synchronize(dev)
        if clocks:
            clocks.start()
            time.sleep(0.3)  # let the sampler attach before the timed region
        start.record(stream)
        for i in range(steps):
            a0[i].record(stream)
            self.attn_section(first_set + i, sh)
            a1[i].record(stream)
            self.cfg_section(sh)
            c1[i].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
        clock_info = clocks.stop() if clocks else None
        barrier(world)
        self.pat.check()
        total = start.elapsed_time(stop)
        attn = sum(a0[i].elapsed_time(a1[i]) for i in range(steps)) / steps
        cfg = sum(a1[i].elapsed_time(c1[i]) for i in range(steps)) / steps
        return total, attn, cfg, clock_info

    def warm(self, steps):
        sh = torch.cuda.current_stream(self.dev).cuda_stream
        for i in range(steps):
            self.attn_section(i + 1, sh)
            self.cfg_section(sh)
        torch.cuda.synchronize(self.dev)
        self.pat.check()

    def close(self):
        self.pat.close()


def attn_kernel_name(wl) -> str:
    """The library's attention kernel for the workload's head_dim."""
    return "patch_attn_hr_kernel" if wl.head_dim == 64 else "patch_attn_sn_kernel"


def per_clock(tflops, clock_info, sms):
    """FLOP per SM per clock at the median SM clock of the timed region, and its fraction
    of the nominal dense bf16 rate (8192 FLOP/clk/SM)."""
    if not clock_info or not clock_info.get("sm_mhz"):
        return None, None
    f = tflops * 1e12 / (sms * clock_info["sm_mhz"] * 1e6)
    return f, f / NOMINAL_FLOP_PER_CLK_SM


def attn_roofline(wl, attn_ms, timed_s, peaks, peak_src, clock_info, sms, traffic):
    """Roofline of the attention kernel: algorithmic FLOP per launch / average launch time
    (events around each step's attention section, launch gaps included).  The peak is the
    measured sustained bf16 rate when the timed region lasts at least 2 s, else the burst."""
    launch_ms = attn_ms / (wl.n_patches * wl.n_layers)
    achieved = wl.flop_per_call() / (launch_ms * 1e-3) / 1e12
    sustained = timed_s >= 2.0
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = float(peaks.get(key, peaks.get("bf16_tflops")))
    fpc, fpc_frac = per_clock(achieved, clock_info, sms)
    return {"bound": "tensor", "kernel": attn_kernel_name(wl), "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
            "peak_source": f"{peak_src} {key} ({'timed region >= 2 s' if sustained else 'timed region < 2 s'})",
            "launch_ms": launch_ms, "flop_per_launch": wl.flop_per_call(),
            "flop_per_clk_sm": fpc, "frac_of_nominal_per_clk": fpc_frac}


def sub_record(pa, name, dev, seed, world, peaks, peak_src, min_timed_s=2.0, max_steps=20000):
    """A workload other than the headline, timed over at least `min_timed_s` of steps so that
    the sustained peak is the right denominator; its own clock samples."""
    wl = synth.ATTN_WORKLOADS[name]
    r = StepRunner(pa, wl, dev, seed if seed is not None else synth.default_seed(name))
    try:
        r.warm(3)
        total, _, _, _ = r.run(3, 4, 1, sample_clocks=False)
        t_step = total / 3 / 1e3
        steps = int(min(max_steps, max(20, math.ceil(min_timed_s * 1.1 / t_step))))
        steps = int(max_over_ranks(float(steps), world))  # every rank times the same count
        total, attn, cfg, clk = r.run(steps, 7, world)
    finally:
        r.close()
    ms = max_over_ranks(total / steps, world)
    flop_step = wl.n_layers * wl.flop_per_layer_step()
    value = world * flop_step / (ms * 1e-3) / 1e12
    sms = n_sms(dev)
    rec = {"workload": name, "steps": steps, "timed_s": total / 1e3, "ms_per_step": ms,
           "value": value, "unit": "TFLOP/s", "attn_ms_per_step": attn, "cfg_ms_per_step": cfg,
           "flop_per_step": flop_step,
           "config": {"heads": wl.heads, "head_dim": wl.head_dim, "n_img": wl.n_img,
                      "n_patches": wl.n_patches, "patch_len": wl.patch_len, "n_txt": wl.n_txt,
                      "layers": wl.n_layers, "buffer_halves": BUFFER_HALVES},
           "l2": f"{r.n_sets} alternating input sets of {r.set_bytes / 1e6:.0f} MB (together > 2x L2)",
           "roofline": attn_roofline(wl, attn, total / 1e3, peaks, peak_src, clk, sms, load_traffic(name)),
           "clocks": clk}
    return rec


def measure_copy_kernels(pa, r: StepRunner, hbm, reps=5):
    """The start-up pass (pf_kvbuf_init) of one layer and the per-head RMS normalisation of a
    full-spatial Q, both HBM bound and both larger than L2; median of `reps` calls."""
    wl, dev = r.wl, r.dev
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            e0, e1 = ev(), ev()
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    t = r.sets[0][0]
    init_ms = timed(lambda: r.pat.init_layer(0, t["k"], t["v"]))
    init_bytes = 2 * 2 * t["k"].numel() * 2  # K and V, read + written
    x = t["q"].clone()
    norm_ms = timed(lambda: pa.pf_qk_rmsnorm(x))
    norm_bytes = 2 * x.numel() * 2
    del x
    # what the separate pass costs one micro-step: Q_p and K_p of one patch normalised before
    # the attention launch (the text keys are normalised once per step and layer)
    P = wl.patch_len
    qp, kp = t["q"][:, :P].clone(), t["k"][:, :P].clone()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def per_call():
        flush.zero_()  # the patch's Q and K come from HBM, as they would after the projection
        e0, e1 = ev(), ev()
        e0.record(stream)
        pa.pf_qk_rmsnorm(qp)
        pa.pf_qk_rmsnorm(kp)
        e1.record(stream)
        return e0, e1

    ts = []
    for i in range(reps + 2):
        e0, e1 = per_call()
        torch.cuda.synchronize(dev)
        if i >= 2:
            ts.append(e0.elapsed_time(e1))
    call_norm_ms = statistics.median(ts)
    del qp, kp, flush
    return {
        "kvbuf_init": {"gb_per_s": init_bytes / (init_ms * 1e-3) / 1e9,
                       "frac_hbm": init_bytes / (init_ms * 1e-3) / 1e9 / hbm, "ms": init_ms,
                       "bytes": init_bytes, "what": f"one {wl.name} layer: K and V [1,{wl.n_img},{wl.heads},{wl.head_dim}] bf16 copied into the buffer"},
        "qk_rmsnorm": {"gb_per_s": norm_bytes / (norm_ms * 1e-3) / 1e9,
                       "frac_hbm": norm_bytes / (norm_ms * 1e-3) / 1e9 / hbm, "ms": norm_ms,
                       "bytes": norm_bytes, "what": f"in place on a full-spatial {wl.name} Q [1,{wl.n_img},{wl.heads},{wl.head_dim}] bf16",
                       "per_micro_step_ms": call_norm_ms,
                       "per_micro_step_what": f"Q_p and K_p of one patch [1,{P},{wl.heads},{wl.head_dim}], L2 flushed"},
    }


def scatter_record(wl, traffic):
    """The fresh-K/V scatter is fused into the attention launch: its algorithmic bytes per
    call (K_p and V_p read and written), and their share of the launch's DRAM traffic."""
    b = 2 * 2 * wl.batch * wl.patch_len * wl.heads * wl.head_dim * 2
    rec = {"bytes_per_call": b, "fused_into": attn_kernel_name(wl),
           "launch_dram_bytes": traffic, "share_of_launch_dram": (b / traffic) if traffic else None}
    return rec


def run_gpu(args, world, rank, local):
    import patch_attention_b200 as pa

    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    sms = n_sms(dev)
    wl = synth.ATTN_WORKLOADS[args.workload]
    r = StepRunner(pa, wl, dev, args.seed if args.seed is not None else synth.default_seed(wl.name))
    r.warm(args.warmup)
    total_ms, attn_ms, cfg_ms, clock_info = r.run(args.steps, args.warmup + 1, world)

    ms_step = max_over_ranks(total_ms / args.steps, world)
    L, M, P = wl.n_layers, wl.n_patches, wl.patch_len
    flop_step = L * wl.flop_per_layer_step()
    value = world * flop_step / (ms_step * 1e-3) / 1e12
    traffic = load_traffic(wl.name)
    roof = attn_roofline(wl, attn_ms, total_ms / 1e3, peaks, peak_src, clock_info, sms, traffic)
    cfg_bytes = wl.batch * r.n_cfg * (4 + 4 + 2)
    cfg_gbs = cfg_bytes / (cfg_ms * 1e-3) / 1e9

    cfg_big = measure_cfg_largest(pa, dev, hbm)
    copies = measure_copy_kernels(pa, r, hbm)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, world, r)
    r.close()
    del r
    torch.cuda.empty_cache()

    subs = {}
    if not args.no_sub:
        for name in ("sd3", "pixart"):
            if name != wl.name:
                subs[name] = sub_record(pa, name, dev, None, world, peaks, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    line = {
        "metric": "patch-attn TFLOP/s (algorithmic, per diffusion step)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                   "n_img": wl.n_img, "n_patches": M, "patch_len": P, "n_txt": wl.n_txt, "layers": L,
                   "calls_per_step": M * L, "flop_per_step": flop_step, "buffer_halves": BUFFER_HALVES,
                   "cfg_latent": list(CFG_SHAPE[wl.name]), "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (alternating input sets of "
                         f"{(3 * wl.n_img + 2 * wl.n_txt) * wl.heads * wl.head_dim * 2 * L / 1e9:.1f} GB)"},
        "pct_bf16_peak": 100.0 * value / world / roof["peak"],
        "roofline": roof,
        "cfg_combine": {"in_step": {"gb_per_s": cfg_gbs, "frac_hbm": cfg_gbs / hbm, "ms": cfg_ms,
                                    "bytes": cfg_bytes, "latent": [wl.batch] + list(CFG_SHAPE[wl.name])},
                        "largest": cfg_big, "peak_gbs": hbm,
                        "peak_source": f"{peak_src} hbm_gbs"},
        "kvbuf_init": copies["kvbuf_init"],
        "scatter": scatter_record(wl, traffic),
        "qk_rmsnorm": dict(copies["qk_rmsnorm"], share_of_micro_step=copies["qk_rmsnorm"]["per_micro_step_ms"]
                           / (copies["qk_rmsnorm"]["per_micro_step_ms"] + roof["launch_ms"])),
        "hbm_peak_gbs": hbm,
        "attn_ms_per_step": attn_ms,
        "gpu_launches": (M * L + 2) * args.steps,
        "clocks": clock_info,
        "workloads": subs,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def measure_cfg_largest(pa, dev, hbm, reps: int = 20):
    """The guidance kernel alone at the largest sweep size (batch 4 x 16x512x512, fp32 and bf16
    outputs: 8 B read + 6 B written per element), L2 flushed (a 512 MB read) before each
    timed call; median of `reps` calls timed with CUDA events."""
    wl = synth.CfgWorkload("cfg", 4, 16, 512, 512)
    c, u = synth.CfgInputs(wl, device=dev).step_tensors(25)
    n = c.numel() // wl.batch
    out_f = torch.empty_like(c)
    out_b = torch.empty(c.shape, dtype=torch.bfloat16, device=dev)
    rel = torch.empty(wl.batch, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, pa.pf_cfg_workspace_bytes(wl.batch, n)), dtype=torch.uint8, device=dev)
    # flush by reading 512 MB (a read leaves clean lines, so the timed call pays no write-backs)
    flush = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(reps + 3):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pa.pf_cfg_combine_relmae(c, u, wl.w, out_f, out_b, rel, ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    nbytes = c.numel() * (4 + 4 + 4 + 2)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"gb_per_s": gbs, "frac_hbm": gbs / hbm, "ms": ms, "bytes": nbytes,
            "shape": [wl.batch, 16, 512, 512], "outputs": "fp32+bf16", "l2": "flushed before each call"}


def run_e2e(args, world, r: StepRunner):
    """The same step through the C ABI with its inputs copied from pinned host memory and its
    outputs copied back, inside the timed region.  Two device input sets and two output sets
    alternate between steps: step s uploads into set s % 2 on a copy stream (per patch, while
    the previous patch computes) after the kernels of step s - 2 that read that set are done,
    and its outputs stream back on a second copy stream before step s + 2 overwrites them.
    The two host input sets alternate as in the device-resident loop."""
    import patch_attention_b200 as pa

    wl, dev = r.wl, r.dev
    B, H, d, N, M, T, L = wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, wl.n_layers
    P = wl.patch_len
    host = [[{k: v.cpu().pin_memory() for k, v in r.sets[hs][l].items()} for l in range(L)] for hs in range(2)]
    host_out = [[torch.empty(B, N, H, d, dtype=torch.bfloat16).pin_memory() for _ in range(L)] for _ in range(2)]
    hc, hu = r.c_in.cpu().pin_memory(), r.u_in.cpu().pin_memory()
    hcfg = [torch.empty(r.cfg_out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hrel = [torch.empty(B, dtype=torch.float32).pin_memory() for _ in range(2)]
    dev_in = [[{k: torch.empty_like(v, device=dev) for k, v in host[0][l].items()} for l in range(L)] for _ in range(2)]
    dev_out = [[torch.empty(B, N, H, d, dtype=torch.bfloat16, device=dev) for _ in range(L)] for _ in range(2)]
    dcu = [(torch.empty_like(r.c_in), torch.empty_like(r.u_in)) for _ in range(2)]
    dcfg = [torch.empty_like(r.cfg_out) for _ in range(2)]
    drel = [torch.empty(B, dtype=torch.float32, device=dev) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    ev_in = [[torch.cuda.Event() for _ in range(M)] for _ in range(2)]
    ev_out = [[torch.cuda.Event() for _ in range(M)] for _ in range(2)]
    ev_txt = [torch.cuda.Event() for _ in range(2)]
    ev_cfg_in = [torch.cuda.Event() for _ in range(2)]
    ev_cfg = [torch.cuda.Event() for _ in range(2)]
    ev_read_done = [None, None]   # compute finished reading dev_in[b] / dcu[b]
    ev_down_done = [None, None]   # outputs of dev_out[b] / dcfg[b] copied back
    Lb = pa._lib()
    row_bytes = H * d * 2
    counts = {"h2d": 0, "d2h": 0}

    def one_step(s):
        b = s % 2
        hs = host[s % 2]
        h2d = d2h = 0
        with torch.cuda.stream(up):
            if ev_read_done[b] is not None:
                up.wait_event(ev_read_done[b])  # step s-2's kernels no longer read set b
            for l in range(L):
                for k in ("k_txt", "v_txt"):
                    dev_in[b][l][k].copy_(hs[l][k], non_blocking=True)
                    h2d += hs[l][k].numel() * 2
            ev_txt[b].record(up)
            for p in range(M):
                sl = slice(p * P, (p + 1) * P)
                for l in range(L):
                    for k in ("q", "k", "v"):
                        dev_in[b][l][k][:, sl].copy_(hs[l][k][:, sl], non_blocking=True)
                        h2d += hs[l][k][:, sl].numel() * 2
                ev_in[b][p].record(up)
            dcu[b][0].copy_(hc, non_blocking=True)
            dcu[b][1].copy_(hu, non_blocking=True)
            h2d += (hc.numel() + hu.numel()) * 4
            ev_cfg_in[b].record(up)
        if ev_down_done[b] is not None:
            comp.wait_event(ev_down_done[b])  # step s-2's outputs have been copied back
        comp.wait_event(ev_txt[b])
        for p in range(M):
            comp.wait_event(ev_in[b][p])
            off = p * P * row_bytes
            for l in range(L):
                t = dev_in[b][l]
                st = Lb.pf_patch_attn_step(r.pat.ctx, l, p, t["q"].data_ptr() + off, t["k"].data_ptr() + off,
                                           t["v"].data_ptr() + off, t["k_txt"].data_ptr() if T else None,
                                           t["v_txt"].data_ptr() if T else None, dev_out[b][l].data_ptr() + off,
                                           comp.cuda_stream)
                if st != 0:
                    raise pa.PatchAttnError(st, "pf_patch_attn_step")
            ev_out[b][p].record(comp)
        comp.wait_event(ev_cfg_in[b])
        st = Lb.pf_cfg_combine_relmae(dcu[b][0].data_ptr(), dcu[b][1].data_ptr(), B, r.n_cfg, r.cwl.w, None,
                                      dcfg[b].data_ptr(), drel[b].data_ptr(), r.cws.data_ptr(), r.cws.numel(),
                                      comp.cuda_stream)
        if st != 0:
            raise pa.PatchAttnError(st, "pf_cfg_combine_relmae")
        ev_cfg[b].record(comp)
        e = torch.cuda.Event()
        e.record(comp)
        ev_read_done[b] = e
        with torch.cuda.stream(down):
            for p in range(M):
                down.wait_event(ev_out[b][p])
                sl = slice(p * P, (p + 1) * P)
                for l in range(L):
                    host_out[b][l][:, sl].copy_(dev_out[b][l][:, sl], non_blocking=True)
                    d2h += dev_out[b][l][:, sl].numel() * 2
            down.wait_event(ev_cfg[b])
            hcfg[b].copy_(dcfg[b], non_blocking=True)
            hrel[b].copy_(drel[b], non_blocking=True)
            d2h += dcfg[b].numel() * 2 + drel[b].numel() * 4
            e2 = torch.cuda.Event()
            e2.record(down)
            ev_down_done[b] = e2
        counts["h2d"], counts["d2h"] = h2d, d2h

    for s in range(max(1, args.warmup)):
        one_step(s)
    torch.cuda.synchronize(dev)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    start.record(comp)
    up.wait_event(start)
    down.wait_event(start)
    s0 = max(1, args.warmup)
    for s in range(s0, s0 + args.steps):
        one_step(s)
    comp.wait_stream(up)
    comp.wait_stream(down)
    stop.record(comp)
    torch.cuda.synchronize(dev)
    barrier(world)
    r.pat.check()
    ms = max_over_ranks(start.elapsed_time(stop) / args.steps, world)
    value = world * L * wl.flop_per_layer_step() / (ms * 1e-3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "ms_per_step": ms, "h2d_bytes_per_step": counts["h2d"],
            "d2h_bytes_per_step": counts["d2h"],
            "copies": "pinned host, two alternating host and device sets, uploads per patch on one "
                      "copy stream and downloads on another, each buffer reused only after the "
                      "kernels and copies of the step two before have finished with it"}


def run_profile_calls(args):
    """For ncu captures: the start-up pass and `n` micro-steps (patches 0..n-1) of one layer of
    the workload, nothing else.  Small device footprint (one layer)."""
    import patch_attention_b200 as pa

    wl0 = synth.ATTN_WORKLOADS[args.workload]
    wl = synth.AttnWorkload(wl0.name, wl0.batch, wl0.heads, wl0.head_dim, wl0.grid_h, wl0.grid_w,
                            wl0.n_patches, wl0.n_txt, 1, 2, wl0.ar_a, wl0.ar_b, wl0.qk_rmsnorm)
    t = synth.AttnInputs(wl, device="cuda").step_tensors(0)
    pat = pa.PatchAttention(wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, 1,
                            schedule=pipefusion_schedule(pa))
    pat.init_layer(0, t["k"], t["v"])
    P = wl.patch_len
    for p in range(min(args.profile_calls, wl.n_patches)):
        sl = slice(p * P, (p + 1) * P)
        pat.step(0, p, t["q"][:, sl].contiguous(), t["k"][:, sl].contiguous(),
                 t["v"][:, sl].contiguous(), t["k_txt"], t["v_txt"])
    torch.cuda.synchronize()
    pat.check()
    pat.close()
    return 0


def run_profile_norm(args):
    """For ncu captures: two per-head RMS normalisations of a full-spatial Q of the workload."""
    import patch_attention_b200 as pa

    wl = synth.ATTN_WORKLOADS[args.workload]
    g = torch.Generator(device="cuda").manual_seed(5)
    x = torch.randn(wl.batch, wl.n_img, wl.heads, wl.head_dim, device="cuda", generator=g).bfloat16()
    for _ in range(2):
        pa.pf_qk_rmsnorm(x)
    torch.cuda.synchronize()
    return 0


def run_profile_cfg(args):
    """For ncu captures: two guidance-kernel calls at the largest sweep size."""
    import patch_attention_b200 as pa

    wl = synth.CfgWorkload("cfg", 4, 16, 512, 512)
    c, u = synth.CfgInputs(wl, device="cuda").step_tensors(25)
    for _ in range(2):
        pa.cfg_combine_relmae(c, u, wl.w)
    torch.cuda.synchronize()
    return 0


def main():
    global BUFFER_HALVES
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run the start-up pass and this many micro-steps of one layer (for ncu)")
    ap.add_argument("--profile-cfg", action="store_true",
                    help="only run two guidance-kernel calls at the largest size (for ncu)")
    ap.add_argument("--profile-norm", action="store_true",
                    help="only run two RMS normalisations of a full-spatial Q of the workload (for ncu)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--buffer-halves", type=int, default=BUFFER_HALVES, choices=[1, 2],
                    help="PipeFusion over one K/V buffer half per layer or two (same results)")
    ap.add_argument("--steps", type=int, default=12)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="patchattn", choices=["patchattn", "reference"])
    ap.add_argument("--workload", default="flux", choices=sorted(synth.ATTN_WORKLOADS))
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true",
                    help="skip the sd3/pixart sub-records (timed over >= 2 s each)")
    args = ap.parse_args()
    BUFFER_HALVES = args.buffer_halves
    if args.warmup < 3 and args.impl != "reference":
        args.warmup = 3
    if args.profile_calls > 0:
        return run_profile_calls(args)
    if args.profile_cfg:
        return run_profile_cfg(args)
    if args.profile_norm:
        return run_profile_norm(args)
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device for the patchattn implementation")
        return run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
