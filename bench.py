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


def run_gpu(args, world, rank, local):
    import patch_attention_b200 as pa

    dev = torch.device("cuda", local)
    wl = synth.ATTN_WORKLOADS[args.workload]
    B, H, d, N, M, T, L = wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, wl.n_layers
    P = wl.patch_len
    assert B == 1, "patch slices are passed as views; batch 1 keeps them contiguous"

    # two input sets so consecutive steps see different activations (AR(1) steps)
    gen = synth.AttnInputs(wl, seed=args.seed, device=dev)
    sets = [[gen.step_tensors(l) for l in range(L)] for _ in range(2)]
    del gen  # drop the fp32 AR(1) state
    torch.cuda.empty_cache()
    pat = pa.PatchAttention(B, H, d, N, M, T, L)
    for l in range(L):
        pat.init_layer(l, sets[0][l]["k"], sets[0][l]["v"])
    outs = [torch.empty(B, N, H, d, dtype=torch.bfloat16, device=dev) for _ in range(L)]

    cshape = CFG_SHAPE[wl.name]
    cwl = synth.CfgWorkload("cfg", B, *cshape)
    c_in, u_in = synth.CfgInputs(cwl, device=dev).step_tensors(25)
    n_cfg = c_in.numel() // B
    cfg_out = torch.empty(c_in.shape, dtype=torch.bfloat16, device=dev)
    rel = torch.empty(B, dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, pa.pf_cfg_workspace_bytes(B, n_cfg)), dtype=torch.uint8, device=dev)

    L_ = pa._lib()
    ctx = pat.ctx
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    row_bytes = H * d * 2

    # precomputed pointers: the timed loop is argument marshalling only
    ptrs = []
    for s in range(2):
        per = []
        for l in range(L):
            t = sets[s][l]
            per.append((t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(),
                        t["k_txt"].data_ptr() if T else None, t["v_txt"].data_ptr() if T else None))
        ptrs.append(per)
    optrs = [o.data_ptr() for o in outs]

    def attn_section(set_idx):
        per = ptrs[set_idx]
        for p in range(M):
            off = p * P * row_bytes
            for l in range(L):
                q, k, v, kt, vt = per[l]
                st = L_.pf_patch_attn_step(ctx, l, p, q + off, k + off, v + off, kt, vt, optrs[l] + off, sh)
                if st != 0:
                    raise pa.PatchAttnError(st, "pf_patch_attn_step")

    def cfg_section():
        st = L_.pf_cfg_combine_relmae(c_in.data_ptr(), u_in.data_ptr(), B, n_cfg, cwl.w, None,
                                      cfg_out.data_ptr(), rel.data_ptr(), ws.data_ptr(), ws.numel(), sh)
        if st != 0:
            raise pa.PatchAttnError(st, "pf_cfg_combine_relmae")

    ev = lambda: torch.cuda.Event(enable_timing=True)
    launches_per_step = M * L + 2

    # warm-up (the first step also validates the whole path)
    for i in range(args.warmup):
        attn_section((i + 1) % 2)
        cfg_section()
    torch.cuda.synchronize(dev)
    pat.check()

    a0 = [ev() for _ in range(args.steps)]
    a1 = [ev() for _ in range(args.steps)]
    c1 = [ev() for _ in range(args.steps)]
    start, stop = ev(), ev()
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler attach before the timed region
    start.record(stream)
    for i in range(args.steps):
        a0[i].record(stream)
        attn_section((args.warmup + i + 1) % 2)
        a1[i].record(stream)
        cfg_section()
        c1[i].record(stream)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    barrier(world)
    pat.check()

    total_ms = start.elapsed_time(stop)
    ms_step = max_over_ranks(total_ms / args.steps, world)
    attn_ms = sum(a0[i].elapsed_time(a1[i]) for i in range(args.steps)) / args.steps
    cfg_ms = sum(a1[i].elapsed_time(c1[i]) for i in range(args.steps)) / args.steps
    flop_step = L * wl.flop_per_layer_step()
    value = world * flop_step / (ms_step * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    launch_ms = attn_ms / (M * L)
    achieved = wl.flop_per_call() / (launch_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    traffic = load_traffic(wl.name)
    cfg_bytes = B * n_cfg * (4 + 4 + 2)
    cfg_gbs = cfg_bytes / (cfg_ms * 1e-3) / 1e9
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    cfg_big = measure_cfg_largest(pa, dev, hbm)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, world, local, wl, sets, pat, outs, c_in, u_in, cfg_out, rel, ws, cwl, n_cfg)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    line = {
        "metric": "patch-attn TFLOP/s (algorithmic, per diffusion step)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "heads": H, "head_dim": d, "n_img": N,
                   "n_patches": M, "patch_len": P, "n_txt": T, "layers": L,
                   "calls_per_step": M * L, "flop_per_step": flop_step,
                   "cfg_latent": list(cshape), "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (two alternating input sets of "
                         f"{2 * L * 3 * N * H * d * 2 / 1e9:.1f} GB)"},
        "pct_bf16_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "kernel": "patch_attn_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)"},
        "cfg_combine": {"in_step": {"gb_per_s": cfg_gbs, "frac_hbm": cfg_gbs / hbm, "ms": cfg_ms,
                                    "bytes": cfg_bytes, "latent": [B] + list(cshape)},
                        "largest": cfg_big, "peak_gbs": hbm,
                        "peak_source": f"{peak_src} hbm_gbs"},
        "attn_ms_per_step": attn_ms,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clock_info,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    pat.close()
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


def run_e2e(args, world, local, wl, sets, pat, outs, c_in, u_in, cfg_out, rel, ws, cwl, n_cfg):
    """Same step, inputs from pinned host memory: per patch, the rows of every layer are
    copied on a copy stream while the previous patch computes; outputs stream back on a
    third stream; the guidance inputs go up and the guided eps + rel-MAE come back."""
    import patch_attention_b200 as pa

    dev = torch.device("cuda", local)
    B, H, d, N, M, T, L = wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, wl.n_layers
    P = wl.patch_len
    host = [{k: v.cpu().pin_memory() for k, v in sets[0][l].items()} for l in range(L)]
    host_out = [torch.empty(B, N, H, d, dtype=torch.bfloat16).pin_memory() for _ in range(L)]
    hc, hu = c_in.cpu().pin_memory(), u_in.cpu().pin_memory()
    hcfg = torch.empty(cfg_out.shape, dtype=torch.bfloat16).pin_memory()
    hrel = torch.empty(B, dtype=torch.float32).pin_memory()
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in host[l].items()} for l in range(L)]
    dc, du = torch.empty_like(c_in), torch.empty_like(u_in)
    comp = torch.cuda.current_stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(M)]
    ev_out = [torch.cuda.Event() for _ in range(M)]
    ev_txt = torch.cuda.Event()
    ev_cfg = torch.cuda.Event()
    Lb = pa._lib()
    row_bytes = H * d * 2
    h2d = 0
    d2h = 0

    def one_step():
        nonlocal h2d, d2h
        h2d = d2h = 0
        with torch.cuda.stream(up):
            for l in range(L):
                for k in ("k_txt", "v_txt"):
                    dev_in[l][k].copy_(host[l][k], non_blocking=True)
                    h2d += host[l][k].numel() * 2
            ev_txt.record(up)
            for p in range(M):
                sl = slice(p * P, (p + 1) * P)
                for l in range(L):
                    for k in ("q", "k", "v"):
                        dev_in[l][k][:, sl].copy_(host[l][k][:, sl], non_blocking=True)
                        h2d += host[l][k][:, sl].numel() * 2
                ev_in[p].record(up)
            dc.copy_(hc, non_blocking=True)
            du.copy_(hu, non_blocking=True)
            h2d += (hc.numel() + hu.numel()) * 4
        comp.wait_event(ev_txt)
        for p in range(M):
            comp.wait_event(ev_in[p])
            off = p * P * row_bytes
            for l in range(L):
                t = dev_in[l]
                st = Lb.pf_patch_attn_step(pat.ctx, l, p, t["q"].data_ptr() + off, t["k"].data_ptr() + off,
                                           t["v"].data_ptr() + off, t["k_txt"].data_ptr() if T else None,
                                           t["v_txt"].data_ptr() if T else None, outs[l].data_ptr() + off,
                                           comp.cuda_stream)
                if st != 0:
                    raise pa.PatchAttnError(st, "pf_patch_attn_step")
            ev_out[p].record(comp)
        comp.wait_stream(up)
        st = Lb.pf_cfg_combine_relmae(dc.data_ptr(), du.data_ptr(), B, n_cfg, cwl.w, None, cfg_out.data_ptr(),
                                      rel.data_ptr(), ws.data_ptr(), ws.numel(), comp.cuda_stream)
        if st != 0:
            raise pa.PatchAttnError(st, "pf_cfg_combine_relmae")
        ev_cfg.record(comp)
        with torch.cuda.stream(down):
            for p in range(M):
                down.wait_event(ev_out[p])
                sl = slice(p * P, (p + 1) * P)
                for l in range(L):
                    host_out[l][:, sl].copy_(outs[l][:, sl], non_blocking=True)
                    d2h += outs[l][:, sl].numel() * 2
            down.wait_event(ev_cfg)
            hcfg.copy_(cfg_out, non_blocking=True)
            hrel.copy_(rel, non_blocking=True)
            d2h += cfg_out.numel() * 2 + rel.numel() * 4
        comp.wait_stream(down)

    for _ in range(max(1, args.warmup)):
        one_step()
    torch.cuda.synchronize(dev)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    start.record(comp)
    for _ in range(args.steps):
        one_step()
    stop.record(comp)
    torch.cuda.synchronize(dev)
    barrier(world)
    pat.check()
    ms = max_over_ranks(start.elapsed_time(stop) / args.steps, world)
    value = world * L * wl.flop_per_layer_step() / (ms * 1e-3) / 1e12
    return {"value": value, "unit": "TFLOP/s", "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "copies": "pinned host, overlapped per patch on two copy streams"}


def run_profile_calls(args):
    """For ncu captures: the start-up pass and `n` micro-steps (patches 0..n-1) of one layer of
    the workload, nothing else.  Small device footprint (one layer)."""
    import patch_attention_b200 as pa

    wl0 = synth.ATTN_WORKLOADS[args.workload]
    wl = synth.AttnWorkload(wl0.name, wl0.batch, wl0.heads, wl0.head_dim, wl0.grid_h, wl0.grid_w,
                            wl0.n_patches, wl0.n_txt, 1, 2, wl0.ar_a, wl0.ar_b, wl0.qk_rmsnorm)
    t = synth.AttnInputs(wl, device="cuda").step_tensors(0)
    pat = pa.PatchAttention(wl.batch, wl.heads, wl.head_dim, wl.n_img, wl.n_patches, wl.n_txt, 1)
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
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="only run the start-up pass and this many micro-steps of one layer (for ncu)")
    ap.add_argument("--profile-cfg", action="store_true",
                    help="only run two guidance-kernel calls at the largest size (for ncu)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="patchattn", choices=["patchattn", "reference"])
    ap.add_argument("--workload", default="flux", choices=sorted(synth.ATTN_WORKLOADS))
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl != "reference":
        args.warmup = 3
    if args.profile_calls > 0:
        return run_profile_calls(args)
    if args.profile_cfg:
        return run_profile_cfg(args)
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
