"""Build ``libpatchattn.so`` in-tree with nvcc for sm_100a.

    python -m patch_attention_b200.build [--force] [--ptxas-verbose]

Every CUDA source is compiled with ``-gencode arch=compute_100a,code=sm_100a -lineinfo``;
the host API is compiled by nvcc's host compiler and everything is linked against the
static CUDA runtime, so the library needs only the driver at run time.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpatchattn.so")
OBJDIR = os.path.join(HERE, "_build")

SOURCES = ["attn_fwd.cu", "cfg_combine.cu", "kvbuf_copy.cu", "qk_rmsnorm.cu", "pf_api.cpp"]
HEADERS = ["pf_internal.h", "sm100_ptx.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True,
          trace: bool = False) -> str:
    """trace=True builds libpatchattn_trace.so with per-tile timestamps of CTA 0 (profiling)."""
    objdir = OBJDIR + ("_trace" if trace else "")
    lib = LIB.replace(".so", "_trace.so") if trace else LIB
    extra = ["-DPF_TRACE"] if trace else []
    os.makedirs(objdir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "patchattn.h")]
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(objdir, src + ".o")
        objs.append(obj)
        if force or _stale(obj, [path] + hdrs):
            cmd = [NVCC] + ARCH + COMMON + extra + ["-c", path, "-o", obj]
            if ptxas_verbose and src.endswith(".cu"):
                cmd += ["-Xptxas", "-v"]
            if src.endswith(".cpp"):
                cmd = [NVCC] + ARCH + COMMON + ["-x", "c++", "-c", path, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0 or not quiet:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}")
    if force or _stale(lib, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--trace", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose, quiet=not a.ptxas_verbose, trace=a.trace))
