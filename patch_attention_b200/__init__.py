"""Python binding of ``libpatchattn.so`` (B200 / sm_100a PipeFusion patch attention).

The functions below carry the C ABI's names (``include/patchattn.h``) and only marshal
arguments: torch tensors are checked for device, dtype, shape and contiguity, then their
``data_ptr()`` and the current CUDA stream are handed to the library.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback.  If the shared
library has not been built, the first call raises ``ImportError``.

``PatchAttention`` bundles a context with caller-side (torch) K/V buffers.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpatchattn.so")

PF_OK = 0
PF_ERR_INVALID_ARG = 1
PF_ERR_SHAPE = 2
PF_ERR_ALIGN = 3
PF_ERR_UNSUPPORTED = 4
PF_ERR_ORDER = 5
PF_ERR_STATE = 6
PF_ERR_CUDA = 7
PF_ERR_TIMEOUT = 8

PF_SCHED_PIPEFUSION = 0
PF_SCHED_DISTRIFUSION = 1
PF_SCHED_PIPEFUSION_2H = 2

EXPORTED = [
    "pf_kvbuf_bytes", "pf_create", "pf_destroy", "pf_kvbuf_init", "pf_patch_attn_step",
    "pf_get_state", "pf_set_state", "pf_workspace_bytes", "pf_set_workspace",
    "pf_cfg_workspace_bytes", "pf_cfg_combine_relmae", "pf_cfg_combine_relmae_static",
    "pf_check_device_status", "pf_selftest_bounded_wait", "pf_status_string", "pf_version", "pf_switch_init",
    "pf_switch_update", "pf_text_attn_step", "pf_qk_rmsnorm", "pf_get_read_half",
]

PF_PHASE_WARMUP = 0
PF_PHASE_PARALLEL = 1
PF_PHASE_FULL = 2


class pf_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("n_img", ctypes.c_int), ("n_patches", ctypes.c_int), ("n_txt", ctypes.c_int),
        ("n_layers", ctypes.c_int), ("softmax_scale", ctypes.c_float), ("schedule", ctypes.c_int),
    ]


class pf_switch(ctypes.Structure):
    _fields_ = [
        ("enter_below", ctypes.c_float), ("enter_patience", ctypes.c_int),
        ("exit_above", ctypes.c_float), ("max_parallel_steps", ctypes.c_int),
        ("phase", ctypes.c_int), ("step", ctypes.c_int), ("below_run", ctypes.c_int),
        ("parallel_steps", ctypes.c_int), ("tau1", ctypes.c_int), ("tau2", ctypes.c_int),
    ]


class PatchAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pf_status_string(status)} (status {status})")


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m patch_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i, i64, f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        cfgp = ctypes.POINTER(pf_config)
        sig = {
            "pf_kvbuf_bytes": (sz, [cfgp]),
            "pf_create": (i, [cfgp, ctypes.POINTER(vp), ctypes.POINTER(vp)]),
            "pf_destroy": (i, [vp]),
            "pf_kvbuf_init": (i, [vp, i, vp, vp, vp]),
            "pf_patch_attn_step": (i, [vp, i, i, vp, vp, vp, vp, vp, vp, vp]),
            "pf_get_state": (i, [vp, i, ctypes.POINTER(i)]),
            "pf_get_read_half": (i, [vp, i, ctypes.POINTER(i)]),
            "pf_workspace_bytes": (sz, [cfgp]),
            "pf_set_workspace": (i, [vp, vp, sz, vp]),
            "pf_set_state": (i, [vp, i, i]),
            "pf_cfg_workspace_bytes": (sz, [i, i64]),
            "pf_cfg_combine_relmae": (i, [vp, vp, i, i64, f, vp, vp, vp, vp, sz, vp]),
            "pf_cfg_combine_relmae_static": (i, [vp, vp, i, i64, f, vp, vp, vp, vp]),
            "pf_check_device_status": (i, [vp, vp]),
            "pf_selftest_bounded_wait": (i, [ctypes.c_uint64, vp]),
            "pf_status_string": (ctypes.c_char_p, [i]),
            "pf_text_attn_step": (i, [vp, i, vp, vp, vp, vp, vp]),
            "pf_qk_rmsnorm": (i, [vp, i64, i, vp, f, vp]),
            "pf_switch_init": (i, [ctypes.POINTER(pf_switch), f, i, f, i]),
            "pf_switch_update": (i, [ctypes.POINTER(pf_switch), f, ctypes.POINTER(i)]),
            "pf_version": (i, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib_handle = L
    return _lib_handle


def library_path() -> str:
    return LIB_PATH


def pf_status_string(status: int) -> str:
    return _lib().pf_status_string(int(status)).decode()


def pf_version() -> int:
    return int(_lib().pf_version())


def _check(st: int, where: str) -> None:
    if st != PF_OK:
        raise PatchAttnError(st, where)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor], dtype, shape=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def make_config(batch, heads, head_dim, n_img, n_patches, n_txt, n_layers, softmax_scale=0.0,
                schedule=PF_SCHED_PIPEFUSION) -> pf_config:
    return pf_config(batch, heads, head_dim, n_img, n_patches, n_txt, n_layers,
                     float(softmax_scale), schedule)


# ------------------------------------------------------------------ C ABI, same names


def pf_kvbuf_bytes(cfg: pf_config) -> int:
    return int(_lib().pf_kvbuf_bytes(ctypes.byref(cfg)))


def pf_create(cfg: pf_config, kvbuf_ptrs: Sequence[int]) -> ctypes.c_void_p:
    arr = (ctypes.c_void_p * len(kvbuf_ptrs))(*[ctypes.c_void_p(p) for p in kvbuf_ptrs])
    out = ctypes.c_void_p()
    _check(_lib().pf_create(ctypes.byref(cfg), arr, ctypes.byref(out)), "pf_create")
    return out


def pf_destroy(ctx) -> None:
    _check(_lib().pf_destroy(ctx), "pf_destroy")


def pf_kvbuf_init(ctx, layer: int, k_full: torch.Tensor, v_full: torch.Tensor, stream=None,
                  shape=None) -> None:
    k = _ptr(k_full, torch.bfloat16, shape, "k_full")
    v = _ptr(v_full, torch.bfloat16, shape, "v_full")
    _check(_lib().pf_kvbuf_init(ctx, layer, k, v, _stream(stream)), "pf_kvbuf_init")


def pf_patch_attn_step(ctx, layer: int, patch: int, q_p, k_p, v_p, k_txt, v_txt, o_p,
                       stream=None, patch_shape=None, txt_shape=None) -> None:
    bf = torch.bfloat16
    args = (_ptr(q_p, bf, patch_shape, "q_p"), _ptr(k_p, bf, patch_shape, "k_p"),
            _ptr(v_p, bf, patch_shape, "v_p"), _ptr(k_txt, bf, txt_shape, "k_txt"),
            _ptr(v_txt, bf, txt_shape, "v_txt"), _ptr(o_p, bf, patch_shape, "o_p"))
    _check(_lib().pf_patch_attn_step(ctx, layer, patch, *args, _stream(stream)),
           "pf_patch_attn_step")


def pf_text_attn_step(ctx, layer: int, q_txt, k_txt, v_txt, o_txt, stream=None,
                      txt_shape=None) -> None:
    bf = torch.bfloat16
    args = (_ptr(q_txt, bf, txt_shape, "q_txt"), _ptr(k_txt, bf, txt_shape, "k_txt"),
            _ptr(v_txt, bf, txt_shape, "v_txt"), _ptr(o_txt, bf, txt_shape, "o_txt"))
    _check(_lib().pf_text_attn_step(ctx, layer, *args, _stream(stream)), "pf_text_attn_step")


def pf_qk_rmsnorm(x: torch.Tensor, gain: Optional[torch.Tensor] = None, eps: float = 1e-6,
                  stream=None) -> None:
    """Normalise every head vector (last dimension) of the bf16 tensor x in place."""
    d = x.shape[-1]
    xp = _ptr(x, torch.bfloat16, None, "x")
    gp = _ptr(gain, torch.bfloat16, (d,), "gain")
    _check(_lib().pf_qk_rmsnorm(xp, x.numel() // d, d, gp, float(eps), _stream(stream)),
           "pf_qk_rmsnorm")


def pf_workspace_bytes(cfg: pf_config) -> int:
    return int(_lib().pf_workspace_bytes(ctypes.byref(cfg)))


def pf_set_workspace(ctx, ws: Optional[torch.Tensor], stream=None) -> None:
    if ws is None:
        _check(_lib().pf_set_workspace(ctx, None, 0, None), "pf_set_workspace")
        return
    ptr = _ptr(ws, torch.uint8, None, "workspace")
    _check(_lib().pf_set_workspace(ctx, ptr, ws.numel(), _stream(stream)), "pf_set_workspace")


def pf_get_state(ctx, layer: int) -> int:
    v = ctypes.c_int()
    _check(_lib().pf_get_state(ctx, layer, ctypes.byref(v)), "pf_get_state")
    return v.value


def pf_set_state(ctx, layer: int, next_patch: int) -> None:
    _check(_lib().pf_set_state(ctx, layer, next_patch), "pf_set_state")


def pf_get_read_half(ctx, layer: int) -> int:
    v = ctypes.c_int()
    _check(_lib().pf_get_read_half(ctx, layer, ctypes.byref(v)), "pf_get_read_half")
    return v.value


def pf_cfg_workspace_bytes(batch: int, n_per_sample: int) -> int:
    return int(_lib().pf_cfg_workspace_bytes(batch, n_per_sample))


def pf_cfg_combine_relmae(eps_c: torch.Tensor, eps_u: torch.Tensor, w: float,
                          out_f32: Optional[torch.Tensor], out_bf16: Optional[torch.Tensor],
                          relmae: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    B = eps_c.shape[0]
    n = eps_c.numel() // B
    c = _ptr(eps_c, torch.float32, None, "eps_c")
    u = _ptr(eps_u, torch.float32, tuple(eps_c.shape), "eps_u")
    of = _ptr(out_f32, torch.float32, tuple(eps_c.shape), "out_f32")
    ob = _ptr(out_bf16, torch.bfloat16, tuple(eps_c.shape), "out_bf16")
    r = _ptr(relmae, torch.float32, (B,), "relmae")
    ws = _ptr(workspace, torch.uint8, None, "workspace")
    _check(_lib().pf_cfg_combine_relmae(c, u, B, n, float(w), of, ob, r, ws, workspace.numel(),
                                        _stream(stream)), "pf_cfg_combine_relmae")


def pf_cfg_combine_relmae_static(eps_c: torch.Tensor, eps_u: torch.Tensor, w: float,
                                 out_f32: Optional[torch.Tensor], out_bf16: Optional[torch.Tensor],
                                 relmae: torch.Tensor, stream=None) -> None:
    """The guidance combine without a workspace argument: the library keeps its partial sums
    in a fixed device array, so nothing is allocated for the call (batch <= 4096).  Calls
    that run concurrently on the GPU share that array and must not overlap."""
    B = eps_c.shape[0]
    n = eps_c.numel() // B
    c = _ptr(eps_c, torch.float32, None, "eps_c")
    u = _ptr(eps_u, torch.float32, tuple(eps_c.shape), "eps_u")
    of = _ptr(out_f32, torch.float32, tuple(eps_c.shape), "out_f32")
    ob = _ptr(out_bf16, torch.bfloat16, tuple(eps_c.shape), "out_bf16")
    r = _ptr(relmae, torch.float32, (B,), "relmae")
    _check(_lib().pf_cfg_combine_relmae_static(c, u, B, n, float(w), of, ob, r, _stream(stream)),
           "pf_cfg_combine_relmae_static")


class HybridCfgSwitch:
    """Warm-Up -> Parallelism -> Fully-Connecting controller driven by rel-MAE_t (one per
    image); see pf_switch_init in include/patchattn.h for the rule and its parameters."""

    def __init__(self, enter_below: float, enter_patience: int = 1, exit_above: float = float("inf"),
                 max_parallel_steps: int = 0):
        self.state = pf_switch()
        _check(_lib().pf_switch_init(ctypes.byref(self.state), enter_below, enter_patience,
                                     exit_above, max_parallel_steps), "pf_switch_init")

    def update(self, relmae: float) -> int:
        ph = ctypes.c_int()
        _check(_lib().pf_switch_update(ctypes.byref(self.state), float(relmae), ctypes.byref(ph)),
               "pf_switch_update")
        return ph.value

    @property
    def phase(self) -> int:
        return self.state.phase

    @property
    def tau(self):
        return self.state.tau1, self.state.tau2


def pf_check_device_status(ctx, stream=None) -> None:
    _check(_lib().pf_check_device_status(ctx, _stream(stream)), "pf_check_device_status")


def pf_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Run the failure-detection self-test; returns the status (PF_ERR_TIMEOUT as designed)."""
    return int(_lib().pf_selftest_bounded_wait(int(limit_ns), _stream(stream)))


# ------------------------------------------------------------------ convenience


class PatchAttention:
    """A context plus its per-layer K/V buffers, allocated by torch on ``device``.

    Buffer layout per layer (uint8 tensor): K [B, N, H, d] bf16 then V of the same size
    (DistriFusion and two-half PipeFusion schedules: two such halves).
    """

    def __init__(self, batch, heads, head_dim, n_img, n_patches, n_txt, n_layers,
                 softmax_scale=0.0, schedule=PF_SCHED_PIPEFUSION, device="cuda", split=True):
        self.cfg = make_config(batch, heads, head_dim, n_img, n_patches, n_txt, n_layers,
                               softmax_scale, schedule)
        nbytes = pf_kvbuf_bytes(self.cfg)
        if nbytes == 0:
            raise PatchAttnError(PF_ERR_SHAPE, "pf_kvbuf_bytes")
        self.buffers: List[torch.Tensor] = [
            torch.empty(nbytes, dtype=torch.uint8, device=device) for _ in range(n_layers)]
        self.ctx = pf_create(self.cfg, [b.data_ptr() for b in self.buffers])
        self.workspace = None
        wsb = pf_workspace_bytes(self.cfg) if split else 0
        if wsb > 0:
            self.workspace = torch.empty(wsb, dtype=torch.uint8, device=device)
            pf_set_workspace(self.ctx, self.workspace)
        self.plen = n_img // n_patches
        self.patch_shape = (batch, self.plen, heads, head_dim)
        self.full_shape = (batch, n_img, heads, head_dim)
        self.txt_shape = (batch, n_txt, heads, head_dim)

    def init_layer(self, layer, k_full, v_full, stream=None):
        pf_kvbuf_init(self.ctx, layer, k_full, v_full, stream, self.full_shape)

    def step(self, layer, patch, q_p, k_p, v_p, k_txt=None, v_txt=None, out=None, stream=None):
        if out is None:
            out = torch.empty(self.patch_shape, dtype=torch.bfloat16, device=q_p.device)
        if self.cfg.n_txt == 0:
            k_txt = v_txt = None
        pf_patch_attn_step(self.ctx, layer, patch, q_p, k_p, v_p, k_txt, v_txt, out, stream,
                           self.patch_shape, self.txt_shape)
        return out

    def text_step(self, layer, q_txt, k_txt, v_txt, out=None, stream=None):
        """Text-token queries against the layer buffer as it stands plus the text tokens."""
        if out is None:
            out = torch.empty(self.txt_shape, dtype=torch.bfloat16, device=q_txt.device)
        pf_text_attn_step(self.ctx, layer, q_txt, k_txt, v_txt, out, stream, self.txt_shape)
        return out

    def buffer_kv(self, layer, half=0):
        """(K, V) views of a layer's buffer as bf16 [B, N, H, d] tensors."""
        e = self.cfg.batch * self.cfg.n_img * self.cfg.heads * self.cfg.head_dim
        flat = self.buffers[layer].view(torch.bfloat16)
        k = flat[(2 * half) * e:(2 * half + 1) * e].view(self.full_shape)
        v = flat[(2 * half + 1) * e:(2 * half + 2) * e].view(self.full_shape)
        return k, v

    def next_patch(self, layer):
        return pf_get_state(self.ctx, layer)

    def read_half(self, layer):
        return pf_get_read_half(self.ctx, layer)

    def buffer_as_it_stands(self, layer):
        """(K, V) copies of the rows a text-token call on the layer would see now: under the
        two-half PipeFusion schedule the step's patches called so far come from the half being
        written and the other rows from the half being read; otherwise the half being read."""
        rd = self.read_half(layer)
        k, v = (t.clone() for t in self.buffer_kv(layer, rd))
        if self.cfg.schedule == PF_SCHED_PIPEFUSION_2H:
            n = self.next_patch(layer) * self.plen
            kw, vw = self.buffer_kv(layer, 1 - rd)
            k[:, :n] = kw[:, :n]
            v[:, :n] = vw[:, :n]
        return k, v

    def check(self, stream=None):
        pf_check_device_status(self.ctx, stream)

    def close(self):
        if self.ctx is not None:
            pf_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def cfg_combine_relmae(eps_c: torch.Tensor, eps_u: torch.Tensor, w: float, want_f32=True,
                       want_bf16=True, stream=None):
    """Allocate outputs and workspace with torch and run the fused guidance kernel."""
    B = eps_c.shape[0]
    n = eps_c.numel() // B
    out_f = torch.empty_like(eps_c) if want_f32 else None
    out_b = torch.empty(eps_c.shape, dtype=torch.bfloat16, device=eps_c.device) if want_bf16 else None
    rel = torch.empty(B, dtype=torch.float32, device=eps_c.device)
    ws = torch.empty(max(16, pf_cfg_workspace_bytes(B, n)), dtype=torch.uint8, device=eps_c.device)
    pf_cfg_combine_relmae(eps_c, eps_u, w, out_f, out_b, rel, ws, stream)
    return out_f, out_b, rel
