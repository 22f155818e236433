"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the fp64 oracle.

This module only draws random numbers and shapes them; it holds none of the
patch-attention or guidance arithmetic.  Both sides consume the *same* tensors
it returns (the oracle after an exact bf16 -> fp64 widening).

Workloads (shapes as listed for the five synthetic configurations):

* Attention inputs follow the temporal-redundancy premise of "기술 요약: PipeFusion"
  (section 핵심 메커니즘, 2. 시간적 중복성 활용): consecutive diffusion steps are similar.
  Every tensor X in {Q, K, V, K_txt, V_txt} of every layer is an AR(1) sequence
      X_0 = Z_0,   X_s = a * X_{s-1} + b * Z_s,   Z_s ~ N(0, 1) i.i.d.
  kept in fp32; the tensor used at step s is bf16(round-to-nearest-even(X_s)).
  The Flux-like workload additionally RMS-normalises Q, K and K_txt per (token, head)
  before rounding (x / sqrt(mean_d x^2 + 1e-6), no gain) -- a model feature of the
  input, not part of the attention method.
* Guidance inputs: eps_u ~ N(0,1) fp32, eps_c = eps_u + s_t * N(0,1) with s_t falling
  linearly from 1.0 (t = 0) to 0.05 (t = T-1).

Every stream is a torch.Generator seeded from (seed, tensor id, layer) so that tensors
are independent of the order in which they are drawn.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

# ----------------------------------------------------------------------------------------
# workload table
# ----------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    name: str
    batch: int
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    n_patches: int
    n_txt: int
    n_layers: int
    n_steps: int
    ar_a: float
    ar_b: float
    qk_rmsnorm: bool = False

    @property
    def n_img(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def patch_len(self) -> int:
        return self.n_img // self.n_patches

    @property
    def n_kv(self) -> int:
        return self.n_img + self.n_txt

    @property
    def softmax_scale(self) -> float:
        return self.head_dim ** -0.5

    def flop_per_layer_step(self) -> float:
        """Algorithmic FLOP of one layer for one diffusion step: QK^T and PV, real head_dim."""
        return 4.0 * self.batch * self.n_img * self.n_kv * self.head_dim * self.heads

    def flop_per_call(self) -> float:
        return 4.0 * self.batch * self.patch_len * self.n_kv * self.head_dim * self.heads


ATTN_WORKLOADS: Dict[str, AttnWorkload] = {
    # 16x16 latent, 4 row-patches of 64 tokens, no text, 3 steps
    "tiny": AttnWorkload("tiny", 1, 2, 64, 16, 16, 4, 0, 1, 3, 0.95, 0.3),
    # PixArt-like 1024px layer: 64x64 latent, 8 patches, 120 text tokens, head_dim 72
    "pixart": AttnWorkload("pixart", 1, 16, 72, 64, 64, 8, 120, 1, 20, 0.95, 0.3),
    # SD3-like 2048px joint attention: 128x128 latent, 8 patches, 154 text tokens, 4 layers
    "sd3": AttnWorkload("sd3", 1, 24, 64, 128, 128, 8, 154, 4, 28, 0.97, 0.25),
    # Flux-like 4096px: 256x256 latent, 16 patches, 512 text tokens, 4 layers, QK RMSNorm
    "flux": AttnWorkload("flux", 1, 24, 128, 256, 256, 16, 512, 4, 8, 0.97, 0.25, True),
}


@dataclasses.dataclass(frozen=True)
class CfgWorkload:
    name: str
    batch: int
    channels: int
    height: int
    width: int
    n_steps: int = 50
    s_first: float = 1.0
    s_last: float = 0.05
    w: float = 7.0

    @property
    def n_per_sample(self) -> int:
        return self.channels * self.height * self.width

    def s_t(self, t: int) -> float:
        if self.n_steps == 1:
            return self.s_first
        return self.s_first + (self.s_last - self.s_first) * t / (self.n_steps - 1)


CFG_SHAPES = [(4, 128, 128), (16, 256, 256), (16, 512, 512)]

TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "k_txt": 4, "v_txt": 5, "eps_u": 6, "eps_c": 7}


def _stream_seed(seed: int, tensor: str, layer: int) -> int:
    # a fixed mixing of (seed, tensor id, layer) into a 63-bit generator seed
    x = (seed * 0x9E3779B97F4A7C15 + TENSOR_IDS[tensor] * 0xBF58476D1CE4E5B9
         + (layer + 1) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    x ^= x >> 31
    x = (x * 0xD6E8FEB86659FD93) & 0xFFFFFFFFFFFFFFFF
    x ^= x >> 32
    return x & 0x7FFFFFFFFFFFFFFF


def default_seed(name: str) -> int:
    order = ["tiny", "pixart", "sd3", "flux", "cfg"]
    if name in order:
        return 20260000 + order.index(name)
    return 20261000 + sum(ord(ch) * 31 ** i for i, ch in enumerate(name)) % 100000


# ----------------------------------------------------------------------------------------
# AR(1) attention inputs
# ----------------------------------------------------------------------------------------


class _AR1:
    """One AR(1) tensor sequence: fp32 state, bf16 view per step."""

    def __init__(self, shape, a, b, seed, device, rmsnorm: bool):
        self.shape = tuple(shape)
        self.a, self.b = float(a), float(b)
        self.gen = torch.Generator(device=device)
        self.gen.manual_seed(seed)
        self.device = device
        self.rmsnorm = rmsnorm
        self.state: Optional[torch.Tensor] = None
        self.step = -1

    def _noise(self) -> torch.Tensor:
        return torch.randn(self.shape, generator=self.gen, device=self.device, dtype=torch.float32)

    def advance(self) -> torch.Tensor:
        z = self._noise()
        if self.state is None:
            self.state = z
        else:
            self.state.mul_(self.a).add_(z, alpha=self.b)
            del z
        self.step += 1
        return self.current()

    def current(self) -> torch.Tensor:
        x = self.state
        if self.rmsnorm and x.numel() > 0:
            x = x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-6)
        return x.to(torch.bfloat16)


class AttnInputs:
    """Per-layer AR(1) streams for one attention workload.

    ``step_tensors(layer)`` advances that layer's five streams by one diffusion step and
    returns a dict of bf16 tensors: q, k, v of shape [B, N_img, H, d] and k_txt, v_txt of
    shape [B, T, H, d].  Layers are independent (no weights link them), so each layer
    keeps its own step counter.
    """

    def __init__(self, wl: AttnWorkload, seed: Optional[int] = None, device="cpu",
                 a: Optional[float] = None, b: Optional[float] = None):
        self.wl = wl
        self.seed = default_seed(wl.name) if seed is None else seed
        self.device = torch.device(device)
        a = wl.ar_a if a is None else a
        b = wl.ar_b if b is None else b
        img = (wl.batch, wl.n_img, wl.heads, wl.head_dim)
        txt = (wl.batch, wl.n_txt, wl.heads, wl.head_dim)
        self.streams: List[Dict[str, _AR1]] = []
        for layer in range(wl.n_layers):
            d = {}
            for name, shape in (("q", img), ("k", img), ("v", img), ("k_txt", txt), ("v_txt", txt)):
                norm = wl.qk_rmsnorm and name in ("q", "k", "k_txt")
                d[name] = _AR1(shape, a, b, _stream_seed(self.seed, name, layer), self.device, norm)
            self.streams.append(d)

    def step_tensors(self, layer: int) -> Dict[str, torch.Tensor]:
        return {name: s.advance() for name, s in self.streams[layer].items()}


def patch_rows(t: torch.Tensor, p: int, n_patches: int) -> torch.Tensor:
    """Rows [p*P, (p+1)*P) of a [B, N, H, d] tensor, as a contiguous tensor."""
    P = t.shape[1] // n_patches
    return t[:, p * P:(p + 1) * P].contiguous()


# ----------------------------------------------------------------------------------------
# guidance inputs
# ----------------------------------------------------------------------------------------


class CfgInputs:
    """eps_u ~ N(0,1), eps_c = eps_u + s_t * N(0,1), fp32 [B, C, H, W], for t = 0..T-1."""

    def __init__(self, wl: CfgWorkload, seed: Optional[int] = None, device="cpu"):
        self.wl = wl
        self.seed = default_seed("cfg") if seed is None else seed
        self.device = torch.device(device)
        shape = (wl.batch, wl.channels, wl.height, wl.width)
        self.shape = shape
        self.gen_u = torch.Generator(device=self.device)
        self.gen_u.manual_seed(_stream_seed(self.seed, "eps_u", wl.channels * 100003 + wl.height))
        self.gen_c = torch.Generator(device=self.device)
        self.gen_c.manual_seed(_stream_seed(self.seed, "eps_c", wl.channels * 100003 + wl.height))

    def step_tensors(self, t: int):
        u = torch.randn(self.shape, generator=self.gen_u, device=self.device, dtype=torch.float32)
        z = torch.randn(self.shape, generator=self.gen_c, device=self.device, dtype=torch.float32)
        c = u + self.wl.s_t(t) * z
        return c, u
