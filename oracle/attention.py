"""Plain fp64 definition of PipeFusion patch attention on one device.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed, and where the pages say so
--------------------------------------------
* Patch partition -- "기술 요약: PipeFusion", 핵심 메커니즘 1 (이중 분할, 패치 분할), and
  "PipeFusion: Patch-level Pipeline Parallelism for Diffusion Transformers Inference",
  Résumé Technique / Double Partitionnement: the image tokens are cut into M
  non-overlapping patches.  Reading used here: patch p is the contiguous row-major token
  range [p*P, (p+1)*P), P = N_img / M (row bands of the latent grid).
* Stale reuse -- same pages, 핵심 메커니즘 2 (시간적 중복성 활용) / Exploitation de la
  Redondance Temporelle: at step T the context of rows that have not been recomputed
  yet comes from step T+1 (the previous sampler step).  Patches of a step are visited
  in order (3. 통신 최적화: micro-step patch activations are sent on in sequence), so when
  patch p is computed at step s the rows of patches <= p are this step's values and the
  rows of patches > p are step s-1's.  At the first step every row is the first step's
  value (the start-up pass before any stale data exists).
* Full attention -- 주요 기여 (the DiT full-attention mechanism): every query of the patch
  attends to every key, no mask.  Text tokens (MM-DiT joint attention, named in
  중요성 및 주장) are appended as always-fresh keys/values.

Arrays are numpy float64 with layout [tokens, H, d] (one batch element) unless stated.
"""
from __future__ import annotations

import numpy as np


def softmax_probs(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Row-stochastic attention weights, [H, n_q, n_k], max-subtracted softmax in fp64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    logits = np.matmul(q.transpose(1, 0, 2), k.transpose(1, 2, 0)) * scale
    logits = logits - logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    return w / w.sum(axis=-1, keepdims=True)


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """O = softmax(scale * Q K^T) V per head.  q [n_q,H,d], k/v [n_k,H,d] -> [n_q,H,d]."""
    w = softmax_probs(q, k, scale)
    v = np.asarray(v, dtype=np.float64)
    return np.matmul(w, v.transpose(1, 0, 2)).transpose(1, 0, 2)


def image_key_rows(x_now: np.ndarray, x_prev: np.ndarray, p: int, n_patches: int) -> np.ndarray:
    """Image-row context seen by patch p: rows of patches <= p from this step, others stale.

    x_now / x_prev: [N_img, ...] (any dtype: also used on raw bf16 bit patterns).
    """
    n_img = x_now.shape[0]
    plen = n_img // n_patches
    fresh = (np.arange(n_img) // plen) <= p
    shape = (n_img,) + (1,) * (x_now.ndim - 1)
    return np.where(fresh.reshape(shape), x_now, x_prev)


def patch_keys(x_now, x_prev, x_txt, p, n_patches):
    """Full key (or value) set of patch p: image rows (fresh/stale) followed by text rows."""
    return np.concatenate([image_key_rows(x_now, x_prev, p, n_patches), x_txt], axis=0)


def patch_attention(q_now, k_now, v_now, k_prev, v_prev, k_txt, v_txt, p, n_patches, scale,
                    rows=None):
    """Output rows of patch p at a step, by the plain definition.

    q_now, k_now, v_now : [N_img, H, d] this step's full-spatial activations
    k_prev, v_prev      : [N_img, H, d] the previous step's (pass k_now/v_now at step 0)
    k_txt, v_txt        : [T, H, d] this step's text keys/values (T may be 0)
    rows                : optional indices *within the patch* to evaluate (default all)
    returns             : [len(rows) or P, H, d] float64
    """
    plen = q_now.shape[0] // n_patches
    idx = np.arange(plen) if rows is None else np.asarray(rows)
    q = q_now[p * plen + idx]
    k = patch_keys(k_now, k_prev, k_txt, p, n_patches)
    v = patch_keys(v_now, v_prev, v_txt, p, n_patches)
    return attend(q, k, v, scale)


def distrifusion_attention(q_now, k_now, v_now, k_prev, v_prev, k_txt, v_txt, p, n_patches,
                           scale, rows=None):
    """Output rows of patch p under the DistriFusion schedule.

    "기술 요약: PipeFusion", 문제 정의 (DistriFusion): every device keeps the full-spatial K/V of
    every layer and works from the previous step's activations; 주요 기여 / 품질 보존: it relies
    on stale data more than PipeFusion.  Reading used here: patch p sees its own rows at this
    step and every other image row at the previous step, whatever order the patches run in.
    """
    plen = q_now.shape[0] // n_patches
    idx = np.arange(plen) if rows is None else np.asarray(rows)
    own = np.zeros(k_now.shape[0], dtype=bool)
    own[p * plen:(p + 1) * plen] = True
    shape = (k_now.shape[0],) + (1,) * (k_now.ndim - 1)
    k_img = np.where(own.reshape(shape), k_now, k_prev)
    v_img = np.where(own.reshape(shape), v_now, v_prev)
    q = q_now[p * plen + idx]
    return attend(q, np.concatenate([k_img, k_txt], axis=0), np.concatenate([v_img, v_txt], axis=0),
                  scale)


def expected_buffer(x_now, x_prev, p, n_patches):
    """Contents of a layer's KV buffer after the call for patch p (image rows only)."""
    return image_key_rows(x_now, x_prev, p, n_patches)


class KVBufferWalk:
    """Stateful restatement: one layer's full-spatial K/V buffer walked patch by patch.

    init(k0, v0) fills the buffer with the first step's activations (the start-up pass).
    step(p, q_p, k_p, v_p, k_txt, v_txt) writes the patch's fresh K/V rows into the
    buffer, then attends the patch's queries to [buffer ; text].  Patches must come in
    order 0..M-1, then wrap to the next step.
    """

    def __init__(self, n_img: int, n_patches: int, scale: float):
        if n_img % n_patches:
            raise ValueError("n_img must be a multiple of n_patches")
        self.n_img, self.n_patches, self.scale = n_img, n_patches, scale
        self.plen = n_img // n_patches
        self.k = None
        self.v = None
        self.next_patch = 0

    def init(self, k0: np.ndarray, v0: np.ndarray) -> None:
        self.k = np.array(k0, dtype=np.float64, copy=True)
        self.v = np.array(v0, dtype=np.float64, copy=True)
        self.next_patch = 0

    def step(self, p, q_p, k_p, v_p, k_txt, v_txt):
        if self.k is None:
            raise RuntimeError("buffer not initialised")
        if p != self.next_patch:
            raise RuntimeError(f"patch {p} out of order (expected {self.next_patch})")
        lo, hi = p * self.plen, (p + 1) * self.plen
        self.k[lo:hi] = k_p
        self.v[lo:hi] = v_p
        self.next_patch = (p + 1) % self.n_patches
        k = np.concatenate([self.k, k_txt], axis=0)
        v = np.concatenate([self.v, v_txt], axis=0)
        return attend(np.asarray(q_p, dtype=np.float64), k, v, self.scale)
