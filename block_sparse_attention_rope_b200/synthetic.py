"""Seeded synthetic inputs and the named workloads.

This module holds no arithmetic of the method: it only names the workload
shapes and draws i.i.d. N(0, 1) tensors from seeded CPU generators.  Both the
GPU path (tests, benchmark) and the fp64 oracle are fed from here, which is the
only thing the two sides share.

Inputs: q, k, v (and the cached condition keys/values) are drawn in fp32 by
``torch.Generator().manual_seed(seed)`` and, for bf16 workloads, rounded to
bf16 (round to nearest even).  Layout [B, N, heads, head_dim], tokens ordered
t-major, then h, then w.  They stand in for the VAE latents of the 480x832 and
720x1280, 93-frame videos the pages' pipeline generates.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

SEED_Q, SEED_K, SEED_V, SEED_COND_K, SEED_COND_V = 1001, 1002, 1003, 1004, 1005
SEED_DOUT = 1006  # output gradient of the backward pass


@dataclass(frozen=True)
class Workload:
    name: str
    T: int          # latent frames, condition frames included
    H: int
    W: int
    n_cond: int     # condition latent frames (0 = text-to-video)
    heads: int
    local: int
    stride: int
    dtype: str      # "bf16" or "f32"
    cached: bool = False   # condition K/V passed separately, queries = noisy tokens
    batch: int = 1
    head_dim: int = 64
    block: int = 64

    @property
    def n_tokens(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_cond_tokens(self) -> int:
        return self.n_cond * self.H * self.W

    @property
    def n_noisy_tokens(self) -> int:
        return (self.T - self.n_cond) * self.H * self.W

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS: Dict[str, Workload] = {
    # 512 tokens, 2 heads, fp32: the small case the oracle finishes instantly.
    "tiny_f32": Workload("tiny_f32", T=4, H=8, W=16, n_cond=0, heads=2,
                         local=2, stride=4, dtype="f32"),
    # 480x832, 93 frames, image-to-video: first latent frame is the condition.
    "i2v_480p": Workload("i2v_480p", T=24, H=30, W=52, n_cond=1, heads=32,
                         local=2, stride=4, dtype="bf16"),
    # continuation: 8 cached condition frames + 24 noisy frames.
    "continuation_cached": Workload("continuation_cached", T=32, H=30, W=52, n_cond=8,
                                    heads=32, local=2, stride=4, dtype="bf16",
                                    cached=True),
    # 720x1280, 93 frames, refinement stage.
    "refine_720p": Workload("refine_720p", T=24, H=45, W=80, n_cond=0, heads=32,
                            local=1, stride=16, dtype="bf16"),
}
_SWEEP = {"dense": (0, 1), "l2s4": (2, 4), "l2s8": (2, 8), "l1s16": (1, 16),
          "l1s32": (1, 32)}
for _k, (_l, _s) in _SWEEP.items():
    WORKLOADS["sweep_" + _k] = Workload("sweep_" + _k, T=24, H=30, W=52, n_cond=0,
                                        heads=32, local=_l, stride=_s, dtype="bf16")


def get(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _randn(shape, seed: int, dtype) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    return x.to(dtype) if dtype != torch.float32 else x


def make_inputs(w: Workload, device: Optional[str] = None, seed_offset: int = 0):
    """Seeded q, k, v (and cond_k, cond_v for cached workloads), CPU tensors
    unless ``device`` is given.

    Uncached: q, k, v hold the whole sequence [B, T*H*W, heads, hd].
    Cached: q, k, v hold the noisy tokens [B, Nn, heads, hd] and cond_k,
    cond_v the condition tokens [B, Nc, heads, hd] (pre-RoPE)."""
    dt = w.torch_dtype()
    s = seed_offset
    if w.cached:
        shp = (w.batch, w.n_noisy_tokens, w.heads, w.head_dim)
        cshp = (w.batch, w.n_cond_tokens, w.heads, w.head_dim)
        out = dict(q=_randn(shp, SEED_Q + s, dt), k=_randn(shp, SEED_K + s, dt),
                   v=_randn(shp, SEED_V + s, dt),
                   cond_k=_randn(cshp, SEED_COND_K + s, dt),
                   cond_v=_randn(cshp, SEED_COND_V + s, dt))
    else:
        shp = (w.batch, w.n_tokens, w.heads, w.head_dim)
        out = dict(q=_randn(shp, SEED_Q + s, dt), k=_randn(shp, SEED_K + s, dt),
                   v=_randn(shp, SEED_V + s, dt))
    if device is not None:
        out = {k: v.to(device) for k, v in out.items()}
    return out


def make_dout(w: Workload, device: Optional[str] = None, seed_offset: int = 0) -> torch.Tensor:
    """Seeded output gradient dO [B, Nq, heads, hd] for the backward pass
    (Nq = all tokens, or the noisy ones for cached workloads), N(0,1) in the
    workload's dtype."""
    nq = w.n_noisy_tokens if w.cached else w.n_tokens
    g = _randn((w.batch, nq, w.heads, w.head_dim), SEED_DOUT + seed_offset, w.torch_dtype())
    return g.to(device) if device is not None else g
