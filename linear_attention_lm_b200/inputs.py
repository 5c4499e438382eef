"""Seeded synthetic inputs for the Based attention path.

This module holds only random-number generation and the synthetic input
recipe (i.i.d. Gaussians, or a Gaussian activation ``x`` pushed through
random Linear projections).  It contains none of the attention arithmetic,
and it is the only module that both the CUDA path's callers and the fp64
oracle's callers share.

Recipe (numpy PCG64; seed = 1000 * workload id + tensor id, plus
16 * step for decode steps):

* iid workloads: q, k = qk_scale * N(0, 1); v = N(0, 1).
* projected workloads (layer shapes of the 360M / 1.3B Based models):
  x ~ N(0, 1) of shape [B, L, d_model]; each of the six projections
  (linear-attention q, k, v; window q, k, v) is a bias-free Linear with
  weight ~ N(0, 0.02^2) of shape [heads * head_dim, d_model]; the result is
  reshaped to [B, L, heads, head_dim] and transposed to [B, heads, L, head_dim].
* decode steps: q, k, v ~ N(0, 1) per step (no extra scaling).

Values are produced in float32 and rounded once to the workload's dtype
(bf16 round-to-nearest-even via torch).  The projections run in float32 on
the requested device; the rounded tensors are what both sides consume.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int            # seed namespace
    B: int
    H: int              # linear-attention heads
    L: int              # prefill length
    d: int              # q/k feature dim (Taylor map input)
    dv: int             # v head dim of the linear attention
    Hw: int             # window-attention heads
    dh: int             # window-attention head dim
    window: int
    dtype: str          # "f32" | "bf16"
    eps: float = 1e-6
    qk_scale: float = 1.0
    d_model: int = 0    # > 0: q/k/v come from random projections of x
    w_std: float = 0.02
    steps: int = 0      # decode steps after the prefill

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, B=1, H=2, L=256, d=16, dv=64, Hw=2, dh=64,
                          window=64, dtype="f32", qk_scale=0.25),
    "layer_360m": Workload("layer_360m", 2, B=8, H=16, L=2048, d=16, dv=64, Hw=16, dh=64,
                           window=64, dtype="bf16", d_model=1024),
    "layer_1b3": Workload("layer_1b3", 3, B=8, H=16, L=2048, d=16, dv=128, Hw=16, dh=128,
                          window=64, dtype="bf16", d_model=2048),
    "long_16k": Workload("long_16k", 4, B=1, H=16, L=16384, d=16, dv=64, Hw=16, dh=64,
                         window=64, dtype="bf16", qk_scale=0.25),
    "decode_b128": Workload("decode_b128", 5, B=128, H=16, L=512, d=16, dv=64, Hw=16, dh=64,
                            window=64, dtype="bf16", steps=1024),
}


def _normal(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    a = g.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def _round(a: np.ndarray, w: Workload, device) -> torch.Tensor:
    return torch.from_numpy(a).to(device=device).to(w.torch_dtype).contiguous()


def prefill_inputs(w: Workload, device="cpu") -> dict:
    """q, k [B,H,L,d]; v [B,H,L,dv]; wq, wk, wv [B,Hw,L,dh] in w's dtype."""
    B, L = w.B, w.L
    base = 1000 * w.wid
    if w.d_model <= 0:
        return {
            "q": _round(_normal(base + 1, (B, w.H, L, w.d), w.qk_scale), w, device),
            "k": _round(_normal(base + 2, (B, w.H, L, w.d), w.qk_scale), w, device),
            "v": _round(_normal(base + 3, (B, w.H, L, w.dv)), w, device),
            "wq": _round(_normal(base + 4, (B, w.Hw, L, w.dh), w.qk_scale), w, device),
            "wk": _round(_normal(base + 5, (B, w.Hw, L, w.dh), w.qk_scale), w, device),
            "wv": _round(_normal(base + 6, (B, w.Hw, L, w.dh)), w, device),
        }
    x = torch.from_numpy(_normal(base + 0, (B, L, w.d_model))).to(device)
    out = {}
    specs = [("q", w.H, w.d, 1), ("k", w.H, w.d, 2), ("v", w.H, w.dv, 3),
             ("wq", w.Hw, w.dh, 4), ("wk", w.Hw, w.dh, 5), ("wv", w.Hw, w.dh, 6)]
    for name, heads, hd, tid in specs:
        W = torch.from_numpy(_normal(base + 10 + tid, (heads * hd, w.d_model), w.w_std)).to(device)
        y = (x @ W.t()).view(B, L, heads, hd).transpose(1, 2)
        out[name] = y.to(w.torch_dtype).contiguous()
    return out


def decode_step_inputs(w: Workload, step: int, device="cpu") -> dict:
    """Fresh per-step q, k [B,H,d]; v [B,H,dv]; wq, wk, wv [B,Hw,dh]."""
    base = 1000 * w.wid + 100 + 16 * step
    B = w.B
    return {
        "q": _round(_normal(base + 1, (B, w.H, w.d)), w, device),
        "k": _round(_normal(base + 2, (B, w.H, w.d)), w, device),
        "v": _round(_normal(base + 3, (B, w.H, w.dv)), w, device),
        "wq": _round(_normal(base + 4, (B, w.Hw, w.dh)), w, device),
        "wk": _round(_normal(base + 5, (B, w.Hw, w.dh)), w, device),
        "wv": _round(_normal(base + 6, (B, w.Hw, w.dh)), w, device),
    }


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a float32/bf16 tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
