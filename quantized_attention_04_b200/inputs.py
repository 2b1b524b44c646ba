"""Seeded synthetic Q/K/V generators shared by the tests, the bench and smoke().

This module holds no part of the attention method's arithmetic: it only draws
random tensors.  Both the CUDA path and the CPU oracle consume the exact same
bytes produced here.

Recipe (one generator per call, seed = 1000 + config index unless given):
  * numpy PCG64 ``default_rng(seed)``;
  * per tensor, in the order Q, K, V: first the per-(head, channel) offsets
    ``N(0, offset_std^2)`` of shape [H, d] (shared by every batch and token),
    then, for K with outliers, the outlier channel indices (``n`` distinct
    channels per head), then the noise ``N(0, 1)`` of shape [B, H, N, d] as
    float32;
  * noise of the outlier channels is multiplied by ``outlier_scale`` first,
    the offsets are added after;
  * the float32 result is rounded (RNE) to the config's dtype by torch.

The configurations mirror the workloads the SageAttention2 pages motivate:
LLM prefill (causal, bf16, d=128), video-DiT-like long non-causal sequences
(d=64) and small cases; channel offsets and a few scaled outlier channels make
the smoothing steps matter.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Dist:
    offset_std: float = 0.0        # std of the per-(head, channel) offset
    outliers: int = 0              # number of outlier channels per head
    outlier_scale: float = 1.0     # factor applied to their noise


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: str                     # "fp16" | "bf16"
    q: Dist
    k: Dist
    v: Dist
    index: int = 0                 # position in the config list (seed = 1000 + index)

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "fp16" else torch.bfloat16

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def ops(self) -> float:
        """Algorithmic operation count 4*B*H*N^2*d, halved for causal."""
        o = 4.0 * self.B * self.H * float(self.N) ** 2 * self.d
        return o / 2 if self.causal else o

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


_LLM = dict(q=Dist(2.0), k=Dist(2.0, outliers=4, outlier_scale=20.0), v=Dist(2.0))

CONFIGS = {
    "C1": Config("C1", 1, 2, 256, 64, False, "fp16",
                 q=Dist(), k=Dist(3.0), v=Dist(), index=0),
    "C2": Config("C2", 2, 8, 2048, 128, True, "fp16",
                 q=Dist(1.0), k=Dist(5.0), v=Dist(), index=1),
    "C3": Config("C3", 4, 32, 8192, 128, True, "bf16", index=2, **_LLM),
    "C4": Config("C4", 1, 24, 17776, 64, False, "fp16",
                 q=Dist(4.0), k=Dist(4.0), v=Dist(1.0), index=3),
    "C5": Config("C5", 1, 32, 32768, 128, True, "bf16", index=4, **_LLM),
}


def sweep_config(N: int, d: int) -> Config:
    """Roofline-curve point: B=1, H=32, causal bf16, LLM-like distributions."""
    return Config(f"S_N{N}_d{d}", 1, 32, N, d, True, "bf16", index=10, **_LLM)


def _draw(rng: np.random.Generator, B, H, N, d, dist: Dist, heads=None) -> np.ndarray:
    off = rng.normal(0.0, dist.offset_std, size=(H, d)).astype(np.float32) \
        if dist.offset_std > 0 else np.zeros((H, d), np.float32)
    chans = None
    if dist.outliers:
        chans = np.stack([rng.choice(d, dist.outliers, replace=False) for _ in range(H)])
    x = rng.standard_normal(size=(B, H, N, d), dtype=np.float32)
    if chans is not None:
        for h in range(H):
            x[:, h, :, chans[h]] *= np.float32(dist.outlier_scale)
    x += off[None, :, None, :]
    return x


def make_qkv(cfg: Config, seed: int | None = None):
    """Return (q, k, v): contiguous CPU tensors [B, H, N, d] in cfg's dtype."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    out = []
    for dist in (cfg.q, cfg.k, cfg.v):
        x = _draw(rng, cfg.B, cfg.H, cfg.N, cfg.d, dist)
        out.append(torch.from_numpy(x).to(cfg.torch_dtype).contiguous())
        del x
    return tuple(out)
