"""Seeded synthetic inputs for the RouteRelay routing path.

This module holds no routing arithmetic.  It only describes the workloads
(shapes, schedules, drift) and draws the chunk representations, so that the
CUDA path and the CPU oracle can be fed identical inputs.

Recipe (the same for every workload, per seed, Q and K drawn independently):
    x_0     = rownorm(N(0, 1/d))                      shape [BH, N, d]
    x_{l+1} = rownorm(x_l + sigma * N(0, I))
with rownorm the Euclidean row normalisation, fp32 throughout, drawn with
torch's seeded generator on the requested device (CPU for small cases, the
GPU for the full-size ones; the two devices give different but equally
seeded streams).  bf16 workloads round each layer's fp32 values to bf16
(round to nearest even); consumers of a bf16 workload see those bf16 values
(the oracle sees them widened to fp32, which is exact).

The pages that define the method evaluate on synthetic "persistent preferred
chunks with layer-local Gaussian drift" whose generator they do not specify;
the recipe above stands in for it.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    bh: int            # batch x heads
    n: int             # query chunks = key chunks
    d: int             # representation dim
    dtype: str         # "f32" | "bf16"
    layers: int
    sigma: float       # drift per layer
    anchor_interval: int
    k: int
    m: int             # near-miss sentinels
    r: int             # random sentinels
    causal: bool
    seed: int = 0
    gamma: float = 0.0

    @property
    def c(self) -> int:
        return self.k + self.m + self.r

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads the routing path is specified and measured on.
PR1 = Workload("pr1_bh1_n128_d64_f32", 1, 128, 64, "f32", 8, 0.01, 4, 12, 12, 4, False)
C2 = Workload("bh128_n256_d64_f32", 128, 256, 64, "f32", 32, 0.03, 8, 12, 12, 8, False)
C3 = Workload("bh128_n512_d64_f32_causal", 128, 512, 64, "f32", 32, 0.06, 8, 12, 12, 8, True)
C4 = Workload("bh64_n1024_d64_f32_causal", 64, 1024, 64, "f32", 32, 0.03, 8, 12, 12, 8, True)
C5 = Workload("bh256_n4096_d128_bf16_causal", 256, 4096, 128, "bf16", 32, 0.03, 16, 32, 32, 16, True)
ALL = [PR1, C2, C3, C4, C5]
BY_NAME = {w.name: w for w in ALL}


def low_drift(w: Workload) -> Workload:
    """Supplementary variant (not one of the five): per-vector noise norm
    sigma instead of sigma * sqrt(d), which exercises the stable-row path."""
    return w.with_(name=w.name + "_lowdrift", sigma=w.sigma / (w.d ** 0.5))


def _rownorm(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


class LayerStream:
    """Draws (Qc, Kc) layer after layer for one workload.

    ``heads`` restricts the draw to a subset of the BH units only when every
    unit has its own generator (``per_head=True``); by default one generator
    covers all BH units of a device."""

    def __init__(self, w: Workload, device="cpu", seed: int | None = None, bh: int | None = None):
        self.w = w
        self.device = torch.device(device)
        self.bh = w.bh if bh is None else bh
        s = w.seed if seed is None else seed
        self.gq = torch.Generator(device=self.device).manual_seed(2 * s + 1)
        self.gk = torch.Generator(device=self.device).manual_seed(2 * s + 2)
        self.layer = -1
        self.q = None
        self.k = None

    def _draw0(self, g):
        x = torch.randn((self.bh, self.w.n, self.w.d), generator=g, device=self.device,
                        dtype=torch.float32) * (1.0 / self.w.d) ** 0.5
        return _rownorm(x)

    def _drift(self, x, g):
        noise = torch.randn(x.shape, generator=g, device=self.device, dtype=torch.float32)
        return _rownorm(x + self.w.sigma * noise)

    def next(self):
        """Returns this layer's (q, k) as fp32 tensors [BH, N, d] holding the
        values the consumers see (bf16-rounded for bf16 workloads), plus the
        tensors in the workload's storage dtype."""
        if self.layer < 0:
            self.q = self._draw0(self.gq)
            self.k = self._draw0(self.gk)
        else:
            self.q = self._drift(self.q, self.gq)
            self.k = self._drift(self.k, self.gk)
        self.layer += 1
        if self.w.dtype == "bf16":
            qs = self.q.to(torch.bfloat16)
            ks = self.k.to(torch.bfloat16)
            return qs.float(), ks.float(), qs, ks
        return self.q, self.k, self.q, self.k


def storage_dtype(w: Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


# ---- token-level inputs of the sparse attention that consumes a route ------
@dataclass(frozen=True)
class AttentionWorkload:
    """One layer's token tensors for the attention over a route: bh heads of
    n_chunks chunks of `chunk` tokens, head dim dh, route width k."""
    name: str
    bh: int
    n_chunks: int
    chunk: int
    dh: int
    k: int
    causal: bool
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.n_chunks * self.chunk


# Four heads of the largest routing workload at token level: 4096 chunks of
# 64 tokens (256K tokens per head), head dim 128, the route width 32.
ATTN_C5 = AttentionWorkload("attn_bh4_n4096_c64_dh128_bf16_causal", 4, 4096, 64, 128, 32, True)


def attention_tokens(bh: int, n_tokens: int, dh: int, seed: int, device="cpu"):
    """q, k, v with N(0, 1) entries, rounded to bf16: [bh, n_tokens, dh] each
    (a head's logits q.k / sqrt(dh) are then about N(0, 1))."""
    g = torch.Generator(device=torch.device(device)).manual_seed(1000 + seed)
    return tuple(torch.randn((bh, n_tokens, dh), generator=g, device=device, dtype=torch.float32)
                 .to(torch.bfloat16) for _ in range(3))


def random_routes(bh: int, nq_chunks: int, nk_chunks: int, width: int, causal: bool, seed: int,
                  stride: int | None = None, pad: float = 0.0, junk: int = 0) -> torch.Tensor:
    """Routes for the attention: per query chunk i, min(width, valid) distinct
    key-chunk ids drawn uniformly from the valid ones (0..i when causal,
    else 0..nk_chunks-1), in random order, then a fraction `pad` of the
    entries replaced by -1; int32 [bh, nq_chunks, stride] on the CPU.
    Columns width..stride-1 hold `junk` (a reader must not use them)."""
    import numpy as np
    stride = width if stride is None else stride
    rng = np.random.default_rng(5000 + seed)
    out = np.full((bh, nq_chunks, stride), junk, dtype=np.int32)
    out[:, :, :width] = -1
    for h in range(bh):
        for i in range(nq_chunks):
            n_valid = min(i + 1, nk_chunks) if causal else nk_chunks
            ids = rng.choice(n_valid, size=min(width, n_valid), replace=False)
            out[h, i, :ids.size] = ids
            if pad > 0:
                drop = rng.random(width) < pad
                out[h, i, :width][drop] = -1
    return torch.from_numpy(out)
