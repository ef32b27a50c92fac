"""Seeded synthetic inputs for the spatial/temporal sparse-attention path.

This module is shared by the tests, the benchmark and the oracle's callers. It
holds the workload shapes and the random draws only -- none of the method's
arithmetic (no masks, no permutation, no attention).

Workloads (Sparse VideoGen, arXiv 2502.01776, abstract: spatial heads and
temporal heads of a video DiT's 3D full attention). The pages give no
activations, so planted-pattern inputs stand in for real DiT activations of
CogVideoX-v1.5 and HunyuanVideo, whose checkpoints are not available:

* V ~ N(0, 1).
* Q, K = 0.5 * N(0, 1) + 2 * e, with the same e added to Q and K of a token and
  independent noise per tensor. For a planted-spatial head e is drawn per frame;
  for a planted-temporal head it is drawn per in-frame grid position and shared
  by all frames.
* Text tokens (appended after the T*P video tokens) get Q, K = 0.5 * N(0, 1)
  without a planted term, V ~ N(0, 1).
* Everything is rounded to bf16 (round to nearest even) once; the same bf16
  values feed the CUDA path and the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch

HEAD_SPATIAL = 0
HEAD_TEMPORAL = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention layer's shape plus its mask widths and profiling sample."""

    name: str
    B: int
    H: int
    d: int
    T: int  # frames
    P: int  # tokens per frame (latent grid rows * cols)
    n_text: int  # global text tokens, appended after the video tokens
    spatial_band: int  # spatial mask: key frames with |df| <= spatial_band
    temporal_width: int  # temporal mask: in-frame index distance <= temporal_width
    block_q: int
    block_k: int
    n_spatial: int  # planted-spatial heads per sample (the rest are temporal)
    sample_frac: float = 0.01  # profiled query rows, as a fraction of N
    n_samples_fixed: Optional[int] = None  # overrides sample_frac when set
    seed: int = 1000
    grid: Tuple[int, int] = (0, 0)  # latent grid (rows, cols), P = rows * cols

    @property
    def N(self) -> int:
        return self.T * self.P + self.n_text

    @property
    def N_v(self) -> int:
        return self.T * self.P

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_samples(self) -> int:
        if self.n_samples_fixed is not None:
            return self.n_samples_fixed
        return max(1, int(math.floor(self.sample_frac * self.N)))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny correctness case, CogVideoX-v1.5-shaped layer,
# HunyuanVideo-shaped layer, density sweep, long-video stress case.
TINY = Workload("tiny_B1_H2_d64_T4_P64", B=1, H=2, d=64, T=4, P=64, n_text=0,
                spatial_band=1, temporal_width=4, block_q=64, block_k=64,
                n_spatial=1, n_samples_fixed=16, seed=1000, grid=(8, 8))
COGVIDEOX = Workload("cogvideox15_B1_H48_d64_T11_P4080_L226", B=1, H=48, d=64, T=11,
                     P=4080, n_text=226, spatial_band=2, temporal_width=256,
                     block_q=128, block_k=128, n_spatial=24, seed=1001, grid=(85, 48))
HUNYUAN = Workload("hunyuan_B1_H24_d128_T33_P3600_L256", B=1, H=24, d=128, T=33,
                   P=3600, n_text=256, spatial_band=2, temporal_width=384,
                   block_q=128, block_k=128, n_spatial=14, seed=1002, grid=(80, 45))
SWEEP_POINTS = [(0, 64), (1, 128), (2, 256), (4, 512), (7, 1024)]
SWEEP_BASE = Workload("sweep_B1_H24_d128_T16_P2048", B=1, H=24, d=128, T=16, P=2048,
                      n_text=0, spatial_band=0, temporal_width=64, block_q=128,
                      block_k=128, n_spatial=12, seed=1003, grid=(64, 32))
LONG = Workload("long_B2_H8_d128_T64_P3600_L256", B=2, H=8, d=128, T=64, P=3600,
                n_text=256, spatial_band=3, temporal_width=512, block_q=128,
                block_k=128, n_spatial=4, sample_frac=0.005, seed=1004, grid=(80, 45))


def sweep_workloads() -> List[Workload]:
    """The density sweep: five zipped (band, width) points."""
    return [SWEEP_BASE.replace(name=f"sweep_s{s}_w{w}", spatial_band=s, temporal_width=w)
            for s, w in SWEEP_POINTS]


WORKLOADS = {w.name: w for w in [TINY, COGVIDEOX, HUNYUAN, LONG] + sweep_workloads()}


def planted_head_kinds(wl: Workload) -> List[int]:
    """Planted pattern per head (same for every sample b).

    The first head is spatial and the second temporal when H == 2 (the tiny
    case); otherwise a seeded random permutation picks which heads are the
    n_spatial planted-spatial ones.
    """
    if wl.H == 2 and wl.n_spatial == 1:
        return [HEAD_SPATIAL, HEAD_TEMPORAL]
    g = torch.Generator().manual_seed(wl.seed * 7 + 3)
    order = torch.randperm(wl.H, generator=g).tolist()
    kinds = [HEAD_TEMPORAL] * wl.H
    for h in order[: wl.n_spatial]:
        kinds[h] = HEAD_SPATIAL
    return kinds


def _head_generator(wl: Workload, b: int, h: int, salt: int = 0) -> torch.Generator:
    return torch.Generator().manual_seed((wl.seed * 1_000_003 + b * 4099 + h * 131 + salt)
                                         & 0x7FFFFFFFFFFF)


def make_head(wl: Workload, b: int, h: int, kind: Optional[int] = None,
              planted: bool = True) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V of one (b, h) as bf16 CPU tensors [N, d] in frame-major order."""
    if kind is None:
        kind = planted_head_kinds(wl)[h]
    g = _head_generator(wl, b, h)
    N, Nv, d = wl.N, wl.N_v, wl.d
    q = torch.randn(N, d, generator=g) * 0.5
    k = torch.randn(N, d, generator=g) * 0.5
    v = torch.randn(N, d, generator=g)
    if planted and Nv > 0:
        if kind == HEAD_SPATIAL:
            e = torch.randn(wl.T, d, generator=g)
            e_tok = e.repeat_interleave(wl.P, dim=0)  # token f*P+p -> e[f]
        else:
            e = torch.randn(wl.P, d, generator=g)
            e_tok = e.repeat(wl.T, 1)  # token f*P+p -> e[p]
        q[:Nv] += 2.0 * e_tok
        k[:Nv] += 2.0 * e_tok
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_unstructured_head(wl: Workload, b: int, h: int):
    """Q, K, V ~ N(0, 1) with no planted pattern (diffuse attention)."""
    g = _head_generator(wl, b, h, salt=977)
    N, d = wl.N, wl.d
    return tuple(torch.randn(N, d, generator=g).to(torch.bfloat16) for _ in range(3))


def make_qkv(wl: Workload, out: Optional[Tuple[torch.Tensor, ...]] = None,
             planted: bool = True):
    """Q, K, V as [B, H, N, d] bf16 CPU tensors (optionally written into `out`)."""
    if out is None:
        shape = (wl.B, wl.H, wl.N, wl.d)
        out = tuple(torch.empty(shape, dtype=torch.bfloat16) for _ in range(3))
    for b in range(wl.B):
        for h in range(wl.H):
            heads = make_head(wl, b, h) if planted else make_unstructured_head(wl, b, h)
            for dst, src in zip(out, heads):
                dst[b, h].copy_(src)
    return out


def sample_rows(wl: Workload, seed_salt: int = 0) -> torch.Tensor:
    """Profiled query rows: n_samples distinct video rows, ascending, int32.

    Drawn uniformly without replacement from [0, T*P); one set serves every
    (b, h). The draw is an input to the method, so the CUDA path and the oracle
    receive the same rows.
    """
    g = torch.Generator().manual_seed(wl.seed * 17 + 5 + seed_salt)
    S = min(wl.n_samples, wl.N_v)
    rows = torch.randperm(wl.N_v, generator=g)[:S]
    return torch.sort(rows).values.to(torch.int32)


def random_labels(wl: Workload, seed_salt: int = 0) -> torch.Tensor:
    """A seeded random spatial/temporal label per (b, h), int8 [B*H]."""
    g = torch.Generator().manual_seed(wl.seed * 31 + 11 + seed_salt)
    return torch.randint(0, 2, (wl.B * wl.H,), generator=g).to(torch.int8)
