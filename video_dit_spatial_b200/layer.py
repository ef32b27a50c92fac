"""One Sparse VideoGen attention layer on the GPU: buffers plus the call sequence.

The path (arXiv 2502.01776, abstract): online profiling labels every head
spatial or temporal; temporal heads are moved to position-major order (the
layout transformation); block-sparse attention runs over each head's block
mask; temporal outputs are moved back. This class only owns device buffers
(allocated with torch) and calls the library's entry points in that order on
one stream; every step is a libsvg kernel.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (Geom, SVG_MASK_DENSE, SVG_MASK_SPATIAL, SVG_MASK_TEMPORAL, svg_build_block_mask,
               svg_mask_nnz, svg_permute_qkv, svg_profile_heads, svg_profile_workspace_bytes,
               svg_sparse_attention, svg_unpermute)


class BlockMaskCSR:
    """Device CSR of one block mask (built once per geometry)."""

    def __init__(self, geom: Geom, kind: int, device):
        self.kind = kind
        self.nnz = svg_mask_nnz(geom, kind)
        self.row_ptr = torch.empty(geom.n_qblocks + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(max(self.nnz, 1), dtype=torch.int32, device=device)

    def build(self, geom: Geom, stream=None) -> None:
        svg_build_block_mask(geom, self.kind, self.row_ptr, self.col_idx, stream=stream)


class SparseVideoGenLayer:
    def __init__(self, geom: Geom, n_samples: int, device="cuda"):
        self.geom = geom
        self.n_samples = n_samples
        self.device = torch.device(device)
        B, H, N, d = geom.B, geom.H, geom.N, geom.head_dim
        shape = (B, H, N, d)
        self.masks = {k: BlockMaskCSR(geom, k, self.device)
                      for k in (SVG_MASK_SPATIAL, SVG_MASK_TEMPORAL)}
        self.dense_mask: Optional[BlockMaskCSR] = None
        wbytes = svg_profile_workspace_bytes(geom, n_samples)
        self.workspace = torch.empty(max(wbytes // 4, 1), dtype=torch.float32, device=self.device)
        self.labels = torch.empty(B * H, dtype=torch.int8, device=self.device)
        self.mse = torch.empty(B * H * 2, dtype=torch.float32, device=self.device)
        self.qp = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.op = torch.empty_like(self.qp)
        self.masks_built = False

    def build_masks(self, stream=None) -> None:
        for m in self.masks.values():
            m.build(self.geom, stream)
        self.masks_built = True

    def profile(self, q, k, v, sample_idx, stream=None) -> None:
        svg_profile_heads(self.geom, q, k, v, sample_idx, self.labels, self.mse, self.workspace,
                          n_samples=self.n_samples, stream=stream)

    def attend(self, q, k, v, o, lse=None, stream=None) -> None:
        """Permute temporal heads, block-sparse attention, un-permute (labels as set)."""
        ms, mt = self.masks[SVG_MASK_SPATIAL], self.masks[SVG_MASK_TEMPORAL]
        svg_permute_qkv(self.geom, q, k, v, self.qp, self.kp, self.vp, self.labels,
                        stream=stream)
        svg_sparse_attention(self.geom, q, k, v, self.qp, self.kp, self.vp, self.labels,
                             ms.row_ptr, ms.col_idx, mt.row_ptr, mt.col_idx, o, self.op, lse,
                             stream=stream)
        svg_unpermute(self.geom, self.op, o, self.labels, stream=stream)

    def forward(self, q, k, v, sample_idx, o, lse=None, rebuild_masks: bool = False,
                stream=None) -> None:
        """The whole path: profile -> (masks) -> permute -> attention -> un-permute."""
        if rebuild_masks or not self.masks_built:
            self.build_masks(stream)
        self.profile(q, k, v, sample_idx, stream)
        self.attend(q, k, v, o, lse, stream)

    def dense(self, q, k, v, o, lse=None, stream=None) -> None:
        """The same attention kernel over the all-blocks mask (the dense baseline)."""
        if self.dense_mask is None:
            self.dense_mask = BlockMaskCSR(self.geom, SVG_MASK_DENSE, self.device)
            self.dense_mask.build(self.geom, stream)
        dm = self.dense_mask
        svg_sparse_attention(self.geom, q, k, v, None, None, None, None, dm.row_ptr, dm.col_idx,
                             None, None, o, None, lse, stream=stream)
