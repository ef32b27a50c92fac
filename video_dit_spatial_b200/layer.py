"""One Sparse VideoGen attention layer on the GPU: buffers plus the call sequence.

The path (arXiv 2502.01776, abstract): online profiling labels every head
spatial or temporal; temporal heads are moved to position-major order (the
layout transformation); block-sparse attention runs over each head's block
mask; temporal outputs are moved back. This class only owns device buffers
(allocated with torch) and calls the library's entry points in that order on
one stream; every step is a libsvg kernel.

`layout` chooses how the layout transformation is done:
  "explicit"  permute Q, K, V of temporal heads, attend, un-permute O (the
              default: the fastest);
  "fused"     permute K, V only; the attention kernel gathers the query rows of
              temporal heads in position-major order and stores each output row
              at its frame-major place (no Q or O copies, no un-permute pass;
              about 1 % slower, since the row gathers cost about what the
              dropped passes save);
  "gathered"  nothing is permuted: key/value rows are gathered in the kernel
              too (least memory; far slower, row gathers move fewer bytes per
              cycle than tiled loads).
"fused" and "gathered" need 128-row query blocks; they give the same bits as
"explicit".

`pv` chooses the arithmetic of the PV product: "bf16" (the default) or
"e4m3" (FP8: V quantised per (head, channel) by svg_quantize_v_e4m3, P
rounded to e4m3 inside the kernel; explicit layout, d = 128, 128-row query
blocks only; a looser tolerance than bf16).
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (Geom, SVG_MASK_DENSE, SVG_MASK_SPATIAL, SVG_MASK_TEMPORAL, svg_build_block_mask,
               svg_mask_nnz, svg_permute_qkv, svg_profile_heads, svg_profile_workspace_bytes,
               svg_quantize_v_e4m3, svg_sparse_attention, svg_sparse_attention_fp8pv,
               svg_sparse_attention_fused, svg_unpermute)


class BlockMaskCSR:
    """Device CSR of one block mask (built once per geometry)."""

    def __init__(self, geom: Geom, kind: int, device):
        self.kind = kind
        self.nnz = svg_mask_nnz(geom, kind)
        self.row_ptr = torch.empty(geom.n_qblocks + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(max(self.nnz, 1), dtype=torch.int32, device=device)

    def build(self, geom: Geom, stream=None) -> None:
        svg_build_block_mask(geom, self.kind, self.row_ptr, self.col_idx, stream=stream)


LAYOUTS = ("explicit", "fused", "gathered")


class SparseVideoGenLayer:
    def __init__(self, geom: Geom, n_samples: int, device="cuda",
                 layout: Optional[str] = None, pv: str = "bf16"):
        self.geom = geom
        if layout is None:
            layout = "explicit"
        if layout not in LAYOUTS:
            raise ValueError(f"layout must be one of {LAYOUTS}")
        if pv not in ("bf16", "e4m3"):
            raise ValueError("pv must be 'bf16' or 'e4m3'")
        if pv == "e4m3" and layout != "explicit":
            raise ValueError("the e4m3 PV product runs on the explicit layout")
        self.layout = layout
        self.pv = pv
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
        self.qp = self.kp = self.vp = self.op = None
        mk = lambda: torch.empty(shape, dtype=torch.bfloat16, device=self.device)  # noqa: E731
        if layout == "explicit":
            self.qp, self.op = mk(), mk()
        if layout in ("explicit", "fused"):
            self.kp, self.vp = mk(), mk()
        self.v8 = self.v_scale = None
        if pv == "e4m3":
            self.v8 = torch.empty(shape, dtype=torch.uint8, device=self.device)
            self.v_scale = torch.empty(B * H * d, dtype=torch.float32, device=self.device)
        self.masks_built = False

    def build_masks(self, stream=None) -> None:
        for m in self.masks.values():
            m.build(self.geom, stream)
        self.masks_built = True

    def profile(self, q, k, v, sample_idx, stream=None) -> None:
        svg_profile_heads(self.geom, q, k, v, sample_idx, self.labels, self.mse, self.workspace,
                          n_samples=self.n_samples, stream=stream)

    def attend(self, q, k, v, o, lse=None, stream=None) -> None:
        """Permute temporal heads, block-sparse attention, un-permute (labels as set).

        lse, if given, is in frame-major rows on the fused layouts and in
        each head's own layout on the explicit one.
        """
        ms, mt = self.masks[SVG_MASK_SPATIAL], self.masks[SVG_MASK_TEMPORAL]
        if self.layout != "explicit":
            if self.layout == "fused":
                svg_permute_qkv(self.geom, None, k, v, None, self.kp, self.vp, self.labels,
                                stream=stream)
            svg_sparse_attention_fused(self.geom, q, k, v, self.kp, self.vp, self.labels,
                                       ms.row_ptr, ms.col_idx, mt.row_ptr, mt.col_idx, o, lse,
                                       stream=stream)
            return
        svg_permute_qkv(self.geom, q, k, v, self.qp, self.kp, self.vp, self.labels,
                        stream=stream)
        if self.pv == "e4m3":
            svg_quantize_v_e4m3(self.geom, v, self.vp, self.labels, self.v8, self.v_scale,
                                stream=stream)
            svg_sparse_attention_fp8pv(self.geom, q, k, self.qp, self.kp, self.v8, self.v_scale,
                                       self.labels, ms.row_ptr, ms.col_idx, mt.row_ptr,
                                       mt.col_idx, o, self.op, lse, stream=stream)
        else:
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


class StreamedLayer:
    """The layer over a sequence of host-resident inputs, with copies overlapped.

    Each item is (q, k, v, sample_idx) in pinned host memory and an output
    buffer o in pinned host memory. Three CUDA streams form a pipeline over
    `depth` device buffer sets: while item i computes, the inputs of item i+1
    are copied in and the output of item i-1 is copied out. All compute of
    every item runs on one stream, so the layer's shared scratch (permuted
    tensors, labels, workspace, masks) is used by one item at a time.
    """

    def __init__(self, geom: Geom, n_samples: int, device="cuda", depth: int = 2):
        self.layer = SparseVideoGenLayer(geom, n_samples, device)
        dev = self.layer.device
        shape = (geom.B, geom.H, geom.N, geom.head_dim)
        self.depth = depth
        self.qkv = [tuple(torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3))
                    for _ in range(depth)]
        self.rows = [torch.empty(n_samples, dtype=torch.int32, device=dev) for _ in range(depth)]
        self.out = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.s_in = torch.cuda.Stream(dev)
        self.s_compute = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        mk = lambda: [torch.cuda.Event() for _ in range(depth)]  # noqa: E731
        self.ev_in, self.ev_done, self.ev_out = mk(), mk(), mk()
        self.started = [False] * depth
        with torch.cuda.stream(self.s_compute):
            self.layer.build_masks(stream=self.s_compute)

    def submit(self, i: int, q_h, k_h, v_h, rows_h, o_h) -> None:
        """Enqueues item number i (the caller numbers items 0, 1, 2, ...)."""
        b = i % self.depth
        q, k, v = self.qkv[b]
        if self.started[b]:
            self.s_in.wait_event(self.ev_done[b])  # inputs of the previous user computed
        with torch.cuda.stream(self.s_in):
            q.copy_(q_h, non_blocking=True)
            k.copy_(k_h, non_blocking=True)
            v.copy_(v_h, non_blocking=True)
            self.rows[b].copy_(rows_h, non_blocking=True)
            self.ev_in[b].record(self.s_in)
        self.s_compute.wait_event(self.ev_in[b])
        if self.started[b]:
            self.s_compute.wait_event(self.ev_out[b])  # output buffer copied out
        self.layer.forward(q, k, v, self.rows[b], self.out[b], stream=self.s_compute)
        self.ev_done[b].record(self.s_compute)
        self.s_out.wait_event(self.ev_done[b])
        with torch.cuda.stream(self.s_out):
            o_h.copy_(self.out[b], non_blocking=True)
            self.ev_out[b].record(self.s_out)
        self.started[b] = True

    def synchronize(self) -> None:
        for s in (self.s_in, self.s_compute, self.s_out):
            s.synchronize()


class SemanticSparseLayer:
    """Semantic-aware sparse attention (Sparse VideoGen 2) over one layer.

    The path (project article "Sparse-VideoGen and the sparsity hiding inside
    video diffusion attention", section "Three generations of the same idea"):
    k-means on the query and on the key vectors of every head, a stable
    cluster-sorted permutation of Q (by query cluster) and of K, V (by key
    cluster), the key clusters each query cluster keeps (top-p of the
    size-weighted centroid softmax), the tile pairs of the sorted layouts that
    hold a kept pair, block-sparse attention over them, and the output
    scattered back to the original order. This class owns the device buffers
    (allocated with torch) and calls the library in that order on one stream.
    """

    def __init__(self, B: int, H: int, N: int, d: int, Cq: int = 256, Ck: int = 256,
                 iters: int = 10, top_p: float = 0.9, block_k: int = 128, scale=None,
                 ear_tau: Optional[float] = None, device="cuda"):
        """ear_tau: None for Sparse VideoGen 2; a threshold for SVG-EAR (error-
        aware routing of skipped cluster pairs whose estimated error exceeds it,
        and centroid compensation of every key left out)."""
        from . import svg2_ear_workspace_bytes, svg2_kmeans_workspace_bytes
        self.B, self.H, self.N, self.d = B, H, N, d
        self.BH = B * H
        self.Cq, self.Ck, self.iters, self.top_p = Cq, Ck, iters, top_p
        self.block_q, self.block_k = 128, block_k
        self.scale = float(d ** -0.5 if scale is None else scale)
        dev = self.device = torch.device(device)
        BH = self.BH
        # the query and key clusterings run side by side on two streams, each
        # with its own workspace
        self.workspace = torch.empty(svg2_kmeans_workspace_bytes(BH, N, d, Cq) // 4 + 64,
                                     dtype=torch.float32, device=dev)
        self.workspace_k = torch.empty(svg2_kmeans_workspace_bytes(BH, N, d, Ck) // 4 + 64,
                                       dtype=torch.float32, device=dev)
        self._side = torch.cuda.Stream(device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        self.cq = torch.empty((BH, Cq, d), dtype=torch.float32, device=dev)
        self.ck = torch.empty((BH, Ck, d), dtype=torch.float32, device=dev)
        self.assign_q, self.assign_k = torch.empty((BH, N), **i32), torch.empty((BH, N), **i32)
        self.order_q, self.order_k = torch.empty((BH, N), **i32), torch.empty((BH, N), **i32)
        self.offsets_q = torch.empty((BH, Cq + 1), **i32)
        self.offsets_k = torch.empty((BH, Ck + 1), **i32)
        self.sel = torch.empty((BH, Cq, (Ck + 31) // 32), **i32)
        self.nqb = -(-N // self.block_q)
        self.nkb = -(-N // block_k)
        self.row_ptr = torch.empty(BH * self.nqb + 1, **i32)
        self.counts = torch.empty(BH * self.nqb, **i32)
        # every tile pair at most: the CSR never needs more
        self.col_idx = torch.empty(BH * self.nqb * self.nkb, **i32)
        shape = (self.B, self.H, N, d)
        self.qs, self.ks, self.vs, self.os = (torch.empty(shape, dtype=torch.bfloat16, device=dev)
                                              for _ in range(4))
        self.ear_tau = ear_tau
        if ear_tau is not None:
            self.vbar = torch.empty((BH, Ck, d), dtype=torch.float32, device=dev)
            self.disp = torch.empty((BH, Ck), dtype=torch.float32, device=dev)
            self.lse = torch.empty((BH, N), dtype=torch.float32, device=dev)
            self.ear_ws = torch.empty(svg2_ear_workspace_bytes(BH, d, Ck) // 4 + 64,
                                      dtype=torch.float32, device=dev)

    def plan(self, q, k, v=None, stream=None) -> None:
        """Clusters, permutations, selection and the tile CSR of q and k (and
        the value statistics of v for SVG-EAR's routing)."""
        if self.ear_tau is not None and v is None:
            raise ValueError("SVG-EAR routing needs v")
        self._v = v
        from . import svg2_build_tile_csr, svg2_kmeans, svg2_select_clusters
        BH, N, d = self.BH, self.N, self.d
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        if isinstance(main, int):
            main = torch.cuda.ExternalStream(main, device=self.device)
        # keys (and the value statistics) on the side stream, joined before the
        # selection; both start after what `main` holds so far (q, k, v written)
        side = self._side
        side.wait_stream(main)
        svg2_kmeans(BH, N, d, self.Cq, self.iters, q, self.cq, self.assign_q, self.order_q,
                    self.offsets_q, self.workspace, stream=main)
        svg2_kmeans(BH, N, d, self.Ck, self.iters, k, self.ck, self.assign_k, self.order_k,
                    self.offsets_k, self.workspace_k, stream=side)
        disp = None
        if self.ear_tau is not None:
            from . import svg2_cluster_value_stats
            svg2_cluster_value_stats(BH, N, d, self.Ck, self._v, self.order_k, self.offsets_k,
                                     self.vbar, self.disp, stream=side)
            disp = self.disp
        main.wait_stream(side)
        svg2_select_clusters(BH, d, self.Cq, self.Ck, self.scale, self.top_p, self.cq, self.ck,
                             self.offsets_k, self.sel, disp=disp, tau=self.ear_tau or 0.0,
                             stream=main)
        svg2_build_tile_csr(BH, N, self.Cq, self.Ck, self.block_q, self.block_k, self.offsets_q,
                            self.offsets_k, self.sel, self.row_ptr, self.col_idx, self.counts,
                            stream=main)

    def attend(self, q, k, v, o, lse=None, stream=None) -> None:
        """Permute, block-sparse attention over the planned tiles, un-permute."""
        from . import svg2_gather_rows, svg2_scatter_rows, svg2_sparse_attention
        BH, N, d = self.BH, self.N, self.d
        svg2_gather_rows(BH, N, d, q, self.order_q, self.qs, stream=stream)
        svg2_gather_rows(BH, N, d, k, self.order_k, self.ks, stream=stream)
        svg2_gather_rows(BH, N, d, v, self.order_k, self.vs, stream=stream)
        if self.ear_tau is None:
            svg2_sparse_attention(BH, N, d, self.block_k, self.scale, self.qs, self.ks, self.vs,
                                  self.row_ptr, self.col_idx, self.os, lse, stream=stream)
        else:
            from . import svg2_ear_compensate
            svg2_sparse_attention(BH, N, d, self.block_k, self.scale, self.qs, self.ks, self.vs,
                                  self.row_ptr, self.col_idx, self.os, self.lse, stream=stream)
            svg2_ear_compensate(BH, N, d, self.Ck, self.block_k, self.scale, self.qs, self.ck,
                                self.vbar, self.offsets_k, self.row_ptr, self.col_idx, self.os,
                                self.lse, self.ear_ws, stream=stream)
        svg2_scatter_rows(BH, N, d, self.os, self.order_q, o, stream=stream)

    def forward(self, q, k, v, o, lse=None, stream=None) -> None:
        self.plan(q, k, v, stream)
        self.attend(q, k, v, o, lse, stream)
