"""Python binding of libsvg, the sm_100a Sparse VideoGen sparse-attention library.

Argument marshalling only: every function here forwards to the C entry point of
the same name declared in include/svg.h (through ctypes) and raises SvgError
when it returns a non-OK status. Tensors are passed as torch tensors (their
data pointer is used), plain integer device addresses or None. All compute runs
in the library's CUDA kernels; there is no fallback. The shared library is
loaded on first use and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvg.so")

SVG_OK = 0
SVG_ERR_INVALID_ARG = 1
SVG_ERR_UNSUPPORTED = 2
SVG_ERR_CAPACITY = 3
SVG_ERR_CUDA = 4
SVG_ERR_DEVICE_TIMEOUT = 5

SVG_HEAD_SPATIAL = 0
SVG_HEAD_TEMPORAL = 1
SVG_MASK_SPATIAL = 0
SVG_MASK_TEMPORAL = 1
SVG_MASK_DENSE = 2

STATUS_NAMES = {0: "SVG_OK", 1: "SVG_ERR_INVALID_ARG", 2: "SVG_ERR_UNSUPPORTED",
                3: "SVG_ERR_CAPACITY", 4: "SVG_ERR_CUDA", 5: "SVG_ERR_DEVICE_TIMEOUT"}

EXPORTED = [
    "svg_mask_nnz", "svg_build_block_mask", "svg_profile_workspace_bytes",
    "svg_profile_heads", "svg_profile_heads_noalloc", "svg_permute", "svg_unpermute", "svg_permute_qkv",
    "svg_sparse_attention", "svg_sparse_attention_fused", "svg_quantize_v_e4m3",
    "svg_sparse_attention_fp8pv", "svg_get_device_status", "svg_selftest_wait_timeout",
    "svg2_kmeans_workspace_bytes", "svg2_kmeans", "svg2_kmeans_step", "svg2_select_clusters",
    "svg2_build_tile_csr", "svg2_gather_rows", "svg2_scatter_rows", "svg2_sparse_attention",
    "svg2_cluster_value_stats", "svg2_ear_workspace_bytes", "svg2_ear_compensate",
    "svg_status_string", "svg_version",
]


class SvgError(RuntimeError):
    def __init__(self, func: str, status: int):
        super().__init__(f"{func} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Geom(ctypes.Structure):
    """svg_geom: geometry of one attention layer."""

    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
                ("P", ctypes.c_int32), ("n_text", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_q", ctypes.c_int32),
                ("block_k", ctypes.c_int32), ("spatial_band", ctypes.c_int32),
                ("temporal_width", ctypes.c_int32), ("scale", ctypes.c_float)]

    @property
    def N(self) -> int:
        return self.T * self.P + self.n_text

    @property
    def n_qblocks(self) -> int:
        return -(-self.N // self.block_q)

    @property
    def n_kblocks(self) -> int:
        return -(-self.N // self.block_k)

    @classmethod
    def from_workload(cls, wl) -> "Geom":
        return cls(wl.B, wl.H, wl.T, wl.P, wl.n_text, wl.d, wl.block_q, wl.block_k,
                   wl.spatial_band, wl.temporal_width, wl.scale)


_lib: Optional[ctypes.CDLL] = None

_c_geom_p = ctypes.POINTER(Geom)
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


def load() -> ctypes.CDLL:
    """Loads libsvg.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OSError(f"libsvg.so not found at {LIB_PATH}; run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "svg_mask_nnz": [_c_geom_p, _i32, ctypes.POINTER(_i64)],
        "svg_build_block_mask": [_c_geom_p, _i32, _vp, _vp, _i64, _vp],
        "svg_profile_workspace_bytes": [_c_geom_p, _i32, ctypes.POINTER(_sz)],
        "svg_profile_heads": [_c_geom_p, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp],
        "svg_profile_heads_noalloc": [_c_geom_p, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp],
        "svg_permute": [_c_geom_p, _vp, _vp, _vp, _vp],
        "svg_unpermute": [_c_geom_p, _vp, _vp, _vp, _vp],
        "svg_permute_qkv": [_c_geom_p, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
        "svg_sparse_attention": [_c_geom_p] + [_vp] * 15,
        "svg_sparse_attention_fused": [_c_geom_p] + [_vp] * 13,
        "svg_quantize_v_e4m3": [_c_geom_p] + [_vp] * 6,
        "svg_sparse_attention_fp8pv": [_c_geom_p] + [_vp] * 15,
        "svg_get_device_status": [_vp, ctypes.POINTER(_i32)],
        "svg_selftest_wait_timeout": [_i64, _vp],
        "svg2_kmeans_workspace_bytes": [_i32, _i32, _i32, _i32, ctypes.POINTER(_sz)],
        "svg2_kmeans": [_i32, _i32, _i32, _i32, _i32] + [_vp] * 6 + [_sz, _vp],
        "svg2_kmeans_step": [_i32, _i32, _i32, _i32] + [_vp] * 7 + [_sz, _vp],
        "svg2_select_clusters": [_i32, _i32, _i32, _i32, ctypes.c_float, ctypes.c_float] +
                                [_vp] * 4 + [ctypes.c_float, _vp, _vp],
        "svg2_cluster_value_stats": [_i32] * 4 + [_vp] * 6,
        "svg2_ear_workspace_bytes": [_i32, _i32, _i32, ctypes.POINTER(_sz)],
        "svg2_ear_compensate": [_i32] * 5 + [ctypes.c_float] + [_vp] * 9 + [_sz, _vp],
        "svg2_build_tile_csr": [_i32] * 6 + [_vp] * 5 + [_i64, _vp, _vp],
        "svg2_gather_rows": [_i32, _i32, _i32, _vp, _vp, _vp, _vp],
        "svg2_scatter_rows": [_i32, _i32, _i32, _vp, _vp, _vp, _vp],
        "svg2_sparse_attention": [_i32, _i32, _i32, _i32, ctypes.c_float] + [_vp] * 8,
        "svg_status_string": [_i32],
        "svg_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "svg_status_string" else ctypes.c_int32
    _lib = lib
    return lib


def _ptr(x) -> Optional[int]:
    """Device address of a buffer argument: None, a plain integer address, or a
    tensor. A tensor must live on a CUDA device and be contiguous: the kernels
    read dense row-major buffers, and a host address would fault on the device."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError(f"libsvg takes device buffers, got a tensor on {x.device}")
    if not x.is_contiguous():
        raise ValueError("libsvg takes contiguous buffers, got a strided view")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name: str, status: int) -> None:
    if status != SVG_OK:
        raise SvgError(name, status)


def svg_status_string(status: int) -> str:
    return load().svg_status_string(status).decode()


def svg_version() -> int:
    return load().svg_version()


def svg_mask_nnz(geom: Geom, kind: int) -> int:
    out = _i64(0)
    _check("svg_mask_nnz", load().svg_mask_nnz(ctypes.byref(geom), kind, ctypes.byref(out)))
    return out.value


def svg_build_block_mask(geom: Geom, kind: int, row_ptr, col_idx, col_capacity=None,
                         stream=None) -> None:
    cap = col_idx.numel() if col_capacity is None else col_capacity
    _check("svg_build_block_mask", load().svg_build_block_mask(
        ctypes.byref(geom), kind, _ptr(row_ptr), _ptr(col_idx), cap, _stream(stream)))


def svg_profile_workspace_bytes(geom: Geom, n_samples: int) -> int:
    out = _sz(0)
    _check("svg_profile_workspace_bytes", load().svg_profile_workspace_bytes(
        ctypes.byref(geom), n_samples, ctypes.byref(out)))
    return out.value


def svg_profile_heads(geom: Geom, q, k, v, sample_idx, labels, mse=None, workspace=None,
                      workspace_bytes=None, n_samples=None, stream=None) -> None:
    n = sample_idx.numel() if n_samples is None else n_samples
    wb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("svg_profile_heads", load().svg_profile_heads(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(sample_idx), n, _ptr(labels),
        _ptr(mse), _ptr(workspace), wb, _stream(stream)))


def svg_profile_heads_noalloc(geom: Geom, q, k, v, sample_idx, labels, mse=None,
                              n_samples=None, stream=None) -> None:
    """svg_profile_heads with the library's fixed internal scratch (no workspace)."""
    n = sample_idx.numel() if n_samples is None else n_samples
    _check("svg_profile_heads_noalloc", load().svg_profile_heads_noalloc(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(sample_idx), n, _ptr(labels),
        _ptr(mse), _stream(stream)))


def svg_permute(geom: Geom, inp, out, labels=None, stream=None) -> None:
    _check("svg_permute", load().svg_permute(ctypes.byref(geom), _ptr(inp), _ptr(out),
                                             _ptr(labels), _stream(stream)))


def svg_unpermute(geom: Geom, inp, out, labels=None, stream=None) -> None:
    _check("svg_unpermute", load().svg_unpermute(ctypes.byref(geom), _ptr(inp), _ptr(out),
                                                 _ptr(labels), _stream(stream)))


def svg_permute_qkv(geom: Geom, q, k, v, qp, kp, vp, labels=None, stream=None) -> None:
    _check("svg_permute_qkv", load().svg_permute_qkv(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp),
        _ptr(labels), _stream(stream)))


def svg_sparse_attention(geom: Geom, q, k, v, qp, kp, vp, labels, row_ptr_s, col_idx_s,
                         row_ptr_t, col_idx_t, o, op, lse=None, stream=None) -> None:
    _check("svg_sparse_attention", load().svg_sparse_attention(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(qp), _ptr(kp), _ptr(vp),
        _ptr(labels), _ptr(row_ptr_s), _ptr(col_idx_s), _ptr(row_ptr_t), _ptr(col_idx_t),
        _ptr(o), _ptr(op), _ptr(lse), _stream(stream)))


def svg_sparse_attention_fused(geom: Geom, q, k, v, kp, vp, labels, row_ptr_s, col_idx_s,
                               row_ptr_t, col_idx_t, o, lse=None, stream=None) -> None:
    _check("svg_sparse_attention_fused", load().svg_sparse_attention_fused(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp), _ptr(labels),
        _ptr(row_ptr_s),
        _ptr(col_idx_s), _ptr(row_ptr_t), _ptr(col_idx_t), _ptr(o), _ptr(lse),
        _stream(stream)))


def svg_quantize_v_e4m3(geom: Geom, v, vp, labels, v8, v_scale, stream=None) -> None:
    _check("svg_quantize_v_e4m3", load().svg_quantize_v_e4m3(
        ctypes.byref(geom), _ptr(v), _ptr(vp), _ptr(labels), _ptr(v8), _ptr(v_scale),
        _stream(stream)))


def svg_sparse_attention_fp8pv(geom: Geom, q, k, qp, kp, v8, v_scale, labels, row_ptr_s,
                               col_idx_s, row_ptr_t, col_idx_t, o, op, lse=None,
                               stream=None) -> None:
    _check("svg_sparse_attention_fp8pv", load().svg_sparse_attention_fp8pv(
        ctypes.byref(geom), _ptr(q), _ptr(k), _ptr(qp), _ptr(kp), _ptr(v8), _ptr(v_scale),
        _ptr(labels), _ptr(row_ptr_s), _ptr(col_idx_s), _ptr(row_ptr_t), _ptr(col_idx_t),
        _ptr(o), _ptr(op), _ptr(lse), _stream(stream)))


def svg_get_device_status(stream=None):
    """(status, bits): synchronises the stream and reads/clears the device status bits."""
    bits = _i32(0)
    st = load().svg_get_device_status(_stream(stream), ctypes.byref(bits))
    return st, bits.value


def svg_selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    _check("svg_selftest_wait_timeout",
           load().svg_selftest_wait_timeout(limit_cycles, _stream(stream)))


# ---------------------------------------------------------------------------
# semantic-aware permutation (Sparse VideoGen 2)
# ---------------------------------------------------------------------------
def svg2_kmeans_workspace_bytes(BH: int, N: int, d: int, C: int) -> int:
    out = _sz(0)
    _check("svg2_kmeans_workspace_bytes",
           load().svg2_kmeans_workspace_bytes(BH, N, d, C, ctypes.byref(out)))
    return out.value


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def svg2_kmeans(BH, N, d, C, iters, x, centroids, assign, order, offsets, workspace,
                stream=None) -> None:
    _check("svg2_kmeans", load().svg2_kmeans(
        BH, N, d, C, iters, _ptr(x), _ptr(centroids), _ptr(assign), _ptr(order), _ptr(offsets),
        _ptr(workspace), _nbytes(workspace), _stream(stream)))


def svg2_kmeans_step(BH, N, d, C, x, centroids_in, centroids_out, assign, order, offsets,
                     workspace, stream=None) -> None:
    _check("svg2_kmeans_step", load().svg2_kmeans_step(
        BH, N, d, C, _ptr(x), _ptr(centroids_in), _ptr(centroids_out), _ptr(assign), _ptr(order),
        _ptr(offsets), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def svg2_select_clusters(BH, d, Cq, Ck, scale, top_p, cq, ck, offsets_k, sel, disp=None,
                         tau=0.0, stream=None) -> None:
    _check("svg2_select_clusters", load().svg2_select_clusters(
        BH, d, Cq, Ck, scale, top_p, _ptr(cq), _ptr(ck), _ptr(offsets_k), _ptr(disp), tau,
        _ptr(sel), _stream(stream)))


def svg2_cluster_value_stats(BH, N, d, Ck, v, order_k, offsets_k, vbar, disp,
                             stream=None) -> None:
    _check("svg2_cluster_value_stats", load().svg2_cluster_value_stats(
        BH, N, d, Ck, _ptr(v), _ptr(order_k), _ptr(offsets_k), _ptr(vbar), _ptr(disp),
        _stream(stream)))


def svg2_ear_workspace_bytes(BH, d, Ck) -> int:
    out = _sz(0)
    _check("svg2_ear_workspace_bytes", load().svg2_ear_workspace_bytes(BH, d, Ck,
                                                                       ctypes.byref(out)))
    return out.value


def svg2_ear_compensate(BH, N, d, Ck, block_k, scale, qs, kbar, vbar, offsets_k, row_ptr,
                        col_idx, os, lse, workspace, stream=None) -> None:
    _check("svg2_ear_compensate", load().svg2_ear_compensate(
        BH, N, d, Ck, block_k, scale, _ptr(qs), _ptr(kbar), _ptr(vbar), _ptr(offsets_k),
        _ptr(row_ptr), _ptr(col_idx), _ptr(os), _ptr(lse), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))


def svg2_build_tile_csr(BH, N, Cq, Ck, block_q, block_k, offsets_q, offsets_k, sel, row_ptr,
                        col_idx, counts, col_capacity=None, stream=None) -> None:
    cap = col_idx.numel() if col_capacity is None else col_capacity
    _check("svg2_build_tile_csr", load().svg2_build_tile_csr(
        BH, N, Cq, Ck, block_q, block_k, _ptr(offsets_q), _ptr(offsets_k), _ptr(sel),
        _ptr(row_ptr), _ptr(col_idx), cap, _ptr(counts), _stream(stream)))


def svg2_gather_rows(BH, N, d, x, order, y, stream=None) -> None:
    _check("svg2_gather_rows", load().svg2_gather_rows(BH, N, d, _ptr(x), _ptr(order), _ptr(y),
                                                       _stream(stream)))


def svg2_scatter_rows(BH, N, d, y_sorted, order, y, stream=None) -> None:
    _check("svg2_scatter_rows", load().svg2_scatter_rows(BH, N, d, _ptr(y_sorted), _ptr(order),
                                                         _ptr(y), _stream(stream)))


def svg2_sparse_attention(BH, N, d, block_k, scale, qs, ks, vs, row_ptr, col_idx, os,
                          lse=None, stream=None) -> None:
    _check("svg2_sparse_attention", load().svg2_sparse_attention(
        BH, N, d, block_k, scale, _ptr(qs), _ptr(ks), _ptr(vs), _ptr(row_ptr), _ptr(col_idx),
        _ptr(os), _ptr(lse), _stream(stream)))
