"""Plain fp64 CPU oracle of Sparse VideoGen (SVG 1) spatial/temporal sparse attention.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The library never calls it
and shares no code with it.

Source: "Sparse VideoGen: Accelerating Video Diffusion Transformers with
Spatial-Temporal Sparsity" (arXiv 2502.01776), abstract. Attention heads of a
video DiT's 3D full attention fall into two groups: spatial heads, whose output
is dominated by tokens of the query's own (and nearby) frames, and temporal
heads, dominated by tokens at the same in-frame position across frames. An
online profiling strategy predicts each head's type; a layout transformation
makes the temporal pattern contiguous; customised kernels compute the sparse
attention. The project article "Sparse-VideoGen and the sparsity hiding inside
video diffusion attention" (section "Three generations of the same idea")
restates the same pieces and mentions block-sparse attention.

The pages leave the exact rules open; the readings this module takes are:

* token (f, p) of a video sits at index f*P + p in frame-major order; text
  tokens follow the T*P video tokens and are global (attend to and are attended
  by every token);
* spatial mask:  |f(i) - f(j)| <= s;  temporal mask: |p(i) - p(j)| <= w
  (in-frame index distance, any frame); both in frame-major indices;
* position-major order puts video token (f, p) at p*T + f (text unchanged);
* sparse attention is block-granular: a (query block, key block) pair is
  computed in full iff some token pair inside it is allowed by the head's mask
  in the head's layout;
* profiling: full, spatial-masked and temporal-masked attention on the sampled
  rows; MSE over rows x channels against the full output; the head is temporal
  iff MSE_temporal < MSE_spatial (a tie is spatial);
* a query row with no allowed key outputs zeros (log-sum-exp -inf).

Everything is fp64 on the exact bf16 input values; matmul, exp and sums are
numpy library primitives. Rows are processed in chunks only to bound memory;
each row's arithmetic is the plain definition.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence, Tuple

import numpy as np

MASK_SPATIAL = 0
MASK_TEMPORAL = 1
MASK_DENSE = 2
HEAD_SPATIAL = 0
HEAD_TEMPORAL = 1

_ROW_CHUNK = 128


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
def from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Exact float64 values of raw bf16 bit patterns (uint16 / int16 array)."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); uint16 bit patterns."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    out[nan] = np.uint16(0x7FC0)
    return out


# ---------------------------------------------------------------------------
# geometry, masks and the layout transformation
# ---------------------------------------------------------------------------
def seq_len(T: int, P: int, n_text: int) -> int:
    return T * P + n_text


def frame_of(i, P: int):
    """Frame of frame-major video index i."""
    return np.asarray(i) // P


def pos_of(i, P: int):
    """In-frame position of frame-major video index i."""
    return np.asarray(i) % P


def spatial_allowed(i, j, T: int, P: int, n_text: int, s: int) -> np.ndarray:
    """Token-level spatial mask M_S(i, j), frame-major indices (broadcasting).

    Spatial heads: keys of the query's frame and of frames within s of it
    (abstract: "spatially-related tokens within each frame"); text is global.
    """
    i = np.asarray(i)
    j = np.asarray(j)
    Nv = T * P
    text = (i >= Nv) | (j >= Nv)
    return text | (np.abs(i // P - j // P) <= s)


def temporal_allowed(i, j, T: int, P: int, n_text: int, w: int) -> np.ndarray:
    """Token-level temporal mask M_T(i, j), frame-major indices (broadcasting).

    Temporal heads: keys at the same or a nearby in-frame position in any frame
    (abstract: "temporally-related tokens across different frames").
    """
    i = np.asarray(i)
    j = np.asarray(j)
    Nv = T * P
    text = (i >= Nv) | (j >= Nv)
    return text | (np.abs(i % P - j % P) <= w)


def permutation(T: int, P: int, n_text: int) -> np.ndarray:
    """pi: frame-major index -> position-major index. pi(f*P+p) = p*T+f; text fixed."""
    N = seq_len(T, P, n_text)
    pi = np.arange(N, dtype=np.int64)
    for f in range(T):
        for p in range(P):
            pi[f * P + p] = p * T + f
    return pi


def inverse_permutation(pi: np.ndarray) -> np.ndarray:
    inv = np.empty_like(pi)
    inv[pi] = np.arange(pi.shape[0], dtype=pi.dtype)
    return inv


def permute(x: np.ndarray, T: int, P: int, n_text: int) -> np.ndarray:
    """Frame-major -> position-major along axis -2: out[pi(i)] = x[i]."""
    pi = permutation(T, P, n_text)
    out = np.empty_like(x)
    out[..., pi, :] = x
    return out


def unpermute(y: np.ndarray, T: int, P: int, n_text: int) -> np.ndarray:
    """Position-major -> frame-major along axis -2: out[i] = y[pi(i)]."""
    pi = permutation(T, P, n_text)
    return y[..., pi, :].copy()


def layout_to_frame_major(kind: int, idx, T: int, P: int, n_text: int):
    """Frame-major index of the token at position idx of the pattern's layout."""
    idx = np.asarray(idx)
    if kind != MASK_TEMPORAL:
        return idx
    Nv = T * P
    p = idx // T
    f = idx % T
    return np.where(idx < Nv, f * P + p, idx)


def layout_allowed(kind: int, a, b, T: int, P: int, n_text: int, s: int, w: int):
    """Token mask of pattern `kind` in that pattern's own layout.

    SPATIAL lives in frame-major order, TEMPORAL in position-major order
    (M_T^pi(pi(i), pi(j)) = M_T(i, j)), DENSE is all ones.
    """
    a = np.asarray(a)
    b = np.asarray(b)
    if kind == MASK_DENSE:
        return np.ones(np.broadcast(a, b).shape, dtype=bool)
    if kind == MASK_SPATIAL:
        return spatial_allowed(a, b, T, P, n_text, s)
    ia = layout_to_frame_major(MASK_TEMPORAL, a, T, P, n_text)
    ib = layout_to_frame_major(MASK_TEMPORAL, b, T, P, n_text)
    return temporal_allowed(ia, ib, T, P, n_text, w)


def n_blocks(N: int, block: int) -> int:
    return (N + block - 1) // block


def block_mask_rows(kind: int, rows: Sequence[int], T: int, P: int, n_text: int, s: int,
                    w: int, block_q: int, block_k: int) -> np.ndarray:
    """Block mask rows by brute force: BM[r][c] = OR of the token mask over the block pair.

    Returns bool [len(rows), n_key_blocks].
    """
    N = seq_len(T, P, n_text)
    nkb = n_blocks(N, block_k)
    cols = np.arange(N)
    out = np.zeros((len(rows), nkb), dtype=bool)
    for n, r in enumerate(rows):
        ti = np.arange(r * block_q, min(N, (r + 1) * block_q))
        if ti.size == 0:
            continue
        allowed = layout_allowed(kind, ti[:, None], cols[None, :], T, P, n_text, s, w)
        any_key = allowed.any(axis=0)  # OR over the block's query rows
        padded = np.zeros(nkb * block_k, dtype=bool)
        padded[:N] = any_key
        out[n] = padded.reshape(nkb, block_k).any(axis=1)  # OR over each key block
    return out


def block_mask(kind: int, T: int, P: int, n_text: int, s: int, w: int, block_q: int,
               block_k: int) -> np.ndarray:
    """Full block mask (bool [nQB, nKB]) by brute force over token pairs."""
    N = seq_len(T, P, n_text)
    return block_mask_rows(kind, range(n_blocks(N, block_q)), T, P, n_text, s, w, block_q,
                           block_k)


def to_csr(bm: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """CSR of a dense bool block mask: row_ptr[nQB+1], col_idx ascending per row (int32)."""
    counts = bm.sum(axis=1)
    row_ptr = np.zeros(bm.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([np.nonzero(bm[r])[0] for r in range(bm.shape[0])]
                             ) if bm.shape[0] else np.zeros(0)
    return row_ptr.astype(np.int32), np.asarray(col_idx, dtype=np.int32)


def from_csr(row_ptr: np.ndarray, col_idx: np.ndarray, n_cols: int) -> np.ndarray:
    nr = len(row_ptr) - 1
    bm = np.zeros((nr, n_cols), dtype=bool)
    for r in range(nr):
        bm[r, col_idx[row_ptr[r]:row_ptr[r + 1]]] = True
    return bm


# ---------------------------------------------------------------------------
# masked softmax attention
# ---------------------------------------------------------------------------
AllowedFn = Callable[[np.ndarray], np.ndarray]  # query rows -> bool [len(rows), N]


def masked_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows: Sequence[int],
                          allowed: Optional[AllowedFn], scale: float
                          ) -> Tuple[np.ndarray, np.ndarray]:
    """O[i] = sum_j softmax_j(scale * q_i . k_j | allowed) v_j for the given rows.

    q, k, v: float64 [N, d] of one head in one layout. allowed(rows) gives the
    bool mask [len(rows), N] (None = all keys). Returns (O [len(rows), d],
    lse [len(rows)]) with lse = log sum_j exp(s_ij) over allowed keys. A row with
    no allowed key gives O = 0 and lse = -inf.
    """
    rows = np.asarray(rows, dtype=np.int64)
    d = q.shape[1]
    O = np.zeros((rows.size, d), dtype=np.float64)
    lse = np.full(rows.size, -np.inf, dtype=np.float64)
    for c0 in range(0, rows.size, _ROW_CHUNK):
        rr = rows[c0:c0 + _ROW_CHUNK]
        s = scale * (q[rr] @ k.T)  # [r, N]
        if allowed is not None:
            a = allowed(rr)
            s = np.where(a, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])
        m[empty] = 0.0
        p = np.exp(s - m)  # exp(-inf) = 0 for masked keys
        l = p.sum(axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            o = (p @ v) / l
            row_lse = m[:, 0] + np.log(l[:, 0])
        o[empty] = 0.0
        row_lse[empty] = -np.inf
        O[c0:c0 + rr.size] = o
        lse[c0:c0 + rr.size] = row_lse
    return O, lse


def attention_weights_rows(q: np.ndarray, k: np.ndarray, rows: Sequence[int],
                           allowed: Optional[AllowedFn], scale: float) -> np.ndarray:
    """Softmax weights [len(rows), N] of the same definition (for invariant tests)."""
    rr = np.asarray(rows, dtype=np.int64)
    s = scale * (q[rr] @ k.T)
    if allowed is not None:
        s = np.where(allowed(rr), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


def block_allowed_fn(bm: np.ndarray, block_q: int, block_k: int, N: int) -> AllowedFn:
    """Token-level view of a block mask: allowed(i, j) = BM[i // Bq][j // Bk]."""
    key_block = np.arange(N) // block_k

    def fn(rows: np.ndarray) -> np.ndarray:
        return bm[np.asarray(rows) // block_q][:, key_block]

    return fn


def sparse_attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, bm: np.ndarray,
                          block_q: int, block_k: int, scale: float,
                          rows: Optional[Sequence[int]] = None):
    """Block-sparse attention of one head in its layout (rows default: all)."""
    N = q.shape[0]
    if rows is None:
        rows = np.arange(N)
    return masked_attention_rows(q, k, v, rows, block_allowed_fn(bm, block_q, block_k, N),
                                 scale)


# ---------------------------------------------------------------------------
# online profiling
# ---------------------------------------------------------------------------
def profile_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, sample_idx: Sequence[int],
                 T: int, P: int, n_text: int, s: int, w: int, scale: float
                 ) -> Tuple[float, float, int]:
    """Online profiling of one head (frame-major q, k, v float64 [N, d]).

    Full attention and the spatial- and temporal-masked attentions are evaluated
    on the sampled query rows; each masked output is compared with the full one
    by the mean squared error over rows x channels. Returns (mse_spatial,
    mse_temporal, label) with label = HEAD_TEMPORAL iff mse_temporal <
    mse_spatial.
    """
    N = q.shape[0]
    rows = np.asarray(sample_idx, dtype=np.int64)
    cols = np.arange(N)
    o_full, _ = masked_attention_rows(q, k, v, rows, None, scale)
    o_s, _ = masked_attention_rows(
        q, k, v, rows, lambda rr: spatial_allowed(rr[:, None], cols[None, :], T, P, n_text, s),
        scale)
    o_t, _ = masked_attention_rows(
        q, k, v, rows, lambda rr: temporal_allowed(rr[:, None], cols[None, :], T, P, n_text, w),
        scale)
    mse_s = float(np.mean((o_s - o_full) ** 2))
    mse_t = float(np.mean((o_t - o_full) ** 2))
    label = HEAD_TEMPORAL if mse_t < mse_s else HEAD_SPATIAL
    return mse_s, mse_t, label


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------
def layer_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, label: int, T: int, P: int,
               n_text: int, s: int, w: int, block_q: int, block_k: int, scale: float,
               rows: Optional[Sequence[int]] = None, bm: Optional[np.ndarray] = None):
    """SVG attention output of one head at frame-major rows (default: all rows).

    A spatial head attends in frame-major order over its spatial block mask. A
    temporal head is permuted to position-major order, attends over the temporal
    block mask there and is permuted back. Returns (O rows [r, d] frame-major,
    lse rows).
    """
    N = q.shape[0]
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows, dtype=np.int64)
    kind = MASK_TEMPORAL if label == HEAD_TEMPORAL else MASK_SPATIAL
    pi = permutation(T, P, n_text) if kind == MASK_TEMPORAL else None
    layout_rows = rows if pi is None else pi[rows]
    if bm is None:
        # Only the block-mask rows the requested query rows fall in are needed.
        needed = np.unique(layout_rows // block_q)
        bm = np.zeros((n_blocks(N, block_q), n_blocks(N, block_k)), dtype=bool)
        bm[needed] = block_mask_rows(kind, needed, T, P, n_text, s, w, block_q, block_k)
    if kind == MASK_SPATIAL:
        return sparse_attention_rows(q, k, v, bm, block_q, block_k, scale, layout_rows)
    qp, kp, vp = (permute(x, T, P, n_text) for x in (q, k, v))
    return sparse_attention_rows(qp, kp, vp, bm, block_q, block_k, scale, layout_rows)


# ---------------------------------------------------------------------------
# FP8 (e4m3) quantisation of V for the FP8 PV product
# ---------------------------------------------------------------------------
# The project article "Sparse-VideoGen and the sparsity hiding inside video
# diffusion attention" (section "Publication record and the road ahead") lists
# FP8 attention as an open item; the pages fix no format or scheme. The one
# checked here: E4M3 in its "fn" form (1 sign, 4 exponent bits with bias 7, 3
# mantissa bits, no infinities, largest finite value 448 = 1.75 * 2^8, smallest
# normal 2^-6, subnormal spacing 2^-9), values rounded to nearest with ties to
# even and saturated to +-448; one scale per (head, channel).
E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value of each x (ties to even), saturating to +-448.

    In a binade [2^e, 2^(e+1)) with e >= -6 the grid spacing is 2^(e-3); below
    2^-6 (subnormals) it is 2^-9. Returns float64 values on the E4M3 grid."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    spacing = np.where(a >= 2.0 ** -6, 2.0 ** (e - 3), 2.0 ** -9)
    q = np.round(a / spacing) * spacing  # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(x < 0, -q, q)


def quantize_v_e4m3(v: np.ndarray):
    """Per-channel e4m3 quantisation of one head's V [N, d] (exact bf16 values).

    amax_c = max_j |v_jc|; the code of v_jc is e4m3_round of the fp32 product
    v_jc * fp32(448 / amax_c) (both the quotient and the product rounded to
    fp32, the precision in which the rounding decision is taken); the scale is
    fp32(amax_c / 448). A zero channel gets scale 0 and codes 0. Returns
    (codes float64 [N, d] on the E4M3 grid, scale float32 [d]); v ~= codes * scale.
    """
    v32 = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v32), axis=0).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0.0)).astype(np.float32)
    x = (v32 * inv[None, :]).astype(np.float32)
    codes = e4m3_round(x.astype(np.float64))
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return codes, scale


def flops_computed_blocks(bm: np.ndarray, N: int, block_q: int, block_k: int, d: int) -> int:
    """Algorithmic FLOPs of block-sparse attention: 4*d per computed (row, key) pair."""
    rows_in = np.minimum(block_q, N - np.arange(bm.shape[0]) * block_q)
    cols_in = np.minimum(block_k, N - np.arange(bm.shape[1]) * block_k)
    pairs = int((bm * rows_in[:, None] * cols_in[None, :]).sum())
    return 4 * d * pairs


__all__ = [n for n, o in list(globals().items())
           if not n.startswith("_") and not isinstance(o, type(math))
           and n not in ("annotations", "Callable", "Optional", "Sequence", "Tuple")]
