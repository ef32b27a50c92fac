"""Plain fp64 CPU oracle of the semantic-aware permutation row (Sparse VideoGen 2).

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The library never calls it
and shares no code with it.

Source: the project article "Sparse-VideoGen and the sparsity hiding inside
video diffusion attention", section "Three generations of the same idea": the
second generation replaces the fixed spatial/temporal patterns with
semantic-aware sparse attention built on an efficient token permutation, run
by a dynamic attention kernel and a flash (batched) k-means kernel; the
install section adds block-sparse attention with varied block sizes, and the
section "Publication record and the road ahead" calls Flash k-Means a batched
k-means clustering algorithm. The pages give no formula, so every rule below is
a reading, the plainest one the rest supports:

* clustering: per (batch, head), Lloyd's k-means with squared Euclidean
  distance, separately on the query vectors (C_q clusters) and on the key
  vectors (C_k clusters); the initial centroids are the rows floor(c * N / C),
  c = 0..C-1 (evenly spaced, deterministic); a fixed number of iterations, each
  an assignment (nearest centroid, ties to the smaller index; the centroids
  rounded to bf16 first, the operand format of the tensor-core distance
  product) followed by an update (each centroid the mean of its members; an
  empty cluster keeps its centroid). The result is the last iteration's
  assignment and the centroids computed from it;
* permutation: tokens stably sorted by cluster index (queries by their query
  cluster, keys and values by their key cluster), so every cluster is one
  contiguous run;
* selection: a query cluster a weighs key cluster b by the softmax over b of
  scale * c_q[a] . c_k[b] + log |b| (the attention a query at the centroid
  would pay to |b| keys at their centroid); it keeps the fewest clusters, in
  descending weight (ties to the smaller index), whose weights add up to at
  least top_p; empty key clusters are never kept;
* attention: block-granular on the sorted layouts, like the spatial/temporal
  path: a (query tile, key tile) pair of the sorted layouts is computed in full
  iff some query of the tile belongs to a cluster that keeps the cluster of
  some key of the tile;
* output rows are returned to the original order.

Everything is fp64 on the exact bf16 input values; matmul, exp and sums are
numpy library primitives.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

from .svg_oracle import (from_bf16_bits, masked_attention_rows, n_blocks, to_bf16_bits)


# ---------------------------------------------------------------------------
# k-means
# ---------------------------------------------------------------------------
def kmeans_init(x: np.ndarray, C: int) -> np.ndarray:
    """Initial centroids: the rows floor(c * N / C) of x (float64 [C, d])."""
    N = x.shape[0]
    idx = (np.arange(C, dtype=np.int64) * N) // C
    return np.asarray(x, dtype=np.float64)[idx].copy()


def bf16_values(c: np.ndarray) -> np.ndarray:
    """c rounded to bf16 (nearest, ties to even), as float64 values."""
    return from_bf16_bits(to_bf16_bits(c))


def kmeans_distances(x: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Squared Euclidean distances [N, C] from every row of x to the centroids
    rounded to bf16, ||x_i - c_k||^2 written out as a sum over channels."""
    cb = bf16_values(centroids)
    x = np.asarray(x, dtype=np.float64)
    return (np.sum(x * x, axis=1)[:, None] - 2.0 * (x @ cb.T) + np.sum(cb * cb, axis=1)[None, :])


def kmeans_assign(x: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Nearest centroid of every row (ties to the smaller index), int64 [N]."""
    return np.argmin(kmeans_distances(x, centroids), axis=1).astype(np.int64)


def kmeans_update(x: np.ndarray, assign: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """Mean of each cluster's members; an empty cluster keeps its centroid."""
    C, d = centroids.shape
    x = np.asarray(x, dtype=np.float64)
    sums = np.zeros((C, d))
    np.add.at(sums, assign, x)
    counts = np.bincount(assign, minlength=C).astype(np.float64)
    out = np.array(centroids, dtype=np.float64, copy=True)
    live = counts > 0
    out[live] = sums[live] / counts[live, None]
    return out


def kmeans(x: np.ndarray, C: int, iters: int) -> Tuple[np.ndarray, np.ndarray]:
    """Lloyd's k-means: init, then `iters` rounds of assignment + update.

    Returns (centroids float64 [C, d], assignment int64 [N]) where the
    centroids are the means of that assignment's clusters."""
    c = kmeans_init(x, C)
    a = None
    for _ in range(iters):
        a = kmeans_assign(x, c)
        c = kmeans_update(x, a, c)
    if a is None:
        a = kmeans_assign(x, c)
    return c, a


def kmeans_objective(x: np.ndarray, centroids: np.ndarray, assign: np.ndarray) -> float:
    """Sum over rows of the squared distance to the assigned (exact) centroid."""
    x = np.asarray(x, dtype=np.float64)
    d = x - np.asarray(centroids, dtype=np.float64)[assign]
    return float(np.sum(d * d))


# ---------------------------------------------------------------------------
# permutation
# ---------------------------------------------------------------------------
def cluster_permutation(assign: np.ndarray, C: int) -> Tuple[np.ndarray, np.ndarray]:
    """Stable sort of the tokens by cluster.

    Returns (order int64 [N]: order[pos] = original index of the token at
    sorted position pos; offsets int64 [C+1]: cluster c occupies sorted
    positions offsets[c] .. offsets[c+1]-1)."""
    assign = np.asarray(assign, dtype=np.int64)
    counts = np.bincount(assign, minlength=C)
    offsets = np.zeros(C + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    order = np.empty(assign.size, dtype=np.int64)
    fill = offsets[:-1].copy()
    for i, c in enumerate(assign):  # tokens in original order: a stable placement
        order[fill[c]] = i
        fill[c] += 1
    return order, offsets


def cluster_of_position(offsets: np.ndarray) -> np.ndarray:
    """Cluster index of every sorted position."""
    sizes = np.diff(offsets)
    return np.repeat(np.arange(sizes.size, dtype=np.int64), sizes)


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------
def select_clusters(cq: np.ndarray, ck: np.ndarray, sizes_k: np.ndarray, scale: float,
                    top_p: float) -> np.ndarray:
    """Key clusters kept by each query cluster, bool [C_q, C_k].

    Weight of key cluster b for query cluster a: softmax over b of
    scale * cq[a] . ck[b] + log(sizes_k[b]) (empty clusters weigh 0). Kept: the
    fewest clusters, taken in descending weight (ties to the smaller index),
    whose weights add up to at least top_p."""
    sizes_k = np.asarray(sizes_k, dtype=np.float64)
    z = scale * (np.asarray(cq, dtype=np.float64) @ np.asarray(ck, dtype=np.float64).T)
    with np.errstate(divide="ignore"):
        z = z + np.log(sizes_k)[None, :]
    z = z - np.max(z, axis=1, keepdims=True)
    w = np.exp(z)
    w = w / np.sum(w, axis=1, keepdims=True)
    sel = np.zeros(w.shape, dtype=bool)
    for a in range(w.shape[0]):
        order = sorted(range(w.shape[1]), key=lambda b: (-w[a, b], b))
        acc = 0.0
        for b in order:
            if sizes_k[b] == 0:
                continue
            sel[a, b] = True
            acc += w[a, b]
            if acc >= top_p:
                break
    return sel


def selection_weights(cq, ck, sizes_k, scale) -> np.ndarray:
    """The weights select_clusters ranks (for near-tie checks in tests)."""
    sizes_k = np.asarray(sizes_k, dtype=np.float64)
    z = scale * (np.asarray(cq, dtype=np.float64) @ np.asarray(ck, dtype=np.float64).T)
    with np.errstate(divide="ignore"):
        z = z + np.log(sizes_k)[None, :]
    z = z - np.max(z, axis=1, keepdims=True)
    w = np.exp(z)
    return w / np.sum(w, axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# block mask and attention on the sorted layouts
# ---------------------------------------------------------------------------
def semantic_block_mask(offsets_q: np.ndarray, offsets_k: np.ndarray, sel: np.ndarray,
                        block_q: int, block_k: int, tiles=None) -> np.ndarray:
    """bool [nQB, nKB]: tile pair (r, c) is on iff some sorted query position of
    tile r and sorted key position of tile c have sel[cluster(q), cluster(k)],
    evaluated token pair by token pair (brute force over positions). With
    `tiles`, only those query tiles are evaluated (the other rows stay off)."""
    cq = cluster_of_position(offsets_q)
    ck = cluster_of_position(offsets_k)
    Nq, Nk = cq.size, ck.size
    nqb, nkb = n_blocks(Nq, block_q), n_blocks(Nk, block_k)
    bm = np.zeros((nqb, nkb), dtype=bool)
    for r in (range(nqb) if tiles is None else sorted(set(int(t) for t in tiles))):
        rows = cq[r * block_q:min(Nq, (r + 1) * block_q)]
        allowed = sel[rows][:, ck]  # [rows of the tile, Nk]
        any_key = allowed.any(axis=0)
        padded = np.zeros(nkb * block_k, dtype=bool)
        padded[:Nk] = any_key
        bm[r] = padded.reshape(nkb, block_k).any(axis=1)
    return bm


def semantic_attention_rows(q, k, v, order_q, order_k, bm, block_q, block_k, scale, rows):
    """Output rows (original indices `rows`) of block-sparse attention over the
    sorted layouts: queries sorted by order_q, keys and values by order_k,
    tile pairs listed in bm. Returns (O [r, d], lse [r])."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    qs, ks, vs = q[order_q], k[order_k], v[order_k]
    pos_of = np.empty(order_q.size, dtype=np.int64)
    pos_of[order_q] = np.arange(order_q.size)
    srows = pos_of[np.asarray(rows, dtype=np.int64)]
    key_block = np.arange(ks.shape[0]) // block_k

    def allowed(rr):
        return bm[np.asarray(rr) // block_q][:, key_block]
    return masked_attention_rows(qs, ks, vs, srows, allowed, scale)


# ---------------------------------------------------------------------------
# SVG-EAR: error-aware routing and centroid compensation
# ---------------------------------------------------------------------------
# The project article, section "Three generations of the same idea": the third
# generation recovers the skipped attention blocks with parameter-free centroid
# compensation and routes high-error blocks to exact computation while the rest
# are compensated. The pages give no formula. The readings checked here:
#
# * statistics of key cluster b (over its members, in the key order): the key
#   centroid kbar_b (the k-means centroid, the members' mean), the value mean
#   vbar_b, and the value dispersion D_b = sqrt(mean over members and channels
#   of (v - vbar_b)^2);
# * routing: a pair (query cluster a, key cluster b) that the top-p selection
#   skips is computed exactly anyway when its estimated compensation error
#   w(a, b) * D_b (the selection weight times the dispersion of what the
#   centroid stands in for) exceeds a threshold tau;
# * compensation: every key that none of the computed tiles of a query's tile
#   covers is stood in for by its cluster: n_b(r) uncovered keys of cluster b
#   for query tile r add n_b(r) * exp(scale * q . kbar_b) to the softmax
#   denominator and the same times vbar_b to the numerator, with kbar_b and
#   vbar_b rounded to bf16 (the operand format of the tensor-core products);
# * every key is thus either attended exactly or compensated, once.
def cluster_value_stats(v: np.ndarray, order_k: np.ndarray, offsets_k: np.ndarray):
    """(vbar [Ck, d], D [Ck]) of the key clusters: the members' mean value and
    RMS dispersion (0 for an empty cluster)."""
    v = np.asarray(v, dtype=np.float64)
    C = offsets_k.size - 1
    vbar = np.zeros((C, v.shape[1]))
    disp = np.zeros(C)
    for b in range(C):
        mem = order_k[offsets_k[b]:offsets_k[b + 1]]
        if mem.size == 0:
            continue
        vbar[b] = v[mem].mean(axis=0)
        disp[b] = np.sqrt(np.mean((v[mem] - vbar[b]) ** 2))
    return vbar, disp


def route_clusters(sel: np.ndarray, weights: np.ndarray, disp: np.ndarray, tau: float):
    """The exact set after error-aware routing: sel, plus every skipped pair
    whose error estimate weights[a, b] * disp[b] exceeds tau."""
    return sel | (weights * disp[None, :] > tau)


def uncovered_counts(offsets_k: np.ndarray, bm_row: np.ndarray, block_k: int) -> np.ndarray:
    """n_b: keys of each key cluster outside the computed key tiles of one row."""
    ck = cluster_of_position(offsets_k)
    covered = np.repeat(bm_row, block_k)[:ck.size]
    return np.bincount(ck[~covered], minlength=offsets_k.size - 1)


def ear_attention_rows(q, k, v, order_q, order_k, offsets_k, kbar, vbar, bm, block_q, block_k,
                       scale, rows):
    """Compensated attention at original query rows `rows`: exact over the
    computed tiles of the sorted layouts, plus the centroid terms of every
    uncovered key (kbar, vbar rounded to bf16). Returns O [r, d]."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    qs, ks, vs = q[order_q], k[order_k], v[order_k]
    kb, vb = bf16_values(kbar), bf16_values(vbar)
    pos_of = np.empty(order_q.size, dtype=np.int64)
    pos_of[order_q] = np.arange(order_q.size)
    key_block = np.arange(ks.shape[0]) // block_k
    out = np.zeros((len(rows), q.shape[1]))
    for n, i in enumerate(np.asarray(rows, dtype=np.int64)):
        ip = pos_of[i]
        r = ip // block_q
        cov = bm[r][key_block]
        s = scale * (ks[cov] @ qs[ip])
        cnt = uncovered_counts(offsets_k, bm[r], block_k).astype(np.float64)
        live = cnt > 0
        z = scale * (kb[live] @ qs[ip]) + np.log(cnt[live])
        m = max(s.max() if s.size else -np.inf, z.max() if z.size else -np.inf)
        es, ez = np.exp(s - m), np.exp(z - m)
        out[n] = (es @ vs[cov] + ez @ vb[live]) / (es.sum() + ez.sum())
    return out


__all__ = ["kmeans_init", "bf16_values", "kmeans_distances", "kmeans_assign", "kmeans_update",
           "kmeans", "kmeans_objective", "cluster_permutation", "cluster_of_position",
           "select_clusters", "selection_weights", "semantic_block_mask",
           "semantic_attention_rows", "cluster_value_stats", "route_clusters",
           "uncovered_counts", "ear_attention_rows"]
