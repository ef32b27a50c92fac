"""Pins of the SVG2 (semantic-aware permutation) oracle, on the CPU.

Each pin holds the oracle against something other than itself: scikit-learn's
Lloyd k-means step, numpy's stable argsort, a selection worked by hand
(tests/golden), an interval formula for the tile mask, dense float64 SDPA, and
closed forms (well-separated blobs, one cluster, one cluster per row).
"""
import os

import numpy as np
import pytest
import torch

import oracle as O
from oracle import svg2_oracle as S2

HERE = os.path.dirname(os.path.abspath(__file__))


def _bf16(x):
    return O.from_bf16_bits(O.to_bf16_bits(x))


def test_kmeans_init_takes_evenly_spaced_rows():
    x = np.arange(40, dtype=np.float64).reshape(10, 4)
    c = S2.kmeans_init(x, 4)  # rows 0, 2, 5, 7
    assert np.array_equal(c[:, 0], [0.0, 8.0, 20.0, 28.0])


def test_one_lloyd_round_matches_scikit_learn():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((600, 16)) + np.repeat(rng.standard_normal((6, 16)) * 3, 100, 0))
    C = 8
    c0 = S2.kmeans_init(x, C)  # data rows: exact in bf16, so the assignment needs no rounding
    a = S2.kmeans_assign(x, c0)
    c1 = S2.kmeans_update(x, a, c0)
    km = KMeans(n_clusters=C, init=c0, n_init=1, max_iter=1, algorithm="lloyd", tol=0.0)
    km.fit(x)
    np.testing.assert_allclose(c1, km.cluster_centers_, rtol=0, atol=1e-12)


def test_well_separated_blobs_are_recovered_exactly():
    rng = np.random.default_rng(4)
    centers = np.array([[0, 0, 0, 0], [40, 0, 0, 0], [0, 40, 0, 0], [0, 0, 40, 0]], float)
    labels = np.repeat(np.arange(4), 50)
    perm = rng.permutation(200)
    x = _bf16(centers[labels[perm]] + rng.standard_normal((200, 4)))
    c, a = S2.kmeans(x, 4, iters=5)
    # every cluster is one blob, and each centroid is its blob's mean
    for k in range(4):
        members = labels[perm][a == k]
        assert members.size > 0 and np.all(members == members[0])
        np.testing.assert_allclose(c[k], x[a == k].mean(axis=0), atol=1e-12)


def test_one_cluster_and_one_cluster_per_row():
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((30, 8)))
    c, a = S2.kmeans(x, 1, iters=3)
    assert np.all(a == 0)
    np.testing.assert_allclose(c[0], x.mean(axis=0), atol=1e-12)
    c, a = S2.kmeans(x, 30, iters=2)  # every row its own centroid
    assert np.array_equal(a, np.arange(30))
    np.testing.assert_array_equal(c, x)


def test_empty_cluster_keeps_its_centroid():
    x = np.array([[0.0, 0.0], [0.0, 1.0], [10.0, 0.0]])
    c0 = np.array([[0.0, 0.5], [10.0, 0.0], [100.0, 100.0]])
    a = S2.kmeans_assign(x, c0)
    assert list(a) == [0, 0, 1]
    c1 = S2.kmeans_update(x, a, c0)
    assert np.array_equal(c1[2], [100.0, 100.0])


def test_assignment_uses_bf16_centroids_and_breaks_ties_low():
    x = np.array([[1.0, 0.0]])
    # 1 + 2^-10 is not a bf16 value: it rounds to 1.0, so both centroids sit at
    # the same distance and the smaller index wins
    c = np.array([[1.0 + 2.0 ** -10, 0.0], [1.0, 0.0]])
    assert S2.kmeans_assign(x, c)[0] == 0
    c = np.array([[1.0 + 2.0 ** -6, 0.0], [1.0, 0.0]])  # representable: index 1 is nearer
    assert S2.kmeans_assign(x, c)[0] == 1


def test_cluster_permutation_is_the_stable_argsort():
    rng = np.random.default_rng(6)
    a = rng.integers(0, 7, 500)
    order, offsets = S2.cluster_permutation(a, 9)
    assert np.array_equal(order, np.argsort(a, kind="stable"))
    assert np.array_equal(np.sort(order), np.arange(500))
    assert np.array_equal(np.diff(offsets), np.bincount(a, minlength=9))
    assert np.array_equal(S2.cluster_of_position(offsets), a[order])


def _golden_selection():
    rows = []
    for line in open(os.path.join(HERE, "golden", "svg2_selection_hand_example.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        rows.append((float(parts[1]), [int(b) for b in parts[3:]]))
    return rows


def test_selection_hand_example():
    cq = np.array([[np.log(2.0), 0.0]])
    ck = np.array([[1.0, 0.0], [0.0, 5.0], [2.0, 0.0]])
    sizes = np.array([1, 3, 1])
    cases = _golden_selection()
    assert len(cases) == 3
    for top_p, keep in cases:
        sel = S2.select_clusters(cq, ck, sizes, 1.0, top_p)
        assert sorted(np.nonzero(sel[0])[0].tolist()) == keep


def test_selection_limits():
    rng = np.random.default_rng(7)
    cq, ck = rng.standard_normal((5, 8)), rng.standard_normal((9, 8))
    sizes = rng.integers(1, 20, 9)
    sizes[3] = 0
    all_sel = S2.select_clusters(cq, ck, sizes, 0.3, 1.0)
    assert np.array_equal(all_sel, np.repeat((sizes > 0)[None], 5, 0))  # p = 1: every non-empty
    one = S2.select_clusters(cq, ck, sizes, 0.3, 1e-9)
    w = S2.selection_weights(cq, ck, sizes, 0.3)
    assert np.all(one.sum(axis=1) == 1) and np.array_equal(np.argmax(one, 1), np.argmax(w, 1))
    # equal centroids: the weights are the cluster sizes' shares
    eq = S2.selection_weights(np.ones((1, 4)), np.ones((3, 4)), np.array([1, 2, 5]), 1.0)
    np.testing.assert_allclose(eq[0], [1 / 8, 2 / 8, 5 / 8])


def _interval_tile_mask(offsets_q, offsets_k, sel, bq, bk):
    """Closed form: cluster a covers sorted query positions [oq[a], oq[a+1]) ->
    tiles oq[a]//bq .. (oq[a+1]-1)//bq; likewise for key clusters."""
    Nq, Nk = offsets_q[-1], offsets_k[-1]
    bm = np.zeros((-(-Nq // bq), -(-Nk // bk)), dtype=bool)
    for a in range(len(offsets_q) - 1):
        if offsets_q[a + 1] == offsets_q[a]:
            continue
        r0, r1 = offsets_q[a] // bq, (offsets_q[a + 1] - 1) // bq
        for b in np.nonzero(sel[a])[0]:
            if offsets_k[b + 1] == offsets_k[b]:
                continue
            c0, c1 = offsets_k[b] // bk, (offsets_k[b + 1] - 1) // bk
            bm[r0:r1 + 1, c0:c1 + 1] = True
    return bm


@pytest.mark.parametrize("seed", range(6))
def test_semantic_block_mask_equals_the_interval_formula(seed):
    rng = np.random.default_rng(100 + seed)
    Cq, Ck = rng.integers(2, 9), rng.integers(2, 9)
    sq, sk = rng.integers(0, 40, Cq), rng.integers(0, 40, Ck)
    oq = np.concatenate([[0], np.cumsum(sq)])
    ok = np.concatenate([[0], np.cumsum(sk)])
    if oq[-1] == 0 or ok[-1] == 0:
        return
    sel = rng.random((Cq, Ck)) < 0.3
    for bq, bk in [(16, 16), (8, 32), (64, 4)]:
        want = _interval_tile_mask(oq, ok, sel, bq, bk)
        assert np.array_equal(S2.semantic_block_mask(oq, ok, sel, bq, bk), want)


def test_semantic_attention_with_every_cluster_kept_is_dense_attention():
    rng = np.random.default_rng(8)
    N, d = 150, 16
    q, k, v = (_bf16(rng.standard_normal((N, d))) for _ in range(3))
    aq, ak = rng.integers(0, 5, N), rng.integers(0, 6, N)
    oq_, offq = S2.cluster_permutation(aq, 5)
    ok_, offk = S2.cluster_permutation(ak, 6)
    sel = np.ones((5, 6), dtype=bool)
    bm = S2.semantic_block_mask(offq, offk, sel, 32, 32)
    got, _ = S2.semantic_attention_rows(q, k, v, oq_, ok_, bm, 32, 32, 0.25, np.arange(N))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        scale=0.25)[0].numpy()
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_semantic_attention_restricted_to_one_cluster_pair():
    # two query clusters, two key clusters, 1x1 tiles: query cluster 0 keeps
    # only key cluster 1, so its rows equal softmax attention over those keys
    rng = np.random.default_rng(9)
    N, d = 20, 8
    q, k, v = (_bf16(rng.standard_normal((N, d))) for _ in range(3))
    aq = np.array([0, 1] * 10)
    ak = np.array([0] * 12 + [1] * 8)
    oq_, offq = S2.cluster_permutation(aq, 2)
    ok_, offk = S2.cluster_permutation(ak, 2)
    sel = np.array([[False, True], [True, True]])
    bm = S2.semantic_block_mask(offq, offk, sel, 1, 1)
    rows = np.nonzero(aq == 0)[0]
    got, _ = S2.semantic_attention_rows(q, k, v, oq_, ok_, bm, 1, 1, 0.5, rows)
    keys = np.nonzero(ak == 1)[0]
    s = 0.5 * q[rows] @ k[keys].T
    p = np.exp(s - s.max(1, keepdims=True))
    want = (p / p.sum(1, keepdims=True)) @ v[keys]
    np.testing.assert_allclose(got, want, atol=1e-12)


# ---------------------------------------------------------------------------
# SVG-EAR readings
# ---------------------------------------------------------------------------
def _plan(rng, N, Cq, Ck):
    aq, ak = rng.integers(0, Cq, N), rng.integers(0, Ck, N)
    oq_, offq = S2.cluster_permutation(aq, Cq)
    ok_, offk = S2.cluster_permutation(ak, Ck)
    return aq, ak, oq_, offq, ok_, offk


def test_compensation_is_exact_when_every_cluster_is_one_point():
    """Keys (and values) identical within each key cluster: a cluster's centroid
    and mean are its members, so compensating any uncovered key is exact and the
    result is dense attention whatever tiles are computed."""
    rng = np.random.default_rng(12)
    N, d, Cq, Ck = 200, 16, 4, 6
    aq, ak, oq_, offq, ok_, offk = _plan(rng, N, Cq, Ck)
    kpts, vpts = _bf16(rng.standard_normal((Ck, d))), _bf16(rng.standard_normal((Ck, d)))
    q = _bf16(rng.standard_normal((N, d)))
    k, v = kpts[ak], vpts[ak]
    kbar, vbar = kpts.copy(), vpts.copy()
    sel = rng.random((Cq, Ck)) < 0.3
    bm = S2.semantic_block_mask(offq, offk, sel, 16, 16)
    got = S2.ear_attention_rows(q, k, v, oq_, ok_, offk, kbar, vbar, bm, 16, 16, 0.3,
                                np.arange(N))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        scale=0.3)[0].numpy()
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_compensation_vanishes_when_every_tile_is_computed():
    rng = np.random.default_rng(13)
    N, d, Cq, Ck = 150, 8, 3, 5
    aq, ak, oq_, offq, ok_, offk = _plan(rng, N, Cq, Ck)
    q, k, v = (_bf16(rng.standard_normal((N, d))) for _ in range(3))
    bm = np.ones((-(-N // 32), -(-N // 32)), dtype=bool)
    kbar = rng.standard_normal((Ck, d))  # unused: nothing is uncovered
    got = S2.ear_attention_rows(q, k, v, oq_, ok_, offk, kbar, kbar, bm, 32, 32, 0.5,
                                np.arange(N))
    want, _ = S2.semantic_attention_rows(q, k, v, oq_, ok_, bm, 32, 32, 0.5, np.arange(N))
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_uncovered_counts_by_hand():
    # clusters of sizes 3, 0, 5, 2 over 10 sorted keys; tiles of 4 keys:
    # tile 0 = keys 0-3 (cluster 0: 0,1,2; cluster 2: 3), tile 1 = keys 4-7
    # (cluster 2: 4-7), tile 2 = keys 8-9 (cluster 3)
    offk = np.array([0, 3, 3, 8, 10])
    assert list(S2.uncovered_counts(offk, np.array([True, False, False]), 4)) == [0, 0, 4, 2]
    assert list(S2.uncovered_counts(offk, np.array([False, True, True]), 4)) == [3, 0, 1, 0]


def test_cluster_value_stats_and_routing():
    v = np.array([[1.0, 3.0], [3.0, 5.0], [2.0, 2.0]])
    order_k = np.array([0, 1, 2])
    offk = np.array([0, 2, 2, 3])  # cluster 0 = rows 0, 1; cluster 1 empty; cluster 2 = row 2
    vbar, disp = S2.cluster_value_stats(v, order_k, offk)
    assert np.array_equal(vbar, [[2.0, 4.0], [0.0, 0.0], [2.0, 2.0]])
    assert np.allclose(disp, [1.0, 0.0, 0.0])  # deviations +-1 in every channel
    sel = np.array([[True, False, False]])
    w = np.array([[0.8, 0.0, 0.2]])
    assert np.array_equal(S2.route_clusters(sel, w, np.array([1.0, 0.0, 0.5]), 0.05),
                          [[True, False, True]])  # 0.2 * 0.5 = 0.1 > 0.05
    assert np.array_equal(S2.route_clusters(sel, w, np.array([1.0, 0.0, 0.1]), 0.05),
                          [[True, False, False]])  # 0.02 <= 0.05
