"""GPU parity of the semantic-aware permutation path (Sparse VideoGen 2) against
the fp64 oracle (oracle/svg2_oracle.py), step by step on shared seeded inputs.

Integer results (cluster orders, offsets, the tile CSR, permuted rows) must be
bit-exact. Where a floating-point comparison decides an integer (the nearest
centroid, whether a cluster is kept) the kernel and the oracle take the
decision from the same inputs (bf16 centroids for the distances, the same fp32
centroids for the selection) in different precisions (fp32 accumulation vs
fp64), so a decision whose margin lies within fp32 rounding is a near tie:
there the kernel's choice must be a valid one (within the rounding bound of the
best), everywhere else it must equal the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import svg2_oracle as S2
from gpu_util import assert_close, rand_bf16, status_clean, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _ws(svg, BH, N, d, C):
    return torch.empty(svg.svg2_kmeans_workspace_bytes(BH, N, d, C) // 4 + 64,
                       dtype=torch.float32, device="cuda")


def _assign_bound(x, cent):
    """Rounding bound of one distance in the kernel (fp32 accumulation of d
    bf16 products and of the squared norm): 2^-14 (|x| max|c| + max|c|^2),
    well above d * 2^-24 of each term for d <= 128."""
    cb = S2.bf16_values(cent)
    cmax = np.sqrt(np.max(np.sum(cb * cb, axis=1)))
    xn = np.sqrt(np.sum(x * x, axis=1))
    return 2.0 ** -14 * (xn * cmax + cmax * cmax)


def _check_assignment(x, cent, got):
    """Exact where the oracle's best centroid beats the runner-up by more than
    the rounding bound; valid (within the bound of the best) elsewhere.
    Returns the rows that were near ties."""
    dist = S2.kmeans_distances(x, cent)
    want = np.argmin(dist, axis=1)
    srt = np.sort(dist, axis=1)
    eps = _assign_bound(x, cent)
    tie = (srt[:, 1] - srt[:, 0]) <= eps
    assert np.array_equal(got[~tie], want[~tie]), "assignment differs outside near ties"
    best = dist[np.arange(x.shape[0]), got]
    assert np.all(best[tie] <= srt[tie, 0] + eps[tie]), "a near-tie choice is not valid"
    return np.nonzero(tie)[0]


# BH, N, d, C, planted
# the last case has more heads than SMs (one assignment CTA per head) and
# chunks shorter than one 256-row chunk per head
STEP_CASES = [(2, 1000, 64, 16, False), (2, 1500, 128, 48, False), (1, 3000, 128, 256, True),
              (3, 777, 128, 32, True), (160, 200, 64, 16, True)]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: "BH{}N{}d{}C{}".format(*c[:4]))
def test_kmeans_step_matches_oracle(svg, case):
    BH, N, d, C, planted = case
    rng = np.random.default_rng(N + C)
    x = rng.standard_normal((BH, N, d))
    if planted:
        x += np.repeat(rng.standard_normal((BH, 8, d)) * 3, -(-N // 8), axis=1)[:, :N]
    xb = torch.from_numpy(O.to_bf16_bits(x).view(np.int16)).view(torch.bfloat16)
    xn = to_f64(xb)
    # input centroids: the oracle's init followed by one oracle iteration
    c_in = np.stack([S2.kmeans_update(xn[h], S2.kmeans_assign(xn[h], S2.kmeans_init(xn[h], C)),
                                      S2.kmeans_init(xn[h], C)) for h in range(BH)])
    c_in32 = c_in.astype(np.float32)
    cin_d = torch.from_numpy(c_in32).cuda()
    cout = torch.full((BH, C, d), float("nan"), device="cuda")
    assign = torch.full((BH, N), -1, dtype=torch.int32, device="cuda")
    order = torch.full((BH, N), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((BH, C + 1), -1, dtype=torch.int32, device="cuda")
    svg.svg2_kmeans_step(BH, N, d, C, xb.cuda(), cin_d, cout, assign, order, offsets,
                         _ws(svg, BH, N, d, C))
    torch.cuda.synchronize()
    a, o, off, co = (t.cpu().numpy() for t in (assign, order, offsets, cout))
    for h in range(BH):
        ties = _check_assignment(xn[h], c_in32[h].astype(np.float64), a[h])
        # the order is the stable sort of the kernel's own assignment
        assert np.array_equal(o[h], np.argsort(a[h], kind="stable"))
        assert np.array_equal(np.diff(off[h]), np.bincount(a[h], minlength=C)) and off[h, 0] == 0
        want_a = S2.kmeans_assign(xn[h], c_in32[h].astype(np.float64))
        want_c = S2.kmeans_update(xn[h], want_a, c_in32[h].astype(np.float64))
        # clusters whose member set is the oracle's: the same mean to fp32 rounding
        touched = set(want_a[ties].tolist()) | set(a[h][ties].tolist())
        same = [c for c in range(C) if c not in touched]
        # fp32 sums of up to a few hundred members in order: relative error well below 1e-5
        np.testing.assert_allclose(co[h][same], want_c[same], rtol=1e-5, atol=1e-5)
        print(f"KMEANS-STEP {case} head {h}: {len(ties)} near-tie rows of {N}")
    status_clean()


def test_kmeans_recovers_planted_frames_exactly(svg):
    """Planted per-frame vectors (the spatial-head input of the synthetic
    workloads) with one cluster per frame: the initial rows c * N / C fall one
    in each frame, every assignment has a wide margin, and the whole k-means
    (assignments, order, offsets) equals the oracle's bit for bit."""
    BH, T, P, d, C, iters = 3, 16, 160, 128, 16, 4
    N = T * P
    rng = np.random.default_rng(11)
    e = rng.standard_normal((BH, T, d)) * 2.0
    x = 0.5 * rng.standard_normal((BH, N, d)) + np.repeat(e, P, axis=1)
    xb = torch.from_numpy(O.to_bf16_bits(x).view(np.int16)).view(torch.bfloat16)
    xn = to_f64(xb)
    cent = torch.empty((BH, C, d), device="cuda")
    assign, order = (torch.empty((BH, N), dtype=torch.int32, device="cuda") for _ in range(2))
    offsets = torch.empty((BH, C + 1), dtype=torch.int32, device="cuda")
    svg.svg2_kmeans(BH, N, d, C, iters, xb.cuda(), cent, assign, order, offsets,
                    _ws(svg, BH, N, d, C))
    torch.cuda.synchronize()
    for h in range(BH):
        wc, wa = S2.kmeans(xn[h], C, iters)
        wo, woff = S2.cluster_permutation(wa, C)
        assert np.array_equal(assign[h].cpu().numpy(), wa)
        assert np.array_equal(order[h].cpu().numpy(), wo)
        assert np.array_equal(offsets[h].cpu().numpy(), woff)
        np.testing.assert_allclose(cent[h].cpu().numpy(), wc, rtol=1e-5, atol=1e-5)
    status_clean()


def test_kmeans_full_size_is_a_valid_lloyd_result(svg):
    """HunyuanVideo-shaped head count and length (N = 119 056, d = 128, C = 256):
    the kernel's result is a fixed point of its own definition (every
    centroid the fp32 mean of its members, every row at a nearest bf16
    centroid of the previous round within rounding), and its objective is
    within 1 % of the oracle's k-means from the same start."""
    import svg_inputs as SI
    wl = SI.HUNYUAN.replace(H=2, n_spatial=1)
    q, _, _ = SI.make_qkv(wl)
    BH, N, d, C, iters = 2, wl.N, wl.d, 256, 3
    qd = q.reshape(BH, N, d).contiguous()
    cent = torch.empty((BH, C, d), device="cuda")
    assign, order = (torch.empty((BH, N), dtype=torch.int32, device="cuda") for _ in range(2))
    offsets = torch.empty((BH, C + 1), dtype=torch.int32, device="cuda")
    svg.svg2_kmeans(BH, N, d, C, iters, qd.cuda(), cent, assign, order, offsets,
                    _ws(svg, BH, N, d, C))
    torch.cuda.synchronize()
    xn = to_f64(qd)
    for h in range(BH):
        a = assign[h].cpu().numpy()
        c = cent[h].cpu().numpy().astype(np.float64)
        sums = np.zeros((C, d))
        np.add.at(sums, a, xn[h])
        cnt = np.bincount(a, minlength=C)
        live = cnt > 0
        # fp32 sums of up to thousands of members: sqrt(n) * 2^-24 typical, n * 2^-24 at worst
        np.testing.assert_allclose(c[live], sums[live] / cnt[live, None], rtol=1e-4, atol=1e-4)
        assert np.array_equal(order[h].cpu().numpy(), np.argsort(a, kind="stable"))
        wc, wa = S2.kmeans(xn[h], C, iters)
        obj_gpu = float(np.sum((xn[h] - c[a]) ** 2))
        obj_ref = S2.kmeans_objective(xn[h], wc, wa)
        print(f"KMEANS-FULL head {h}: objective {obj_gpu:.6e} oracle {obj_ref:.6e} "
              f"assignments equal {np.mean(a == wa):.5f}")
        assert abs(obj_gpu - obj_ref) <= 1e-2 * obj_ref
    status_clean()


def _selection_valid(w, sizes, got_row, top_p, eps=1e-5):
    """A kept set is valid if it is a prefix of the weight order up to eps
    ties, reaches top_p - eps, and would not reach top_p + eps without its
    lightest member."""
    live = sizes > 0
    kept = got_row & live
    if not np.any(kept):
        return False
    tot = w[kept].sum()
    lightest = w[kept].min()
    heaviest_out = w[live & ~kept].max() if np.any(live & ~kept) else -1.0
    return tot >= top_p - eps and tot - lightest < top_p + eps and lightest >= heaviest_out - eps


@pytest.mark.parametrize("Cq,Ck,top_p", [(8, 16, 0.9), (33, 256, 0.5), (256, 256, 0.95),
                                         (5, 1000, 0.8)])
def test_select_clusters_matches_oracle(svg, Cq, Ck, top_p):
    BH, d, scale = 3, 128, 1.0 / np.sqrt(128)
    rng = np.random.default_rng(Cq * 7 + Ck)
    cq = (rng.standard_normal((BH, Cq, d)) * 2).astype(np.float32)
    ck = (rng.standard_normal((BH, Ck, d)) * 2).astype(np.float32)
    sizes = rng.integers(0, 600, (BH, Ck))
    sizes[:, ::7] = 0  # empty clusters
    offsets = np.concatenate([np.zeros((BH, 1), np.int64), np.cumsum(sizes, 1)], 1).astype(np.int32)
    words = (Ck + 31) // 32
    sel = torch.full((BH, Cq, words), -1, dtype=torch.int32, device="cuda")
    svg.svg2_select_clusters(BH, d, Cq, Ck, scale, top_p, torch.from_numpy(cq).cuda(),
                             torch.from_numpy(ck).cuda(), torch.from_numpy(offsets).cuda(), sel)
    torch.cuda.synchronize()
    bits = sel.cpu().numpy().view(np.uint32)
    got = ((bits[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(BH, Cq, -1)[..., :Ck]
    got = got.astype(bool)
    exact = 0
    for h in range(BH):
        want = S2.select_clusters(cq[h].astype(np.float64), ck[h].astype(np.float64), sizes[h],
                                  scale, top_p)
        w = S2.selection_weights(cq[h].astype(np.float64), ck[h].astype(np.float64), sizes[h],
                                 scale)
        for a in range(Cq):
            if np.array_equal(got[h, a], want[a]):
                exact += 1
                continue
            assert _selection_valid(w[a], sizes[h], got[h, a], top_p), (h, a)
    print(f"SELECT Cq{Cq} Ck{Ck} p{top_p}: {exact} of {BH * Cq} rows equal to the oracle's")
    assert exact >= BH * Cq - max(1, BH * Cq // 50)
    status_clean()


@pytest.mark.parametrize("N,Cq,Ck,bk,density", [(1000, 7, 9, 128, 0.3), (5000, 32, 40, 64, 0.1),
                                                (20000, 256, 256, 128, 0.05), (300, 3, 2, 64, 1.0)])
def test_tile_csr_bit_exact(svg, N, Cq, Ck, bk, density):
    BH = 3
    rng = np.random.default_rng(N + Cq)
    offs_q, offs_k, sels = [], [], []
    for _ in range(BH):
        sq = rng.multinomial(N, rng.dirichlet(np.ones(Cq) * 0.5))
        sk = rng.multinomial(N, rng.dirichlet(np.ones(Ck) * 0.5))
        offs_q.append(np.concatenate([[0], np.cumsum(sq)]))
        offs_k.append(np.concatenate([[0], np.cumsum(sk)]))
        sels.append(rng.random((Cq, Ck)) < density)
    words = (Ck + 31) // 32
    packed = np.zeros((BH, Cq, words), dtype=np.uint32)
    for h in range(BH):
        for b in range(Ck):
            packed[h, :, b // 32] |= sels[h][:, b].astype(np.uint32) << np.uint32(b % 32)
    nqb, nkb = -(-N // 128), -(-N // bk)
    row_ptr = torch.full((BH * nqb + 1,), -1, dtype=torch.int32, device="cuda")
    col_idx = torch.full((BH * nqb * nkb,), -1, dtype=torch.int32, device="cuda")
    counts = torch.empty(BH * nqb, dtype=torch.int32, device="cuda")
    oq = torch.from_numpy(np.stack(offs_q).astype(np.int32)).cuda()
    ok = torch.from_numpy(np.stack(offs_k).astype(np.int32)).cuda()
    svg.svg2_build_tile_csr(BH, N, Cq, Ck, 128, bk, oq, ok,
                            torch.from_numpy(packed.view(np.int32)).cuda(), row_ptr, col_idx,
                            counts)
    torch.cuda.synchronize()
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    want_rp, want_ci = [0], []
    for h in range(BH):
        bm = S2.semantic_block_mask(offs_q[h], offs_k[h], sels[h], 128, bk)
        for r in range(nqb):
            cols = np.nonzero(bm[r])[0]
            want_ci.extend(cols.tolist())
            want_rp.append(want_rp[-1] + cols.size)
    assert np.array_equal(rp, np.array(want_rp))
    assert np.array_equal(ci[:rp[-1]], np.array(want_ci, dtype=np.int64))
    status_clean()


def test_gather_scatter_rows_bit_exact(svg):
    BH, N, d = 3, 1234, 128
    x = rand_bf16((BH, N, d), seed=5).cuda()
    order = torch.stack([torch.randperm(N, generator=torch.Generator().manual_seed(h))
                         for h in range(BH)]).to(torch.int32).cuda()
    y, back = torch.empty_like(x), torch.empty_like(x)
    svg.svg2_gather_rows(BH, N, d, x, order, y)
    svg.svg2_scatter_rows(BH, N, d, y, order, back)
    torch.cuda.synchronize()
    for h in range(BH):
        assert torch.equal(y[h].view(torch.int16), x[h, order[h].long()].view(torch.int16))
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    status_clean()


@pytest.mark.parametrize("N,d,bk,Cq,Ck,density", [(1000, 128, 128, 5, 7, 0.4),
                                                  (3000, 64, 64, 16, 20, 0.15),
                                                  (2600, 128, 128, 12, 12, 1.0)])
def test_sparse_attention_on_sorted_layouts(svg, N, d, bk, Cq, Ck, density):
    """Seeded plans (orders, cluster sizes, kept pairs) drive both sides: the
    kernel path (gather, tile CSR, attention, scatter) against the oracle's
    attention over the same plan."""
    BH, scale = 2, 1.0 / np.sqrt(d)
    rng = np.random.default_rng(N + d)
    q, k, v = (rand_bf16((BH, N, d), seed=N + i) for i in range(3))
    plans = []
    for h in range(BH):
        aq, ak = rng.integers(0, Cq, N), rng.integers(0, Ck, N)
        oq_, offq = S2.cluster_permutation(aq, Cq)
        ok_, offk = S2.cluster_permutation(ak, Ck)
        sel = rng.random((Cq, Ck)) < density
        sel[np.arange(Cq), rng.integers(0, Ck, Cq)] = True  # every query cluster keeps one
        plans.append((oq_, offq, ok_, offk, sel))
    stackd = lambda i: torch.from_numpy(np.stack([p[i] for p in plans]).astype(np.int32)).cuda()  # noqa: E731
    order_q, off_q, order_k, off_k = stackd(0), stackd(1), stackd(2), stackd(3)
    words = (Ck + 31) // 32
    packed = np.zeros((BH, Cq, words), dtype=np.uint32)
    for h in range(BH):
        for b in range(Ck):
            packed[h, :, b // 32] |= plans[h][4][:, b].astype(np.uint32) << np.uint32(b % 32)
    nqb, nkb = -(-N // 128), -(-N // bk)
    row_ptr = torch.empty(BH * nqb + 1, dtype=torch.int32, device="cuda")
    col_idx = torch.empty(BH * nqb * nkb, dtype=torch.int32, device="cuda")
    counts = torch.empty(BH * nqb, dtype=torch.int32, device="cuda")
    svg.svg2_build_tile_csr(BH, N, Cq, Ck, 128, bk, off_q, off_k,
                            torch.from_numpy(packed.view(np.int32)).cuda(), row_ptr, col_idx,
                            counts)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    qs, ks, vs, os_, o = (torch.empty_like(qd) for _ in range(5))
    svg.svg2_gather_rows(BH, N, d, qd, order_q, qs)
    svg.svg2_gather_rows(BH, N, d, kd, order_k, ks)
    svg.svg2_gather_rows(BH, N, d, vd, order_k, vs)
    svg.svg2_sparse_attention(BH, N, d, bk, scale, qs, ks, vs, row_ptr, col_idx, os_)
    svg.svg2_scatter_rows(BH, N, d, os_, order_q, o)
    torch.cuda.synchronize()
    got = to_f64(o)
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    for h in range(BH):
        oq_, offq, ok_, offk, sel = plans[h]
        bm = S2.semantic_block_mask(offq, offk, sel, 128, bk)
        want, _ = S2.semantic_attention_rows(qn[h], kn[h], vn[h], oq_, ok_, bm, 128, bk, scale,
                                             np.arange(N))
        assert_close(got[h], want, f"sorted-layout attention N{N} d{d} head {h}")
    status_clean()


def test_semantic_layer_end_to_end_on_planted_frames(svg):
    """The whole path through SemanticSparseLayer on planted per-frame heads
    with one cluster per frame: k-means, permutation, selection and tiles are
    unambiguous, so the plan equals the oracle's and the output matches the
    oracle's semantic attention within the attention bars."""
    from video_dit_spatial_b200.layer import SemanticSparseLayer
    B, H, T, P, d = 1, 2, 16, 200, 128
    N = T * P
    rng = np.random.default_rng(21)
    e = np.repeat(rng.standard_normal((H, T, d)) * 2.0, P, axis=1)  # one vector per frame
    qkv = [0.5 * rng.standard_normal((H, N, d)) + e, 0.5 * rng.standard_normal((H, N, d)) + e,
           rng.standard_normal((H, N, d))]
    q, k, v = (torch.from_numpy(O.to_bf16_bits(x).view(np.int16)).view(torch.bfloat16)
               .reshape(B, H, N, d) for x in qkv)
    layer = SemanticSparseLayer(B, H, N, d, Cq=T, Ck=T, iters=4, top_p=0.9)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    layer.forward(q.cuda(), k.cuda(), v.cuda(), o)
    torch.cuda.synchronize()
    got = to_f64(o)
    scale = 1.0 / np.sqrt(d)
    for h in range(H):
        qn, kn, vn = to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h])
        cq, aq = S2.kmeans(qn, T, 4)
        ck, ak = S2.kmeans(kn, T, 4)
        oq_, offq = S2.cluster_permutation(aq, T)
        ok_, offk = S2.cluster_permutation(ak, T)
        assert np.array_equal(layer.order_q[h].cpu().numpy(), oq_)
        assert np.array_equal(layer.order_k[h].cpu().numpy(), ok_)
        sel = S2.select_clusters(cq, ck, np.diff(offk), scale, 0.9)
        bm = S2.semantic_block_mask(offq, offk, sel, 128, 128)
        rp = layer.row_ptr.cpu().numpy()
        ci = layer.col_idx.cpu().numpy()
        nqb = layer.nqb
        for r in range(nqb):
            row = h * nqb + r
            assert np.array_equal(ci[rp[row]:rp[row + 1]], np.nonzero(bm[r])[0]), (h, r)
        want, _ = S2.semantic_attention_rows(qn, kn, vn, oq_, ok_, bm, 128, 128, scale,
                                             np.arange(N))
        assert_close(got[0, h], want, f"semantic layer head {h}")
        print(f"SEMANTIC head {h}: tile density {bm.mean():.4f}")
    status_clean()


def _unpack_sel(sel, Ck):
    bits = sel.cpu().numpy().view(np.uint32)
    return (((bits[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1)
            .reshape(bits.shape[0], bits.shape[1], -1)[..., :Ck].astype(bool))


@pytest.mark.parametrize("wname", ["hunyuan_B1_H24_d128_T33_P3600_L256",
                                   "cogvideox15_B1_H48_d64_T11_P4080_L226"],
                         ids=["hunyuan_d128", "cogvideox_d64"])
@pytest.mark.parametrize("ear_tau", [None, 0.01], ids=["svg2", "ear"])
def test_semantic_layer_full_size_sampled_rows(svg, ear_tau, wname):
    """Full-length workloads (HunyuanVideo-shaped N = 119 056, d = 128, and
    CogVideoX-shaped N = 45 106, d = 64), 2 heads of the seeded layer, C = 256
    clusters, 10 iterations, top-p 0.9, with and without SVG-EAR routing: every
    part of the plan the GPU builds is checked against what defines it, and the
    output against the oracle's attention over that plan on sampled rows.
      - order and offsets: the stable cluster order of the GPU's own assignment;
      - selection: each query cluster's kept set is a valid top-p prefix of the
        oracle's weights from the GPU's centroids (with routing: every cluster
        whose estimate clears tau is kept, and what is kept otherwise is a valid
        prefix);
      - value statistics (SVG-EAR): the oracle's means and dispersions;
      - tile CSR: bit-exact against the oracle's block mask of that plan on
        sampled query tiles (the first, the ragged last, random ones);
      - output: element-wise within the attention bars on sampled rows."""
    import svg_inputs as SI
    from video_dit_spatial_b200.layer import SemanticSparseLayer
    wl = SI.WORKLOADS[wname].replace(H=2, n_spatial=1)
    q, k, v = SI.make_qkv(wl)
    B, H, N, d, C, top_p = 1, 2, wl.N, wl.d, 256, 0.9
    layer = SemanticSparseLayer(B, H, N, d, Cq=C, Ck=C, iters=10, top_p=top_p, ear_tau=ear_tau)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    layer.forward(q.cuda(), k.cuda(), v.cuda(), o)
    torch.cuda.synchronize()
    scale = layer.scale
    got = to_f64(o)
    sel_all = _unpack_sel(layer.sel, C)
    rp, ci, nqb = layer.row_ptr.cpu().numpy(), layer.col_idx.cpu().numpy(), layer.nqb
    rng = np.random.default_rng(77 if ear_tau is None else 78)
    for h in range(H):
        qn, kn, vn = to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h])
        plan = {}
        for name in ("q", "k"):
            a = getattr(layer, "assign_" + name)[h].cpu().numpy()
            order = getattr(layer, "order_" + name)[h].cpu().numpy()
            offs = getattr(layer, "offsets_" + name)[h].cpu().numpy()
            want_order, want_offs = S2.cluster_permutation(a, C)
            assert np.array_equal(order, want_order) and np.array_equal(offs, want_offs), name
            plan[name] = (order, offs)
        (oq_, offq), (ok_, offk) = plan["q"], plan["k"]
        cq = layer.cq[h].cpu().numpy().astype(np.float64)
        ck = layer.ck[h].cpu().numpy().astype(np.float64)
        sizes = np.diff(offk)
        w = S2.selection_weights(cq, ck, sizes, scale)
        sel = sel_all[h]
        if ear_tau is None:
            for a in range(C):
                if offq[a + 1] > offq[a]:
                    assert _selection_valid(w[a], sizes, sel[a], top_p), f"head {h} cluster {a}"
        else:
            vbar = layer.vbar[h].cpu().numpy().astype(np.float64)
            disp = layer.disp[h].cpu().numpy().astype(np.float64)
            want_vbar, want_disp = S2.cluster_value_stats(vn, ok_, offk)
            np.testing.assert_allclose(vbar, want_vbar, rtol=1e-4, atol=1e-5)
            np.testing.assert_allclose(disp, want_disp, rtol=1e-4, atol=1e-5)
            est = w * disp[None, :]
            must = (est > ear_tau * (1 + 1e-4)) & (sizes > 0)[None, :]
            may = est > ear_tau * (1 - 1e-4)
            routed_only = 0
            for a in range(C):
                if offq[a + 1] <= offq[a]:
                    continue
                assert not np.any(must[a] & ~sel[a]), f"head {h} cluster {a}: a routed pair is missing"
                # what is kept beyond the routable clusters is a top-p prefix
                base = sel[a] & ~may[a]
                live = sizes > 0
                out = live & ~sel[a]
                if np.any(base):
                    assert w[a][base].min() >= (w[a][out].max() if np.any(out) else -1) - 1e-5
                    assert w[a][base].sum() - w[a][base].min() < top_p + 1e-5
                assert w[a][sel[a] & live].sum() >= top_p - 1e-5
                routed_only += int(np.sum(sel[a] & may[a] & ~must[a]))
        # tile CSR on sampled query tiles, and the output on sampled rows
        pos = np.unique(np.concatenate([np.arange(4), np.arange(N - 4, N),
                                        rng.choice(N, 40, replace=False)]))
        tiles = np.unique(np.concatenate([pos // 128, rng.choice(nqb, 12, replace=False)]))
        bm = S2.semantic_block_mask(offq, offk, sel, 128, 128, tiles=tiles)
        for r in tiles:
            row = h * nqb + r
            assert np.array_equal(ci[rp[row]:rp[row + 1]], np.nonzero(bm[r])[0]), (h, r)
        rows = oq_[pos]
        if ear_tau is None:
            want, _ = S2.semantic_attention_rows(qn, kn, vn, oq_, ok_, bm, 128, 128, scale, rows)
        else:
            want = S2.ear_attention_rows(qn, kn, vn, oq_, ok_, offk, ck, vbar, bm, 128, 128,
                                         scale, rows)
        density = float(np.diff(rp[h * nqb:(h + 1) * nqb + 1]).sum()) / (nqb * layer.nkb)
        label = f"{'ear' if ear_tau else 'svg2'} d{d} head {h}"
        print(f"SVG2-FULL {label}: tile density {density:.3f}, "
              f"{len(tiles)} tiles and {len(rows)} rows checked")
        assert_close(got[0, h][rows], want, f"SVG2 full size {label}")
    status_clean()
