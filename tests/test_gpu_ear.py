"""GPU parity of SVG-EAR (error-aware routing and centroid compensation) against
the fp64 oracle (oracle/svg2_oracle.py), step by step on shared seeded inputs.

The compensated output is an attention over every key (exact ones plus the
centroid stand-ins of the rest) in bf16-in / fp32-accumulate arithmetic, so it
is held to the same bars as the other attention outputs; the cluster
statistics are fp32 means of bf16 values; routing decisions follow the
selection's near-tie rule.
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


def _plans(rng, BH, N, Cq, Ck, density):
    plans = []
    for _ in range(BH):
        aq, ak = rng.integers(0, Cq, N), rng.integers(0, Ck, N)
        oq_, offq = S2.cluster_permutation(aq, Cq)
        ok_, offk = S2.cluster_permutation(ak, Ck)
        sel = rng.random((Cq, Ck)) < density
        sel[np.arange(Cq), rng.integers(0, Ck, Cq)] = True
        plans.append((oq_, offq, ok_, offk, sel))
    return plans


def _dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).cuda()


def _pack(sel_list, Ck):
    words = (Ck + 31) // 32
    packed = np.zeros((len(sel_list), sel_list[0].shape[0], words), dtype=np.uint32)
    for h, sel in enumerate(sel_list):
        for b in range(Ck):
            packed[h, :, b // 32] |= sel[:, b].astype(np.uint32) << np.uint32(b % 32)
    return torch.from_numpy(packed.view(np.int32)).cuda()


def test_cluster_value_stats(svg):
    BH, N, d, Ck = 3, 2000, 128, 48
    rng = np.random.default_rng(31)
    v = rand_bf16((BH, N, d), seed=31)
    plans = _plans(rng, BH, N, 8, Ck, 0.2)
    offk0 = plans[0][3]
    offk0[6] = offk0[5]  # cluster 5 of head 0 empty (cluster 6 takes its positions)
    order_k = _dev_i32(np.stack([p[2] for p in plans]))
    offs_k = _dev_i32(np.stack([p[3] for p in plans]))
    vbar = torch.full((BH, Ck, d), float("nan"), device="cuda")
    disp = torch.full((BH, Ck), float("nan"), device="cuda")
    svg.svg2_cluster_value_stats(BH, N, d, Ck, v.cuda(), order_k, offs_k, vbar, disp)
    torch.cuda.synchronize()
    vn = to_f64(v)
    for h in range(BH):
        want_v, want_d = S2.cluster_value_stats(vn[h], plans[h][2], plans[h][3])
        np.testing.assert_allclose(vbar[h].cpu().numpy(), want_v, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(disp[h].cpu().numpy(), want_d, rtol=1e-5, atol=1e-6)
    status_clean()


@pytest.mark.parametrize("tau", [0.005, 0.02])
def test_selection_with_error_aware_routing(svg, tau):
    BH, d, Cq, Ck, top_p, scale = 2, 128, 24, 64, 0.7, 1.0 / np.sqrt(128)
    rng = np.random.default_rng(int(tau * 1e4))
    cq = (rng.standard_normal((BH, Cq, d)) * 1.5).astype(np.float32)
    ck = (rng.standard_normal((BH, Ck, d)) * 1.5).astype(np.float32)
    sizes = rng.integers(0, 300, (BH, Ck))
    offs = np.concatenate([np.zeros((BH, 1), np.int64), np.cumsum(sizes, 1)], 1)
    disp = rng.uniform(0.2, 2.0, (BH, Ck)).astype(np.float32)
    sel = torch.empty((BH, Cq, (Ck + 31) // 32), dtype=torch.int32, device="cuda")
    svg.svg2_select_clusters(BH, d, Cq, Ck, scale, top_p, torch.from_numpy(cq).cuda(),
                             torch.from_numpy(ck).cuda(), _dev_i32(offs), sel,
                             disp=torch.from_numpy(disp).cuda(), tau=tau)
    torch.cuda.synchronize()
    bits = sel.cpu().numpy().view(np.uint32)
    got = ((bits[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(BH, Cq, -1)[..., :Ck]
    routed_any = 0
    for h in range(BH):
        c64q, c64k = cq[h].astype(np.float64), ck[h].astype(np.float64)
        base = S2.select_clusters(c64q, c64k, sizes[h], scale, top_p)
        w = S2.selection_weights(c64q, c64k, sizes[h], scale)
        want = S2.route_clusters(base, w, disp[h].astype(np.float64), tau)
        est = w * disp[h][None, :]
        routed_any += int(np.sum(want & ~base))
        # decisions far from both boundaries must match exactly
        near = np.abs(est - tau) <= 1e-5 * np.maximum(tau, est)
        diff = (got[h].astype(bool) != want) & ~near
        assert not np.any(diff & ~base & (est > tau + 1e-5)), "a routed pair is missing"
        assert np.mean(got[h].astype(bool) == want) > 0.98
    assert routed_any > 0  # the case exercises routing
    status_clean()


@pytest.mark.parametrize("N,d,Ck,density", [(1500, 128, 32, 0.2), (2600, 64, 48, 0.1),
                                            (1000, 128, 16, 1.0)])
def test_ear_compensation_matches_oracle(svg, N, d, Ck, density):
    """Seeded plans drive both sides: gather, tile CSR, attention with its
    log-sum-exp, compensation and scatter on the GPU against the oracle's
    compensated attention (exact tiles + bf16 centroid stand-ins)."""
    BH, Cq, bk, scale = 2, 8, 128, 1.0 / np.sqrt(d)
    rng = np.random.default_rng(N + Ck)
    q, k, v = (rand_bf16((BH, N, d), seed=N + 7 * i) for i in range(3))
    plans = _plans(rng, BH, N, Cq, Ck, density)
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    kbar = np.zeros((BH, Ck, d))
    vbar = np.zeros((BH, Ck, d))
    for h in range(BH):
        ok_, offk = plans[h][2], plans[h][3]
        for b in range(Ck):
            mem = ok_[offk[b]:offk[b + 1]]
            if mem.size:
                kbar[h, b] = kn[h, mem].mean(axis=0)
        vbar[h] = S2.cluster_value_stats(vn[h], ok_, offk)[0]
    order_q = _dev_i32(np.stack([p[0] for p in plans]))
    offs_q = _dev_i32(np.stack([p[1] for p in plans]))
    order_k = _dev_i32(np.stack([p[2] for p in plans]))
    offs_k = _dev_i32(np.stack([p[3] for p in plans]))
    nqb, nkb = -(-N // 128), -(-N // bk)
    row_ptr = torch.empty(BH * nqb + 1, dtype=torch.int32, device="cuda")
    col_idx = torch.empty(BH * nqb * nkb, dtype=torch.int32, device="cuda")
    counts = torch.empty(BH * nqb, dtype=torch.int32, device="cuda")
    svg.svg2_build_tile_csr(BH, N, Cq, Ck, 128, bk, offs_q, offs_k,
                            _pack([p[4] for p in plans], Ck), row_ptr, col_idx, counts)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    qs, ks, vs, os_, o = (torch.empty_like(qd) for _ in range(5))
    lse = torch.empty((BH, N), device="cuda")
    svg.svg2_gather_rows(BH, N, d, qd, order_q, qs)
    svg.svg2_gather_rows(BH, N, d, kd, order_k, ks)
    svg.svg2_gather_rows(BH, N, d, vd, order_k, vs)
    svg.svg2_sparse_attention(BH, N, d, bk, scale, qs, ks, vs, row_ptr, col_idx, os_, lse)
    ws = torch.empty(svg.svg2_ear_workspace_bytes(BH, d, Ck) // 4 + 64, device="cuda")
    svg.svg2_ear_compensate(BH, N, d, Ck, bk, scale, qs,
                            torch.from_numpy(kbar.astype(np.float32)).cuda(),
                            torch.from_numpy(vbar.astype(np.float32)).cuda(), offs_k, row_ptr,
                            col_idx, os_, lse, ws)
    svg.svg2_scatter_rows(BH, N, d, os_, order_q, o)
    torch.cuda.synchronize()
    got = to_f64(o)
    for h in range(BH):
        oq_, offq, ok_, offk, sel = plans[h]
        bm = S2.semantic_block_mask(offq, offk, sel, 128, bk)
        rows = np.arange(N)
        want = S2.ear_attention_rows(qn[h], kn[h], vn[h], oq_, ok_, offk,
                                     kbar[h].astype(np.float32).astype(np.float64),
                                     vbar[h].astype(np.float32).astype(np.float64), bm, 128, bk,
                                     scale, rows)
        assert_close(got[h], want, f"EAR compensation N{N} d{d} Ck{Ck} head {h}")
    status_clean()


def test_ear_layer_end_to_end_on_planted_frames(svg):
    """SemanticSparseLayer with SVG-EAR on planted per-frame heads (one cluster
    per frame, unambiguous plans): plan and output equal the oracle's."""
    from video_dit_spatial_b200.layer import SemanticSparseLayer
    B, H, T, P, d, tau = 1, 2, 16, 200, 128, 0.01
    N = T * P
    rng = np.random.default_rng(41)
    e = np.repeat(rng.standard_normal((H, T, d)) * 2.0, P, axis=1)
    qkv = [0.5 * rng.standard_normal((H, N, d)) + e, 0.5 * rng.standard_normal((H, N, d)) + e,
           rng.standard_normal((H, N, d))]
    q, k, v = (torch.from_numpy(O.to_bf16_bits(x).view(np.int16)).view(torch.bfloat16)
               .reshape(B, H, N, d) for x in qkv)
    layer = SemanticSparseLayer(B, H, N, d, Cq=T, Ck=T, iters=4, top_p=0.9, ear_tau=tau)
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
        vbar, disp = S2.cluster_value_stats(vn, ok_, offk)
        base = S2.select_clusters(cq, ck, np.diff(offk), scale, 0.9)
        w = S2.selection_weights(cq, ck, np.diff(offk), scale)
        sel = S2.route_clusters(base, w, disp, tau)
        bm = S2.semantic_block_mask(offq, offk, sel, 128, 128)
        rp, ci, nqb = layer.row_ptr.cpu().numpy(), layer.col_idx.cpu().numpy(), layer.nqb
        for r in range(nqb):
            row = h * nqb + r
            assert np.array_equal(ci[rp[row]:rp[row + 1]], np.nonzero(bm[r])[0]), (h, r)
        want = S2.ear_attention_rows(qn, kn, vn, oq_, ok_, offk, ck, vbar, bm, 128, 128, scale,
                                     np.arange(N))
        assert_close(got[0, h], want, f"EAR layer head {h}")
    status_clean()


def test_ear_compensation_many_short_heads(svg):
    """96 heads of 3 query tiles each (288 tiles over at most one CTA per SM):
    the persistent compensation kernel moves between heads inside most CTAs,
    reloading the centroids each time; sampled rows of every head against the
    oracle."""
    BH, N, d, Ck, Cq, bk, scale = 96, 300, 64, 16, 4, 128, 1.0 / 8.0
    rng = np.random.default_rng(96)
    q, k, v = (rand_bf16((BH, N, d), seed=960 + i) for i in range(3))
    plans = _plans(rng, BH, N, Cq, Ck, 0.3)
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    kbar = np.zeros((BH, Ck, d))
    vbar = np.zeros((BH, Ck, d))
    for h in range(BH):
        ok_, offk = plans[h][2], plans[h][3]
        for b in range(Ck):
            mem = ok_[offk[b]:offk[b + 1]]
            if mem.size:
                kbar[h, b] = kn[h, mem].mean(axis=0)
        vbar[h] = S2.cluster_value_stats(vn[h], ok_, offk)[0]
    order_q = _dev_i32(np.stack([p[0] for p in plans]))
    offs_q = _dev_i32(np.stack([p[1] for p in plans]))
    order_k = _dev_i32(np.stack([p[2] for p in plans]))
    offs_k = _dev_i32(np.stack([p[3] for p in plans]))
    nqb, nkb = -(-N // 128), -(-N // bk)
    row_ptr = torch.empty(BH * nqb + 1, dtype=torch.int32, device="cuda")
    col_idx = torch.empty(BH * nqb * nkb, dtype=torch.int32, device="cuda")
    counts = torch.empty(BH * nqb, dtype=torch.int32, device="cuda")
    svg.svg2_build_tile_csr(BH, N, Cq, Ck, 128, bk, offs_q, offs_k,
                            _pack([p[4] for p in plans], Ck), row_ptr, col_idx, counts)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    qs, ks, vs, os_, o = (torch.empty_like(qd) for _ in range(5))
    lse = torch.empty((BH, N), device="cuda")
    svg.svg2_gather_rows(BH, N, d, qd, order_q, qs)
    svg.svg2_gather_rows(BH, N, d, kd, order_k, ks)
    svg.svg2_gather_rows(BH, N, d, vd, order_k, vs)
    svg.svg2_sparse_attention(BH, N, d, bk, scale, qs, ks, vs, row_ptr, col_idx, os_, lse)
    ws = torch.empty(svg.svg2_ear_workspace_bytes(BH, d, Ck) // 4 + 64, device="cuda")
    svg.svg2_ear_compensate(BH, N, d, Ck, bk, scale, qs,
                            torch.from_numpy(kbar.astype(np.float32)).cuda(),
                            torch.from_numpy(vbar.astype(np.float32)).cuda(), offs_k, row_ptr,
                            col_idx, os_, lse, ws)
    svg.svg2_scatter_rows(BH, N, d, os_, order_q, o)
    torch.cuda.synchronize()
    got = to_f64(o)
    for h in range(BH):
        oq_, offq, ok_, offk, sel = plans[h]
        bm = S2.semantic_block_mask(offq, offk, sel, 128, bk)
        rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 10, replace=False)]))
        want = S2.ear_attention_rows(qn[h], kn[h], vn[h], oq_, ok_, offk,
                                     kbar[h].astype(np.float32).astype(np.float64),
                                     vbar[h].astype(np.float32).astype(np.float64), bm, 128, bk,
                                     scale, rows)
        assert_close(got[h][rows], want, f"EAR many heads head {h}")
    status_clean()
