"""GPU parity of the block-mask builder and the layout transformation (bit-exact).

Block masks are compared with the oracle's brute-force OR over token pairs
(all rows for small geometries, sampled rows at the full workload sizes);
permutations with the oracle's gather, head by head.
"""
import numpy as np
import pytest
import torch

import oracle as O
import svg_inputs as SI
from gpu_util import rand_bf16, status_clean, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


SMALL_GEOMS = [
    # T, P, L, bq, bk, s, w
    (4, 64, 0, 64, 64, 1, 4),
    (5, 100, 37, 128, 128, 1, 10),
    (3, 7, 5, 64, 128, 0, 2),
    (9, 33, 200, 128, 64, 2, 5),
    (1, 300, 1, 64, 64, 0, 0),
    (40, 3, 0, 128, 128, 3, 1),
    (7, 129, 129, 64, 64, 1, 64),
    (6, 50, 10, 64, 64, 5, 49),     # s = T-1, w = P-1: both masks are every block
    (3, 40, 0, 128, 64, 7, 100),    # bands wider than the grid
]


def _build(svg, g, kind):
    from video_dit_spatial_b200.layer import BlockMaskCSR
    m = BlockMaskCSR(g, kind, "cuda")
    m.build(g)
    torch.cuda.synchronize()
    return m.row_ptr.cpu().numpy(), m.col_idx.cpu().numpy()[:m.nnz], m.nnz


@pytest.mark.parametrize("geo", SMALL_GEOMS)
def test_block_mask_csr_bit_exact_small(svg, geo):
    T, P, L, bq, bk, s, w = geo
    g = svg.Geom(1, 1, T, P, L, 64, bq, bk, s, w, 0.125)
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL, O.MASK_DENSE):
        rp, ci, nnz = _build(svg, g, kind)
        want_rp, want_ci = O.to_csr(O.block_mask(kind, T, P, L, s, w, bq, bk))
        assert np.array_equal(rp, want_rp), kind
        assert np.array_equal(ci, want_ci), kind
        assert nnz == want_rp[-1]
    status_clean()


@pytest.mark.parametrize("wl", [SI.TINY, SI.COGVIDEOX, SI.HUNYUAN, SI.LONG] + SI.sweep_workloads(),
                         ids=lambda w: w.name)
def test_block_mask_csr_bit_exact_workloads(svg, wl):
    g = svg.Geom.from_workload(wl)
    rng = np.random.default_rng(7)
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
        rp, ci, nnz = _build(svg, g, kind)
        nqb = g.n_qblocks
        assert rp[0] == 0 and rp[-1] == nnz and np.all(np.diff(rp) >= 1)
        rows = sorted({0, 1, nqb // 2, nqb - 2, nqb - 1, (wl.N_v - 1) // wl.block_q,
                       *rng.choice(nqb, size=min(12, nqb), replace=False).tolist()})
        rows = [r for r in rows if 0 <= r < nqb]
        want = O.block_mask_rows(kind, rows, wl.T, wl.P, wl.n_text, wl.spatial_band,
                                 wl.temporal_width, wl.block_q, wl.block_k)
        for n, r in enumerate(rows):
            got = ci[rp[r]:rp[r + 1]]
            assert np.array_equal(got, np.nonzero(want[n])[0]), (kind, r)
    status_clean()


def _labels(BH, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 2, (BH,), generator=g).to(torch.int8)


@pytest.mark.parametrize("T,P,L,d", [(4, 64, 0, 64), (5, 100, 37, 128), (3, 7, 5, 64),
                                     (1, 50, 3, 128), (6, 1, 2, 64), (33, 120, 16, 128)])
def test_permute_unpermute_bit_exact(svg, T, P, L, d):
    B, H = 2, 3
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, d, 64, 64, 0, 0, 0.1)
    x = rand_bf16((B, H, N, d), seed=T * 1000 + P)
    labels = _labels(B * H, seed=N)
    labels[0] = 1
    labels[1] = 0
    xd = x.cuda()
    sentinel = torch.full_like(xd, 7.0)
    out = sentinel.clone()
    svg.svg_permute(g, xd, out, labels.cuda())
    back = sentinel.clone()
    svg.svg_unpermute(g, out, back, labels.cuda())
    allh = torch.empty_like(xd)
    svg.svg_permute(g, xd, allh, None)
    torch.cuda.synchronize()
    xn = to_f64(x)
    want = O.permute(xn, T, P, L)
    o, b, a = to_f64(out), to_f64(back), to_f64(allh)
    for bh in range(B * H):
        bb, hh = divmod(bh, H)
        assert np.array_equal(a[bb, hh], want[bb, hh])
        if labels[bh] == 1:
            assert np.array_equal(o[bb, hh], want[bb, hh])
            assert np.array_equal(b[bb, hh], xn[bb, hh])
        else:
            assert np.all(o[bb, hh] == 7.0) and np.all(b[bb, hh] == 7.0)
    status_clean()


def test_permute_qkv_matches_single_permutes(svg):
    T, P, L, d = 5, 100, 37, 128
    B, H = 1, 4
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, d, 128, 128, 0, 0, 0.1)
    q, k, v = (rand_bf16((B, H, N, d), seed=s).cuda() for s in (1, 2, 3))
    labels = torch.tensor([1, 0, 1, 1], dtype=torch.int8, device="cuda")
    outs = [torch.zeros_like(q) for _ in range(3)]
    svg.svg_permute_qkv(g, q, k, v, *outs, labels)
    for x, o in zip((q, k, v), outs):
        ref = torch.zeros_like(x)
        svg.svg_permute(g, x, ref, labels)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    status_clean()


def test_permute_full_size_hunyuan(svg):
    wl = SI.HUNYUAN
    g = svg.Geom.from_workload(wl)
    x = rand_bf16((1, 4, wl.N, wl.d), seed=5)
    gg = svg.Geom(1, 4, wl.T, wl.P, wl.n_text, wl.d, 128, 128, 0, 0, wl.scale)
    labels = torch.tensor([1, 0, 1, 0], dtype=torch.int8)
    xd = x.cuda()
    out = torch.zeros_like(xd)
    svg.svg_permute(gg, xd, out, labels.cuda())
    back = torch.zeros_like(xd)
    svg.svg_unpermute(gg, out, back, labels.cuda())
    torch.cuda.synchronize()
    xn = to_f64(x)
    for h in (0, 2):
        assert np.array_equal(to_f64(out[0, h]), O.permute(xn[0, h], wl.T, wl.P, wl.n_text))
        assert np.array_equal(to_f64(back[0, h]), xn[0, h])
    assert torch.count_nonzero(out[0, 1].view(torch.int16)) == 0
    del g
    status_clean()
