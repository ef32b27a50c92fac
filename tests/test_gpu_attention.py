"""GPU parity of block-sparse attention and the whole layer against the fp64 oracle.

Tolerance (bf16 in, fp32 accumulate, bf16 out): max-abs 2e-2 and mean-abs 2e-3
per compared tensor; log-sum-exp within 2e-3 absolute.
"""
import numpy as np
import pytest
import torch

import oracle as O
import svg_inputs as SI
from gpu_util import assert_close, edge_rows, rand_bf16, status_clean, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _layer(svg, g, n_samples=16):
    # the explicit layout path (permute -> attention -> unpermute); the fused
    # path is compared with it in test_gpu_fused_layout.py
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    return SparseVideoGenLayer(g, n_samples, layout="explicit")


# T, P, L, d, bq, bk, s, w, B, H
CASES = [
    (4, 64, 0, 64, 64, 64, 1, 4, 1, 2),
    (5, 100, 37, 128, 128, 128, 1, 10, 1, 3),
    (3, 200, 50, 64, 128, 128, 0, 16, 2, 2),
    (6, 90, 20, 128, 128, 64, 1, 8, 1, 2),
    (4, 150, 3, 64, 64, 128, 1, 30, 1, 2),
    (16, 256, 64, 128, 128, 128, 2, 32, 1, 2),
    (2, 61, 0, 128, 64, 64, 0, 3, 1, 2),
]


def _inputs(case, kind, seed):
    T, P, L, d, bq, bk, s, w, B, H = case
    N = T * P + L
    if kind == "random":
        return tuple(rand_bf16((B, H, N, d), seed=seed + i) for i in range(3))
    wl = SI.Workload("t", B, H, d, T, P, L, s, w, bq, bk, n_spatial=H // 2, seed=seed)
    return SI.make_qkv(wl)


def _oracle_head(qn, kn, vn, label, case, rows=None):
    T, P, L, d, bq, bk, s, w, B, H = case
    return O.layer_rows(qn, kn, vn, label, T, P, L, s, w, bq, bk, 1.0 / np.sqrt(d), rows=rows)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}P{}L{}d{}bq{}bk{}".format(*c[:6]))
@pytest.mark.parametrize("kind", ["random", "planted"])
def test_sparse_attention_all_rows(svg, case, kind):
    T, P, L, d, bq, bk, s, w, B, H = case
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, d, bq, bk, s, w, 1.0 / np.sqrt(d))
    q, k, v = _inputs(case, kind, seed=hash(case) % 10000)
    labels = torch.tensor([(i + (N % 2)) % 2 for i in range(B * H)], dtype=torch.int8)
    layer = _layer(svg, g)
    layer.build_masks()
    layer.labels.copy_(labels)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qd, float("nan"))
    lse_p = torch.full((B, H, N), float("nan"), device="cuda")
    # lse is reported in each head's own layout
    layer.attend(qd, kd, vd, o, lse=lse_p)
    torch.cuda.synchronize()
    got = to_f64(o)
    lse_g = lse_p.cpu().numpy()
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        want, lse_w = _oracle_head(qn[b, h], kn[b, h], vn[b, h], int(labels[bh]), case)
        assert_close(got[b, h], want, f"head {bh} label {int(labels[bh])}")
        if int(labels[bh]) == O.HEAD_TEMPORAL:
            lse_w = O.permute(lse_w[:, None], T, P, L)[:, 0]
        np.testing.assert_allclose(lse_g[b, h], lse_w, atol=2e-3, rtol=0)
    status_clean()


@pytest.mark.parametrize("case", CASES[:3] + CASES[5:6], ids=lambda c: "T{}P{}L{}d{}".format(*c[:4]))
def test_dense_baseline_is_full_attention(svg, case):
    T, P, L, d, bq, bk, s, w, B, H = case
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, d, bq, bk, s, w, 1.0 / np.sqrt(d))
    q, k, v = _inputs(case, "random", seed=77)
    layer = _layer(svg, g)
    o = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    layer.dense(q.cuda(), k.cuda(), v.cuda(), o)
    torch.cuda.synchronize()
    got = to_f64(o)
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    for b in range(B):
        for h in range(H):
            want, _ = O.masked_attention_rows(qn[b, h], kn[b, h], vn[b, h], np.arange(N), None,
                                              1.0 / np.sqrt(d))
            assert_close(got[b, h], want, f"dense b{b} h{h}")
    status_clean()


@pytest.mark.parametrize("T,P,L,d,bq,bk", [(6, 50, 10, 64, 64, 64), (5, 100, 37, 128, 128, 128),
                                           (3, 40, 0, 128, 128, 64)])
def test_full_width_bands_equal_the_dense_run(svg, T, P, L, d, bq, bk):
    # With s >= T-1 and w >= P-1 both masks list every key block: the spatial CSR is the
    # dense one, so spatial heads must give the dense run's bits, and temporal heads
    # (position-major, the same keys in another order) the oracle's full attention.
    N = T * P + L
    g = svg.Geom(1, 2, T, P, L, d, bq, bk, T - 1, P - 1, 1.0 / np.sqrt(d))
    q, k, v = (rand_bf16((1, 2, N, d), seed=900 + i) for i in range(3))
    layer = _layer(svg, g)
    layer.build_masks()
    layer.labels.copy_(torch.tensor([0, 1], dtype=torch.int8))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    od = torch.empty_like(qd)
    layer.attend(qd, kd, vd, o)
    layer.dense(qd, kd, vd, od)
    torch.cuda.synchronize()
    assert torch.equal(layer.masks[0].row_ptr, layer.dense_mask.row_ptr)
    assert torch.equal(o[0, 0].view(torch.int16), od[0, 0].view(torch.int16))
    want, _ = O.masked_attention_rows(to_f64(q[0, 1]), to_f64(k[0, 1]), to_f64(v[0, 1]),
                                      np.arange(N), None, 1.0 / np.sqrt(d))
    assert_close(to_f64(o[0, 1]), want, "temporal head, full-width band")
    status_clean()


def test_empty_csr_rows_give_zero(svg):
    T, P, L, d = 2, 128, 0, 128
    N = T * P
    g = svg.Geom(1, 1, T, P, L, d, 128, 128, 0, 0, 1.0 / np.sqrt(d))
    q, k, v = (rand_bf16((1, 1, N, d), seed=i).cuda() for i in range(3))
    row_ptr = torch.tensor([0, 0, 1], dtype=torch.int32, device="cuda")  # row 0 empty
    col_idx = torch.tensor([0], dtype=torch.int32, device="cuda")
    o = torch.full_like(q, 3.0)
    lse = torch.zeros((1, 1, N), device="cuda")
    svg.svg_sparse_attention(g, q, k, v, None, None, None, None, row_ptr, col_idx, None, None,
                             o, None, lse)
    torch.cuda.synchronize()
    assert torch.count_nonzero(o[0, 0, :128].float()) == 0
    assert torch.all(torch.isinf(lse[0, 0, :128]))
    want, _ = O.masked_attention_rows(to_f64(q[0, 0]), to_f64(k[0, 0]), to_f64(v[0, 0]),
                                      np.arange(128, N), lambda rr: np.repeat(
                                          (np.arange(N) < 128)[None], len(rr), 0), 1 / np.sqrt(d))
    assert_close(to_f64(o[0, 0, 128:]), want, "row with one block")
    status_clean()


# planted inputs for every workload, plus unstructured ones (Q, K, V ~ N(0, 1):
# diffuse attention, every computed block matters) at the two model shapes
FULL = [(w, True) for w in [SI.COGVIDEOX, SI.HUNYUAN, SI.LONG] + SI.sweep_workloads()] + \
    [(SI.COGVIDEOX, False), (SI.HUNYUAN, False)]


@pytest.mark.parametrize("wl,planted", FULL,
                         ids=lambda x: x if not isinstance(x, bool) else
                         ("planted" if x else "unstructured"))
def test_sparse_attention_full_size_sampled_rows(svg, wl, planted):
    """The full workload through the same launch as the benchmark; the oracle
    checks sampled rows (edges + random) of a few heads of each label."""
    g = svg.Geom.from_workload(wl)
    q, k, v = SI.make_qkv(wl, planted=planted)
    kinds = SI.planted_head_kinds(wl)
    labels = torch.tensor(kinds * wl.B, dtype=torch.int8)
    layer = _layer(svg, g, n_samples=wl.n_samples)
    layer.build_masks()
    layer.labels.copy_(labels)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    layer.attend(qd, kd, vd, o)
    torch.cuda.synchronize()
    del qd, kd, vd
    sp = [h for h in range(wl.H) if kinds[h] == 0][:2]
    tp = [h for h in range(wl.H) if kinds[h] == 1][:2]
    inv_pi = O.inverse_permutation(O.permutation(wl.T, wl.P, wl.n_text))
    for b in range(wl.B):
        for h in sp + tp:
            rows = edge_rows(wl.N, wl.N_v, wl.block_q, 40, seed=11 + h,
                             layout_to_frame_major=inv_pi if kinds[h] == 1 else None)
            qn, kn, vn = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
            want, _ = O.layer_rows(qn, kn, vn, kinds[h], wl.T, wl.P, wl.n_text, wl.spatial_band,
                                   wl.temporal_width, wl.block_q, wl.block_k, wl.scale, rows=rows)
            assert_close(to_f64(o[b, h, torch.from_numpy(rows)]), want,
                         f"{wl.name} {'planted' if planted else 'unstructured'} b{b} h{h} "
                         f"label {kinds[h]}")
    status_clean()
