"""GPU parity of the FP8 PV path: the e4m3 quantisation of V bit for bit, and
the block-sparse attention with an e4m3 PV product against the fp64 oracle.

The FP8 attention is the same block-sparse attention as the bf16 kernel's;
only the PV product's operands are rounded to E4M3 (P scaled by 2^6, V with
one scale per (head, channel)). It is held to an element-wise tolerance
derived from that rounding (gpu_util.fp8_reference): six standard deviations
of the error the rounding of P and V induces, plus the bf16 rounding of the
output. The log-sum-exp does not involve the PV product and keeps the bf16
path's 2e-3 bar.
"""
import numpy as np
import pytest
import torch

import oracle as O
import svg_inputs as SI
from gpu_util import assert_within, edge_rows, fp8_reference, rand_bf16, status_clean, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _fp8_codes_as_bytes(codes: np.ndarray) -> torch.Tensor:
    # exact E4M3 values, so the conversion only encodes them
    return torch.from_numpy(codes.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)


# T, P, L, bk, s, w, B, H (d = 128, block_q = 128)
CASES = [
    (5, 100, 37, 128, 1, 10, 1, 3),
    (3, 200, 50, 128, 0, 16, 2, 2),
    (6, 90, 20, 64, 1, 8, 1, 2),
    (16, 256, 64, 128, 2, 32, 1, 2),
    (7, 33, 0, 128, 2, 5, 1, 2),
    (1, 300, 20, 128, 0, 8, 1, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}P{}L{}bk{}".format(*c[:4]))
def test_quantize_v_bit_exact(svg, case):
    T, P, L, bk, s, w, B, H = case
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, 128, 128, bk, s, w, 1.0 / np.sqrt(128))
    v = rand_bf16((B, H, N, 128), seed=hash(case) % 7919, scale=1.7).cuda()
    v[0, 0, :, 3] = 0  # an all-zero channel
    labels = torch.tensor([i % 2 for i in range(B * H)], dtype=torch.int8, device="cuda")
    vp = torch.empty_like(v)
    svg.svg_permute(g, v, vp, labels)
    v8 = torch.full((B, H, N, 128), 0x55, dtype=torch.uint8, device="cuda")
    vs = torch.full((B * H * 128,), float("nan"), device="cuda")
    svg.svg_quantize_v_e4m3(g, v, vp, labels, v8, vs)
    torch.cuda.synchronize()
    vn = to_f64(v)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        src = O.permute(vn[b, h], T, P, L) if bh % 2 else vn[b, h]
        codes, scale = O.quantize_v_e4m3(src)
        assert torch.equal(v8[b, h].cpu(), _fp8_codes_as_bytes(codes)), f"codes of head {bh}"
        assert np.array_equal(vs[bh * 128:(bh + 1) * 128].cpu().numpy().view(np.int32),
                              scale.view(np.int32)), f"scales of head {bh}"
    status_clean()


def _layer(svg, g):
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    layer = SparseVideoGenLayer(g, 16, layout="explicit", pv="e4m3")
    layer.build_masks()
    return layer


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}P{}L{}bk{}".format(*c[:4]))
@pytest.mark.parametrize("kind", ["random", "planted"])
def test_fp8_attention_all_rows(svg, case, kind):
    T, P, L, bk, s, w, B, H = case
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, 128, 128, bk, s, w, 1.0 / np.sqrt(128))
    if kind == "random":
        q, k, v = (rand_bf16((B, H, N, 128), seed=hash(case) % 10007 + i) for i in range(3))
    else:
        wl = SI.Workload("t", B, H, 128, T, P, L, s, w, 128, bk, n_spatial=H // 2,
                         seed=hash(case) % 10007)
        q, k, v = SI.make_qkv(wl)
    labels = torch.tensor([(i + (N % 2)) % 2 for i in range(B * H)], dtype=torch.int8)
    layer = _layer(svg, g)
    layer.labels.copy_(labels)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    layer.attend(qd, kd, vd, o, lse=lse)
    torch.cuda.synchronize()
    got = to_f64(o)
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        lab = int(labels[bh])
        want, tol = fp8_reference(qn[b, h], kn[b, h], vn[b, h], lab, T, P, L, s, w, 128, bk,
                                  1.0 / np.sqrt(128), np.arange(N))
        assert_within(got[b, h], want, tol, f"{kind} head {bh} label {lab}")
        _, lse_w = O.layer_rows(qn[b, h], kn[b, h], vn[b, h], lab, T, P, L, s, w, 128, bk,
                                1.0 / np.sqrt(128))
        if lab == O.HEAD_TEMPORAL:
            lse_w = O.permute(lse_w[:, None], T, P, L)[:, 0]
        np.testing.assert_allclose(lse.cpu().numpy()[b, h], lse_w, atol=2e-3, rtol=0)
    status_clean()


@pytest.mark.parametrize("planted", [True, False], ids=["planted", "unstructured"])
def test_fp8_attention_full_size_sampled_rows(svg, planted):
    """The HunyuanVideo-shaped layer through the benchmark's FP8 launch; the
    oracle checks sampled rows of two heads of each label."""
    wl = SI.HUNYUAN
    g = svg.Geom.from_workload(wl)
    q, k, v = SI.make_qkv(wl, planted=planted)
    kinds = SI.planted_head_kinds(wl)
    layer = _layer(svg, g)
    layer.labels.copy_(torch.tensor(kinds * wl.B, dtype=torch.int8))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    layer.attend(qd, kd, vd, o)
    torch.cuda.synchronize()
    del qd, kd, vd
    inv_pi = O.inverse_permutation(O.permutation(wl.T, wl.P, wl.n_text))
    for h in [h for h in range(wl.H) if kinds[h] == 0][:2] + \
            [h for h in range(wl.H) if kinds[h] == 1][:2]:
        rows = edge_rows(wl.N, wl.N_v, wl.block_q, 24, seed=51 + h,
                         layout_to_frame_major=inv_pi if kinds[h] == 1 else None)
        qn, kn, vn = to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h])
        want, tol = fp8_reference(qn, kn, vn, kinds[h], wl.T, wl.P, wl.n_text, wl.spatial_band,
                                  wl.temporal_width, wl.block_q, wl.block_k, wl.scale, rows)
        assert_within(to_f64(o[0, h, torch.from_numpy(rows)]), want, tol,
                      f"{wl.name} {'planted' if planted else 'unstructured'} h{h} "
                      f"label {kinds[h]}")
    status_clean()


def test_fp8_rejects_unsupported_shapes(svg):
    g = svg.Geom(1, 1, 4, 64, 0, 64, 128, 128, 1, 4, 0.125)  # d = 64
    x = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device="cuda")
    v8 = torch.zeros((1, 1, 256, 64), dtype=torch.uint8, device="cuda")
    vs = torch.zeros(64, device="cuda")
    with pytest.raises(svg.SvgError) as ei:
        svg.svg_quantize_v_e4m3(g, x, None, None, v8, vs)
    assert ei.value.status == svg.SVG_ERR_UNSUPPORTED
