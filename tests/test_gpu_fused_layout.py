"""GPU parity of the fused layout path.

The layout transformation of the Sparse VideoGen abstract happens inside the
attention kernel: temporal heads gather their query rows (and, in the
"gathered" layout, their key/value rows) in position-major order straight from
the frame-major tensors (TMA row gathers) and store each output row at its
frame-major place. The tile contents and the arithmetic are those of the
explicit path (permute -> attention -> unpermute), so the outputs must be
identical bit for bit; the fp64 oracle then bounds both.
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


def _layers(svg, g, layout, n_samples=16):
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    fused = SparseVideoGenLayer(g, n_samples, layout=layout)
    explicit = SparseVideoGenLayer(g, n_samples, layout="explicit")
    for layer in (fused, explicit):
        layer.build_masks()
    return fused, explicit


def _run_both(svg, g, q, k, v, labels, layout, with_lse=True):
    """(o_fused, o_explicit, lse_fused, lse_explicit) on the device."""
    B, H, N = g.B, g.H, g.N
    fused, explicit = _layers(svg, g, layout)
    outs = []
    for layer in (fused, explicit):
        layer.labels.copy_(labels)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, N), float("nan"), device="cuda") if with_lse else None
        layer.attend(q, k, v, o, lse=lse)
        outs.append((o, lse))
    torch.cuda.synchronize()
    return outs[0][0], outs[1][0], outs[0][1], outs[1][1]


def _bits(t):
    return t.contiguous().view(torch.int16) if t.dtype == torch.bfloat16 else \
        t.contiguous().view(torch.int32)


# T, P, L, d, bk, s, w, B, H  (block_q = 128: the paired kernel)
CASES = [
    (5, 100, 37, 128, 128, 1, 10, 1, 3),   # T does not divide 128; text rows
    (3, 200, 50, 64, 128, 0, 16, 2, 2),    # batch of two
    (6, 90, 20, 128, 64, 1, 8, 1, 2),      # 64-key blocks
    (16, 256, 64, 128, 128, 2, 32, 1, 2),
    (4, 64, 0, 64, 128, 1, 4, 1, 2),       # N = 256: whole blocks, no text
    (1, 300, 20, 128, 128, 0, 8, 1, 2),    # T = 1: the layout map is the identity
    (40, 1, 9, 64, 64, 1, 0, 1, 2),        # P = 1: the identity again
    (7, 33, 0, 128, 128, 2, 5, 1, 2),      # N = 231: the pair's second tile is ragged
    (3, 40, 0, 64, 64, 0, 2, 1, 2),        # N = 120: one ragged query block
    (33, 36, 7, 128, 128, 2, 3, 1, 2),     # the HunyuanVideo frame count, small frames
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}P{}L{}d{}bk{}".format(*c[:5]))
@pytest.mark.parametrize("labels_kind", ["alternating", "all_temporal"])
@pytest.mark.parametrize("layout", ["fused", "gathered"])
def test_fused_equals_explicit_bitwise_and_oracle(svg, case, labels_kind, layout):
    T, P, L, d, bk, s, w, B, H = case
    N = T * P + L
    g = svg.Geom(B, H, T, P, L, d, 128, bk, s, w, 1.0 / np.sqrt(d))
    q, k, v = (rand_bf16((B, H, N, d), seed=hash(case) % 9973 + i).cuda() for i in range(3))
    lab = [(i % 2) for i in range(B * H)] if labels_kind == "alternating" else [1] * (B * H)
    labels = torch.tensor(lab, dtype=torch.int8)
    o_f, o_e, lse_f, lse_e = _run_both(svg, g, q, k, v, labels, layout)
    assert torch.equal(_bits(o_f), _bits(o_e)), "fused and explicit outputs differ"
    # lse: frame-major rows on the fused path, each head's own layout otherwise
    pi = torch.from_numpy(O.permutation(T, P, L)).cuda()
    for bh in range(B * H):
        b, h = divmod(bh, H)
        want = lse_e[b, h, pi] if lab[bh] == O.HEAD_TEMPORAL else lse_e[b, h]
        assert torch.equal(_bits(lse_f[b, h]), _bits(want)), f"lse of head {bh}"
    # and the fp64 oracle, every row
    qn, kn, vn = to_f64(q), to_f64(k), to_f64(v)
    got = to_f64(o_f)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        want, _ = O.layer_rows(qn[b, h], kn[b, h], vn[b, h], lab[bh], T, P, L, s, w, 128, bk,
                               1.0 / np.sqrt(d))
        assert_close(got[b, h], want, f"fused head {bh} label {lab[bh]}")
    status_clean()


FULL = [(SI.COGVIDEOX, "fused", True), (SI.HUNYUAN, "fused", True), (SI.LONG, "fused", True),
        (SI.sweep_workloads()[4], "fused", True), (SI.HUNYUAN, "gathered", True),
        (SI.HUNYUAN, "fused", False)]


@pytest.mark.parametrize("wl,layout,planted", FULL,
                         ids=lambda x: x if isinstance(x, str) else
                         (("planted" if x else "unstructured") if isinstance(x, bool) else x.name))
def test_fused_full_size(svg, wl, layout, planted):
    """The benchmark's workloads: fused == explicit bit for bit over every
    output element, and sampled rows of a few heads of each label against the
    oracle (planted inputs, and unstructured N(0, 1) ones)."""
    g = svg.Geom.from_workload(wl)
    q, k, v = SI.make_qkv(wl, planted=planted)
    kinds = SI.planted_head_kinds(wl)
    labels = torch.tensor(kinds * wl.B, dtype=torch.int8)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o_f, o_e, _, _ = _run_both(svg, g, qd, kd, vd, labels, layout, with_lse=False)
    assert torch.equal(_bits(o_f), _bits(o_e)), "fused and explicit outputs differ"
    del qd, kd, vd, o_e
    inv_pi = O.inverse_permutation(O.permutation(wl.T, wl.P, wl.n_text))
    sp = [h for h in range(wl.H) if kinds[h] == 0][:1]
    tp = [h for h in range(wl.H) if kinds[h] == 1][:2]
    b = wl.B - 1
    for h in sp + tp:
        rows = edge_rows(wl.N, wl.N_v, wl.block_q, 24, seed=31 + h,
                         layout_to_frame_major=inv_pi if kinds[h] == 1 else None)
        qn, kn, vn = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
        want, _ = O.layer_rows(qn, kn, vn, kinds[h], wl.T, wl.P, wl.n_text, wl.spatial_band,
                               wl.temporal_width, wl.block_q, wl.block_k, wl.scale, rows=rows)
        assert_close(to_f64(o_f[b, h, torch.from_numpy(rows)]), want, f"{wl.name} b{b} h{h}")
    status_clean()


def test_fused_layer_forward_matches_explicit_forward(svg):
    """The whole layer (profiling labels included) on both paths."""
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    wl = SI.TINY.replace(name="fwd", seed=3101, d=128, T=9, P=120, n_text=40, H=4,
                         n_spatial=2, n_samples_fixed=200, spatial_band=1, temporal_width=12,
                         block_q=128, block_k=128)
    g = svg.Geom.from_workload(wl)
    q, k, v = (t.cuda() for t in SI.make_qkv(wl))
    rows = SI.sample_rows(wl).cuda()
    outs = []
    for layout in ("fused", "explicit", "gathered"):
        layer = SparseVideoGenLayer(g, wl.n_samples, layout=layout)
        o = torch.empty_like(q)
        layer.forward(q, k, v, rows, o)
        torch.cuda.synchronize()
        outs.append((o, layer.labels.clone()))
    assert list(outs[0][1].cpu().numpy()) == SI.planted_head_kinds(wl)
    for o, labels in outs[1:]:
        assert torch.equal(outs[0][1], labels)
        assert torch.equal(_bits(outs[0][0]), _bits(o))
    status_clean()
