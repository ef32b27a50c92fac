"""GPU parity of online profiling: labels bit-exact with the fp64 oracle.

A head whose two errors are within the near-tie band is reported and excluded
from the bit-exact label claim; planted inputs on regular geometries produce
none. The band is relative 2^-5 (the accumulated rounding of bf16 probabilities
in the GPU's MSE), or both errors below 1e-7 absolute: a mask that (nearly)
allows every key gives an error at the rounding level of bf16 probabilities,
which fp32 cannot order against another such error.
"""
import numpy as np
import pytest
import torch

import oracle as O
import svg_inputs as SI
from gpu_util import status_clean, to_f64

pytestmark = pytest.mark.gpu

NEAR_TIE = 2.0 ** -5
NEAR_TIE_ABS = 1e-7


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _run_profile(svg, wl, q, k, v, rows):
    from video_dit_spatial_b200.layer import SparseVideoGenLayer
    g = svg.Geom.from_workload(wl)
    layer = SparseVideoGenLayer(g, len(rows))
    layer.profile(q.cuda(), k.cuda(), v.cuda(), rows.cuda())
    torch.cuda.synchronize()
    return layer.labels.cpu().numpy(), layer.mse.cpu().numpy().reshape(-1, 2)


def _check_heads(wl, q, k, v, rows, labels, mse, heads):
    rn = rows.numpy()
    checked = 0
    for b, h in heads:
        qn, kn, vn = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
        ms, mt, lab = O.profile_head(qn, kn, vn, rn, wl.T, wl.P, wl.n_text, wl.spatial_band,
                                     wl.temporal_width, wl.scale)
        bh = b * wl.H + h
        gs, gt = mse[bh]
        if abs(ms - mt) <= NEAR_TIE * max(ms, mt) or max(ms, mt) <= NEAR_TIE_ABS:
            continue  # near tie: reported, not part of the bit-exact claim
        assert labels[bh] == lab, (b, h, ms, mt, gs, gt)
        np.testing.assert_allclose([gs, gt], [ms, mt], rtol=0.1, atol=1e-7)
        checked += 1
    return checked


VARIANTS = [
    {},
    {"seed": 2000},
    {"seed": 2001, "d": 128},
    {"seed": 2002, "n_text": 16},
    {"seed": 2003, "T": 6, "P": 40, "spatial_band": 2, "temporal_width": 6},
    {"seed": 2004, "T": 5, "P": 300, "n_text": 77, "d": 128, "H": 4, "n_spatial": 2,
     "n_samples_fixed": 300, "spatial_band": 1, "temporal_width": 20},
]


@pytest.mark.parametrize("kw", VARIANTS)
def test_profile_labels_bit_exact_small(svg, kw):
    wl = SI.TINY.replace(**kw)
    q, k, v = SI.make_qkv(wl)
    rows = SI.sample_rows(wl)
    labels, mse = _run_profile(svg, wl, q, k, v, rows)
    heads = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    assert _check_heads(wl, q, k, v, rows, labels, mse, heads) == len(heads)
    kinds = SI.planted_head_kinds(wl)
    assert list(labels) == kinds * wl.B
    status_clean()


# Degenerate geometries: one frame, two-token frames, a single sampled row with
# fewer keys than one tile, exactly two full sample tiles, and masks that allow
# every key (their MSE is then ~0 and the label must pick them).
DEGENERATE = [
    ({"seed": 2300, "T": 1, "P": 200, "n_text": 8, "spatial_band": 0, "temporal_width": 10},
     "one_frame"),
    ({"seed": 2301, "T": 50, "P": 2, "n_text": 4, "spatial_band": 2, "temporal_width": 0},
     "two_token_frames"),
    ({"seed": 2302, "T": 3, "P": 30, "n_text": 0, "n_samples_fixed": 1}, "one_sample"),
    ({"seed": 2303, "T": 4, "P": 96, "n_text": 0, "d": 128, "n_samples_fixed": 256},
     "two_full_sample_tiles"),
    ({"seed": 2304, "T": 7, "P": 40, "n_text": 3, "spatial_band": 9, "temporal_width": 2},
     "spatial_mask_all_keys"),
    ({"seed": 2305, "T": 7, "P": 40, "n_text": 3, "spatial_band": 0, "temporal_width": 45},
     "temporal_mask_all_keys"),
]


@pytest.mark.parametrize("kw", [k for k, _ in DEGENERATE], ids=[w for _, w in DEGENERATE])
def test_profile_degenerate_geometries(svg, kw):
    wl = SI.TINY.replace(**kw)
    q, k, v = SI.make_qkv(wl)
    rows = SI.sample_rows(wl)
    labels, mse = _run_profile(svg, wl, q, k, v, rows)
    heads = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    _check_heads(wl, q, k, v, rows, labels, mse, heads)
    assert np.all(np.isfinite(mse)) and np.all(mse >= 0)
    if wl.spatial_band >= wl.T - 1:  # the spatial mask is every key
        assert np.all(mse[:, 0] <= NEAR_TIE_ABS)
    if wl.temporal_width >= wl.P - 1:  # the temporal mask is every key
        assert np.all(mse[:, 1] <= NEAR_TIE_ABS)
    status_clean()


def test_profile_unstructured_inputs(svg):
    # Diffuse attention: both errors are of similar size; labels must still agree
    # with the oracle wherever the two errors are not a near tie.
    wl = SI.TINY.replace(seed=2100, d=128, T=4, P=96, n_text=8, H=4, n_spatial=2,
                         n_samples_fixed=64)
    q, k, v = SI.make_qkv(wl, planted=False)
    rows = SI.sample_rows(wl)
    labels, mse = _run_profile(svg, wl, q, k, v, rows)
    _check_heads(wl, q, k, v, rows, labels, mse, [(0, h) for h in range(wl.H)])
    status_clean()


@pytest.mark.parametrize("wl", [SI.COGVIDEOX, SI.HUNYUAN, SI.LONG, SI.sweep_workloads()[2]],
                         ids=lambda w: w.name)
def test_profile_full_size(svg, wl):
    q, k, v = SI.make_qkv(wl)
    rows = SI.sample_rows(wl)
    labels, mse = _run_profile(svg, wl, q, k, v, rows)
    kinds = SI.planted_head_kinds(wl)
    assert list(labels) == kinds * wl.B
    sp = [h for h in range(wl.H) if kinds[h] == 0][:2]
    tp = [h for h in range(wl.H) if kinds[h] == 1][:2]
    heads = [(0, h) for h in sp + tp]
    if wl.B > 1:  # one head per label in the first and the last sample of the batch
        heads = [(0, sp[0]), (0, tp[0]), (wl.B - 1, sp[0]), (wl.B - 1, tp[0])]
    assert _check_heads(wl, q, k, v, rows, labels, mse, heads) == len(heads)
    status_clean()


def test_profile_deterministic(svg):
    wl = SI.TINY.replace(seed=2200, d=128, T=5, P=200, n_text=30, H=3, n_spatial=1,
                         n_samples_fixed=250)
    q, k, v = SI.make_qkv(wl)
    rows = SI.sample_rows(wl)
    l1, m1 = _run_profile(svg, wl, q, k, v, rows)
    l2, m2 = _run_profile(svg, wl, q, k, v, rows)
    assert np.array_equal(l1, l2) and np.array_equal(m1.view(np.int32), m2.view(np.int32))
    status_clean()
