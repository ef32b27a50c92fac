"""Pins of the oracle's online profiling rule (CPU only).

Hand-computed examples (tests/golden/profile_hand_example.txt), the q = 0 closed
form (every allowed key weighs the same, so each output is a plain mean of V),
the tie rule, and planted-pattern heads of the tiny workload and variants.
"""
import math
import os

import numpy as np
import pytest

import oracle as O
import svg_inputs as SI

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_cases():
    cases = {}
    with open(os.path.join(GOLDEN, "profile_hand_example.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            name, of, os_, ot, ms, mt, lab = line.split()
            vec = lambda s: [float(x) for x in s.split(",")]  # noqa: E731
            cases[name] = (vec(of), vec(os_), vec(ot), float(ms), float(mt), int(lab))
    return cases


def _masked_outputs(q, k, v, rows, T, P, L, s, w, scale):
    N = q.shape[0]
    cols = np.arange(N)
    rows = np.asarray(rows)
    full, _ = O.masked_attention_rows(q, k, v, rows, None, scale)
    sp, _ = O.masked_attention_rows(
        q, k, v, rows, lambda rr: O.spatial_allowed(rr[:, None], cols[None, :], T, P, L, s), scale)
    tp, _ = O.masked_attention_rows(
        q, k, v, rows, lambda rr: O.temporal_allowed(rr[:, None], cols[None, :], T, P, L, w), scale)
    return full, sp, tp


def test_hand_example_uniform():
    of, os_, ot, ms, mt, lab = _golden_cases()["uniform"]
    q = np.zeros((4, 1))
    k = np.zeros((4, 1))
    v = np.array([[1.0], [2.0], [3.0], [4.0]])
    full, sp, tp = _masked_outputs(q, k, v, [0, 3], 2, 2, 0, 0, 0, 1.0)
    np.testing.assert_allclose(full[:, 0], of, rtol=1e-15)
    np.testing.assert_allclose(sp[:, 0], os_, rtol=1e-15)
    np.testing.assert_allclose(tp[:, 0], ot, rtol=1e-15)
    mse_s, mse_t, label = O.profile_head(q, k, v, [0, 3], 2, 2, 0, 0, 0, 1.0)
    assert abs(mse_s - ms) < 1e-15 and abs(mse_t - mt) < 1e-15 and label == lab


def test_hand_example_weighted():
    of, os_, ot, ms, mt, lab = _golden_cases()["weighted"]
    q = np.array([[1.0], [0.0], [0.0], [0.0]])
    k = np.array([[0.0], [math.log(3.0)], [0.0], [0.0]])
    v = np.array([[1.0], [2.0], [3.0], [4.0]])
    full, sp, tp = _masked_outputs(q, k, v, [0], 2, 2, 0, 0, 0, 1.0)
    assert abs(full[0, 0] - of[0]) < 1e-14
    assert abs(sp[0, 0] - os_[0]) < 1e-14
    assert abs(tp[0, 0] - ot[0]) < 1e-14
    mse_s, mse_t, label = O.profile_head(q, k, v, [0], 2, 2, 0, 0, 0, 1.0)
    assert abs(mse_s - ms) < 1e-14 and abs(mse_t - mt) < 1e-14 and label == lab


@pytest.mark.parametrize("T,P,L,s,w", [(3, 5, 0, 0, 1), (4, 6, 3, 1, 2), (2, 9, 1, 0, 0)])
def test_zero_query_closed_form(T, P, L, s, w):
    # q = 0: every allowed key weighs 1, so each output is the mean of V over the
    # allowed keys, and the MSEs follow from those means directly.
    N = T * P + L
    rng = np.random.default_rng(T * 31 + P)
    v = rng.standard_normal((N, 3))
    q = np.zeros((N, 3))
    k = rng.standard_normal((N, 3))
    rows = np.arange(0, T * P, 2)
    mean_full = v.mean(0)
    sp_want, tp_want = [], []
    for i in rows:
        f, p = divmod(i, P)
        keys_s = [j for j in range(N) if j >= T * P or abs(j // P - f) <= s]
        keys_t = [j for j in range(N) if j >= T * P or abs(j % P - p) <= w]
        sp_want.append(v[keys_s].mean(0))
        tp_want.append(v[keys_t].mean(0))
    sp_want, tp_want = np.array(sp_want), np.array(tp_want)
    full, sp, tp = _masked_outputs(q, k, v, rows, T, P, L, s, w, 1.0)
    np.testing.assert_allclose(full, np.tile(mean_full, (len(rows), 1)), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(sp, sp_want, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(tp, tp_want, rtol=1e-13, atol=1e-14)
    mse_s, mse_t, _ = O.profile_head(q, k, v, rows, T, P, L, s, w, 1.0)
    assert abs(mse_s - np.mean((sp_want - mean_full) ** 2)) < 1e-13
    assert abs(mse_t - np.mean((tp_want - mean_full) ** 2)) < 1e-13


def test_full_width_masks_tie_to_spatial():
    T, P, L = 3, 4, 2
    N = T * P + L
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((N, 4)) for _ in range(3))
    mse_s, mse_t, label = O.profile_head(q, k, v, [0, 4, 7], T, P, L, T - 1, P - 1, 0.5)
    assert mse_s == 0.0 and mse_t == 0.0 and label == O.HEAD_SPATIAL


def _head64(t):
    return O.from_bf16_bits(t.view(__import__("torch").int16).numpy())


@pytest.mark.parametrize("wl_kw", [
    {},
    {"seed": 2000},
    {"seed": 2001, "d": 128},
    {"seed": 2002, "n_text": 16},
    {"seed": 2003, "T": 6, "P": 40, "spatial_band": 2, "temporal_width": 6},
])
def test_planted_heads_are_classified(wl_kw):
    wl = SI.TINY.replace(**wl_kw)
    rows = SI.sample_rows(wl).numpy()
    kinds = SI.planted_head_kinds(wl)
    for h in range(wl.H):
        q, k, v = (_head64(t) for t in SI.make_head(wl, 0, h))
        mse_s, mse_t, label = O.profile_head(q, k, v, rows, wl.T, wl.P, wl.n_text,
                                             wl.spatial_band, wl.temporal_width, wl.scale)
        assert label == kinds[h], (h, mse_s, mse_t)
        lo, hi = sorted((mse_s, mse_t))
        assert hi > 10 * lo  # far from a tie


def test_planted_spatial_head_attends_within_its_frame():
    # Planted-spatial logits inside the query's frame exceed the others by ~26
    # nats, so full attention equals own-frame (band 0) attention to ~1e-6.
    wl = SI.TINY
    q, k, v = (_head64(t) for t in SI.make_head(wl, 0, 0))
    rows = np.arange(0, wl.N_v, 5)
    N = wl.N
    cols = np.arange(N)
    full, _ = O.masked_attention_rows(q, k, v, rows, None, wl.scale)
    own, _ = O.masked_attention_rows(
        q, k, v, rows, lambda rr: O.spatial_allowed(rr[:, None], cols[None, :], wl.T, wl.P, 0, 0),
        wl.scale)
    assert np.max(np.abs(full - own)) < 1e-6
