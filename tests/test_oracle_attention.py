"""Pins of the oracle's masked softmax attention (CPU only).

The oracle is held against torch's scaled_dot_product_attention in float64 (a
library routine, with and without a boolean mask), a pure-Python double loop on
tiny inputs, and the textbook invariants of softmax attention.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _sdpa(q, k, v, mask, scale):
    qt, kt, vt = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=m, scale=scale)[0, 0].numpy()


def _rand(n, d, seed, sd=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((n, d)) * sd for _ in range(3)]


@pytest.mark.parametrize("n,d", [(1, 4), (17, 8), (130, 64), (257, 128)])
def test_all_ones_mask_is_dense_attention(n, d):
    q, k, v = _rand(n, d, n + d, sd=1.5)
    scale = 1 / math.sqrt(d)
    got, lse = O.masked_attention_rows(q, k, v, np.arange(n), None, scale)
    np.testing.assert_allclose(got, _sdpa(q, k, v, None, scale), rtol=1e-12, atol=1e-12)
    s = scale * q @ k.T
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(1)), rtol=1e-12)
    # an explicit all-ones mask follows exactly the same arithmetic
    ones, _ = O.masked_attention_rows(q, k, v, np.arange(n),
                                      lambda rr: np.ones((len(rr), n), bool), scale)
    assert np.array_equal(ones, got)


@pytest.mark.parametrize("seed", range(4))
def test_masked_attention_matches_sdpa_with_bool_mask(seed):
    n, d = 96, 16
    q, k, v = _rand(n, d, seed, sd=2.0)
    rng = np.random.default_rng(100 + seed)
    mask = rng.random((n, n)) < 0.3
    mask[np.arange(n), np.arange(n)] = True
    got, _ = O.masked_attention_rows(q, k, v, np.arange(n), lambda rr: mask[rr], 0.37)
    np.testing.assert_allclose(got, _sdpa(q, k, v, mask, 0.37), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("bq,bk", [(4, 4), (8, 4), (4, 8), (16, 16)])
def test_block_sparse_attention_matches_sdpa_on_expanded_mask(bq, bk):
    T, P, L = 3, 9, 5
    N = T * P + L
    q, k, v = _rand(N, 8, bq * 10 + bk)
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
        bm = O.block_mask(kind, T, P, L, 0, 1, bq, bk)
        tok = np.kron(bm, np.ones((bq, bk), bool))[:N, :N]
        got, _ = O.sparse_attention_rows(q, k, v, bm, bq, bk, 0.5)
        np.testing.assert_allclose(got, _sdpa(q, k, v, tok, 0.5), rtol=1e-11, atol=1e-12)


def test_pure_python_double_loop():
    n, d = 11, 3
    q, k, v = _rand(n, d, 7)
    rng = np.random.default_rng(8)
    mask = rng.random((n, n)) < 0.5
    mask[:, 0] = True
    scale = 0.8
    got, lse = O.masked_attention_rows(q, k, v, np.arange(n), lambda rr: mask[rr], scale)
    for i in range(n):
        logits = [scale * sum(q[i, c] * k[j, c] for c in range(d)) if mask[i, j] else None
                  for j in range(n)]
        mx = max(x for x in logits if x is not None)
        wts = [math.exp(x - mx) if x is not None else 0.0 for x in logits]
        tot = sum(wts)
        for c in range(d):
            assert abs(got[i, c] - sum(wts[j] * v[j, c] for j in range(n)) / tot) < 1e-12
        assert abs(lse[i] - (mx + math.log(tot))) < 1e-12


def test_softmax_rows_sum_to_one_and_constant_v():
    n, d = 64, 16
    q, k, _ = _rand(n, d, 9, sd=3.0)
    rng = np.random.default_rng(10)
    mask = rng.random((n, n)) < 0.2
    mask[np.arange(n), np.arange(n)] = True
    fn = lambda rr: mask[rr]  # noqa: E731
    wts = O.attention_weights_rows(q, k, np.arange(n), fn, 0.25)
    assert np.max(np.abs(wts.sum(1) - 1.0)) < 1e-12
    assert np.all(wts[~mask] == 0.0)
    ones = np.ones((n, d))
    o, _ = O.masked_attention_rows(q, k, ones, np.arange(n), fn, 0.25)
    assert np.max(np.abs(o - 1.0)) < 1e-12


def test_single_key_row_returns_that_value():
    n, d = 20, 5
    q, k, v = _rand(n, d, 11, sd=4.0)
    mask = np.zeros((n, n), bool)
    keys = (np.arange(n) * 7) % n
    mask[np.arange(n), keys] = True
    o, _ = O.masked_attention_rows(q, k, v, np.arange(n), lambda rr: mask[rr], 1.0)
    assert np.array_equal(o, v[keys])


def test_empty_row_gives_zeros():
    n, d = 6, 4
    q, k, v = _rand(n, d, 12)
    mask = np.ones((n, n), bool)
    mask[2] = False
    o, lse = O.masked_attention_rows(q, k, v, np.arange(n), lambda rr: mask[rr], 1.0)
    assert np.all(o[2] == 0.0) and lse[2] == -np.inf
    assert np.all(np.isfinite(lse[[0, 1, 3, 4, 5]]))


def test_large_logits_do_not_overflow():
    # max subtraction: logits of ~1e4 still give finite, exact results
    n, d = 8, 2
    q = np.full((n, d), 100.0)
    k = np.zeros((n, d))
    k[3] = 1.0
    v = np.arange(n * d, dtype=float).reshape(n, d)
    o, _ = O.masked_attention_rows(q, k, v, np.arange(n), None, 50.0)
    np.testing.assert_allclose(o, np.tile(v[3], (n, 1)), rtol=0, atol=1e-300)


def test_position_major_attention_is_equivariant():
    # Attention with M_T in position-major order = permute(attention with M_T in
    # frame-major order): the layout transformation does not change the result.
    T, P, L, w = 4, 6, 3, 1
    N = T * P + L
    q, k, v = _rand(N, 4, 13)
    cols = np.arange(N)
    fm, _ = O.masked_attention_rows(
        q, k, v, np.arange(N),
        lambda rr: O.temporal_allowed(rr[:, None], cols[None, :], T, P, L, w), 0.6)
    qp, kp, vp = (O.permute(x, T, P, L) for x in (q, k, v))
    pm, _ = O.masked_attention_rows(
        qp, kp, vp, np.arange(N),
        lambda rr: O.layout_allowed(O.MASK_TEMPORAL, rr[:, None], cols[None, :], T, P, L, 0, w),
        0.6)
    np.testing.assert_allclose(O.unpermute(pm, T, P, L), fm, rtol=1e-12, atol=1e-14)


def test_layer_rows_matches_full_layer_for_both_labels():
    T, P, L = 3, 8, 2
    N = T * P + L
    q, k, v = _rand(N, 4, 14)
    for label in (O.HEAD_SPATIAL, O.HEAD_TEMPORAL):
        full, _ = O.layer_rows(q, k, v, label, T, P, L, 0, 2, 4, 4, 0.5)
        rows = [0, 5, N - 1]
        part, _ = O.layer_rows(q, k, v, label, T, P, L, 0, 2, 4, 4, 0.5, rows=rows)
        np.testing.assert_array_equal(part, full[rows])
    # temporal label with the whole sequence in one block is dense attention
    full, _ = O.layer_rows(q, k, v, O.HEAD_TEMPORAL, T, P, L, 0, 0, 32, 32, 0.5)
    np.testing.assert_allclose(full, _sdpa(q, k, v, None, 0.5), rtol=1e-12, atol=1e-13)
