"""Pins of the oracle's masks, block masks and layout transformation (CPU only).

The oracle's block mask is the brute-force OR over token pairs; here it is held
against an independent interval formula, against token-pair counts in closed
form, against hand-derived values for the tiny workload, and against numpy's own
transpose for the permutation.
"""
import itertools
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden_matrices(name):
    mats, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.isalpha():
                cur = line
                mats[cur] = []
            else:
                mats[cur].append([int(x) for x in line.split()])
    return {k: np.array(v, dtype=bool) for k, v in mats.items()}


def interval_block_mask(kind, T, P, n_text, s, w, bq, bk):
    """Closed form: video groups of a block form an integer interval.

    Group = frame (spatial, frame-major) or position (temporal, position-major).
    A (r, c) pair is on iff either block holds a text token, or the group
    intervals come within the band of each other.
    """
    N = T * P + n_text
    Nv = T * P
    G, band = (P, s) if kind == O.MASK_SPATIAL else (T, w)
    nqb, nkb = -(-N // bq), -(-N // bk)
    bm = np.zeros((nqb, nkb), dtype=bool)

    def span(b, size):
        lo, hi = b * size, min((b + 1) * size, N)
        text = hi > Nv
        vhi = min(hi, Nv)
        if lo >= vhi:
            return text, None
        return text, (lo // G, (vhi - 1) // G)

    for r in range(nqb):
        tr, ir = span(r, bq)
        for c in range(nkb):
            tc, ic = span(c, bk)
            if kind == O.MASK_DENSE or tr or tc:
                bm[r, c] = True
            elif ir is not None and ic is not None:
                bm[r, c] = ic[0] <= ir[1] + band and ic[1] >= ir[0] - band
    return bm


TINY_GEOMS = [(T, P, L) for T in (1, 2, 3, 5, 9) for P in (1, 2, 3, 7, 9) for L in (0, 1, 5)]


@pytest.mark.parametrize("T,P,L", TINY_GEOMS)
def test_block_mask_brute_force_matches_interval_form(T, P, L):
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL, O.MASK_DENSE):
        for bq, bk in ((1, 1), (2, 3), (3, 2), (4, 4), (8, 8), (2, 8)):
            for band in (0, 1, 2, 8):
                s = w = band
                got = O.block_mask(kind, T, P, L, s, w, bq, bk)
                want = interval_block_mask(kind, T, P, L, s, w, bq, bk)
                assert np.array_equal(got, want), (kind, T, P, L, bq, bk, band)


def _pairs_spatial(T, P, L, s):
    N, Nv = T * P + L, T * P
    inner = T + 2 * sum(T - dlt for dlt in range(1, min(s, T - 1) + 1))
    return P * P * inner + (N * N - Nv * Nv)


def _pairs_temporal(T, P, L, w):
    N, Nv = T * P + L, T * P
    inner = P + 2 * sum(P - dlt for dlt in range(1, min(w, P - 1) + 1))
    return T * T * inner + (N * N - Nv * Nv)


@pytest.mark.parametrize("T,P,L,band", [(1, 1, 0, 0), (4, 64, 0, 1), (5, 7, 3, 2),
                                         (3, 10, 4, 0), (6, 5, 0, 9), (11, 40, 2, 3)])
def test_token_pair_counts_closed_form(T, P, L, band):
    N = T * P + L
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    assert int(O.spatial_allowed(i, j, T, P, L, band).sum()) == _pairs_spatial(T, P, L, band)
    assert int(O.temporal_allowed(i, j, T, P, L, band).sum()) == _pairs_temporal(T, P, L, band)
    # The temporal mask moved to position-major order keeps its pair count.
    assert int(O.layout_allowed(O.MASK_TEMPORAL, i, j, T, P, L, band, band).sum()) == \
        _pairs_temporal(T, P, L, band)


def test_tiny_block_masks_by_hand():
    gold = _read_golden_matrices("tiny_block_masks.txt")
    bs = O.block_mask(O.MASK_SPATIAL, 4, 64, 0, 1, 4, 64, 64)
    bt = O.block_mask(O.MASK_TEMPORAL, 4, 64, 0, 1, 4, 64, 64)
    assert np.array_equal(bs, gold["spatial"])
    assert np.array_equal(bt, gold["temporal"])
    assert bs.sum() == 10 and bt.sum() == 10


def test_full_width_masks_are_all_ones():
    for T, P, L in [(3, 5, 2), (4, 64, 0), (2, 9, 0)]:
        for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
            bm = O.block_mask(kind, T, P, L, T - 1, P - 1, 4, 4)
            assert bm.all()


def test_csr_roundtrip_and_order():
    rng = np.random.default_rng(3)
    bm = rng.random((7, 9)) < 0.4
    rp, ci = O.to_csr(bm)
    assert rp[0] == 0 and rp[-1] == bm.sum()
    for r in range(7):
        row = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(row) > 0)
    assert np.array_equal(O.from_csr(rp, ci, 9), bm)


def test_block_mask_rows_matches_full():
    T, P, L = 5, 37, 11
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
        full = O.block_mask(kind, T, P, L, 1, 6, 16, 8)
        rows = [0, 3, full.shape[0] - 1]
        part = O.block_mask_rows(kind, rows, T, P, L, 1, 6, 16, 8)
        assert np.array_equal(part, full[rows])


# ---------------------------------------------------------------------------
# layout transformation
# ---------------------------------------------------------------------------
def test_permutation_hand_values():
    pi = O.permutation(4, 64, 0)
    with open(os.path.join(GOLDEN, "tiny_permutation.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            a, b = (int(x) for x in line.split())
            assert pi[a] == b


@pytest.mark.parametrize("T,P,L", [(1, 7, 0), (5, 1, 3), (4, 64, 0), (3, 5, 4), (33, 12, 7)])
def test_permutation_is_the_grid_transpose(T, P, L):
    pi = O.permutation(T, P, L)
    N = T * P + L
    assert sorted(pi.tolist()) == list(range(N))  # bijection
    if T == 1 or P == 1:
        assert np.array_equal(pi, np.arange(N))
    rng = np.random.default_rng(T * 100 + P)
    x = rng.standard_normal((2, N, 3))
    y = O.permute(x, T, P, L)
    # Independent formulation: the video part is a [T, P] -> [P, T] transpose.
    want = x.copy()
    want[:, :T * P] = x[:, :T * P].reshape(2, T, P, 3).transpose(0, 2, 1, 3).reshape(2, T * P, 3)
    assert np.array_equal(y, want)
    assert np.array_equal(O.unpermute(y, T, P, L), x)
    assert np.array_equal(O.inverse_permutation(pi)[pi], np.arange(N))


def test_layout_to_frame_major_inverts_pi():
    for T, P, L in [(3, 5, 2), (6, 4, 0)]:
        pi = O.permutation(T, P, L)
        idx = np.arange(T * P + L)
        assert np.array_equal(O.layout_to_frame_major(O.MASK_TEMPORAL, pi[idx], T, P, L), idx)


def test_temporal_mask_becomes_banded_in_position_major_order():
    # In position-major order, |dp| <= w covers index distance < (w+1)*T around the
    # diagonal: each video row's allowed keys form ONE contiguous run.
    T, P, L, w = 4, 9, 0, 2
    N = T * P
    a = np.arange(N)
    m = O.layout_allowed(O.MASK_TEMPORAL, a[:, None], a[None, :], T, P, L, 0, w)
    for r in range(N):
        nz = np.nonzero(m[r])[0]
        assert np.all(np.diff(nz) == 1)
        p = r // T
        assert nz[0] == max(0, p - w) * T and nz[-1] == min(P, p + w + 1) * T - 1


def test_bf16_bits_roundtrip():
    import torch
    x = torch.randn(1000, dtype=torch.float64) * 10
    bits = x.to(torch.bfloat16).view(torch.int16).numpy()
    vals = O.from_bf16_bits(bits)
    assert np.array_equal(vals, x.to(torch.bfloat16).to(torch.float64).numpy())
    assert np.array_equal(O.to_bf16_bits(x.numpy()), bits.view(np.uint16))


def test_flops_computed_blocks_counts_ragged_edges():
    N, bq, bk, d = 10, 4, 4, 2
    bm = np.ones((3, 3), dtype=bool)
    assert O.flops_computed_blocks(bm, N, bq, bk, d) == 4 * d * N * N
    bm[2, 2] = False
    assert O.flops_computed_blocks(bm, N, bq, bk, d) == 4 * d * (N * N - 4)


def test_exhaustive_small_bands():
    # every (s, w) up to the full width on a ragged geometry with text
    T, P, L = 4, 6, 3
    for s, w in itertools.product(range(0, 4), range(0, 6)):
        for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
            got = O.block_mask(kind, T, P, L, s, w, 5, 3)
            want = interval_block_mask(kind, T, P, L, s, w, 5, 3)
            assert np.array_equal(got, want)
