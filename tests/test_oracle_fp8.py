"""Pins of the oracle's e4m3 rounding and per-channel V quantisation (CPU).

The FP8 PV product rounds softmax probabilities and V to E4M3 (the "fn"
variant: bias 7, 3 mantissa bits, largest finite 448, no infinities). The
oracle's rounding is pinned against hand-worked values (tests/golden), against
an independent implementation (torch's float8_e4m3fn conversion) over every
fp32 value class in range, and its quantiser against the invariants of its
definition.
"""
import os

import numpy as np
import pytest
import torch

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = []
    for line in open(os.path.join(HERE, "golden", "e4m3_rounding.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()[:2]
        rows.append((float(a), float(b)))
    return rows


def test_e4m3_round_hand_values():
    rows = _golden()
    assert len(rows) >= 12
    got = O.e4m3_round([a for a, _ in rows])
    assert list(got) == [b for _, b in rows]


def test_e4m3_round_matches_torch_float8_on_a_sweep():
    # every e4m3 grid point, the midpoints between neighbours (the ties), and
    # random fp32 values across all binades, below the value (464) at which
    # torch's conversion stops saturating to 448 and returns NaN
    grid = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    grid = grid[torch.isfinite(grid)].unique().double().numpy()
    mids = (grid[1:] + grid[:-1]) / 2
    rng = np.random.default_rng(5)
    rnd = np.exp2(rng.uniform(-14, np.log2(463.0), 200000)) * rng.choice([-1.0, 1.0], 200000)
    xs = np.concatenate([grid, mids, rnd]).astype(np.float32)
    xs = xs[np.abs(xs) < 464.0]
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).double().numpy()
    got = O.e4m3_round(xs.astype(np.float64))
    assert np.array_equal(got, want)


def test_quantize_v_invariants():
    rng = np.random.default_rng(7)
    v = O.from_bf16_bits(O.to_bf16_bits(rng.standard_normal((1000, 128))))
    v[:, 5] = 0.0  # an all-zero channel
    codes, scale = O.quantize_v_e4m3(v)
    assert scale.dtype == np.float32 and codes.shape == v.shape
    assert scale[5] == 0 and np.all(codes[:, 5] == 0)
    live = np.arange(128) != 5
    # the largest |v| of a channel lands exactly on the top code 448
    assert np.all(np.max(np.abs(codes[:, live]), axis=0) == 448.0)
    # every code is an e4m3 value and re-rounding it changes nothing
    assert np.array_equal(O.e4m3_round(codes), codes)
    # the scale undoes the quantisation to the format's relative precision
    # (half a grid spacing <= 2^-4 of the value for normals, 2^-10 * scale below)
    deq = codes * scale[None, :].astype(np.float64)
    x = np.abs(v / np.where(scale > 0, scale, 1)[None, :])
    bound = np.where(x >= 2.0 ** -6, 2.0 ** -4 * np.abs(v), 2.0 ** -10 * scale[None, :]) * (1 + 1e-6)
    assert np.all(np.abs(deq - v)[:, live] <= bound[:, live] + 1e-12)
    # scale = fp32(amax / 448)
    amax = np.max(np.abs(v), axis=0).astype(np.float32)
    assert np.array_equal(scale, (amax / np.float32(448.0)).astype(np.float32))


@pytest.mark.parametrize("bad", ["no_saturation", "round_half_up", "wrong_subnormal"])
def test_planted_rounding_mistakes_are_caught(bad):
    """A plausible mistake in the rounding fails the torch sweep or the hand values."""
    rows = _golden()
    xs = np.array([a for a, _ in rows])
    want = np.array([b for _, b in rows])

    def wrong(x):
        a = np.abs(x)
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
        sp_sub = 2.0 ** -10 if bad == "wrong_subnormal" else 2.0 ** -9
        sp = np.where(a >= 2.0 ** -6, 2.0 ** (e - 3), sp_sub)
        q = (np.floor(a / sp + 0.5) if bad == "round_half_up" else np.round(a / sp)) * sp
        if bad != "no_saturation":
            q = np.minimum(q, 448.0)
        return np.where(x < 0, -q, q)
    assert not np.array_equal(wrong(xs), want)
