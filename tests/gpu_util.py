"""Helpers shared by the GPU parity tests (no method arithmetic here beyond
error bounds; the reference values all come from the oracle)."""
import numpy as np
import torch

import oracle as O

# bf16-in / fp32-accumulate attention outputs vs the fp64 oracle: the absolute
# bars, and the relative L2 error of every compared head (the absolute bars
# alone are weak where |O| is small, e.g. planted spatial heads average V over
# a whole frame, |O| ~ 1/sqrt(P)). A correct kernel sits near the bf16
# rounding of P and O, a few 1e-3 relative.
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3
REL_L2 = 1e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a bf16 tensor (any device)."""
    return O.from_bf16_bits(t.detach().cpu().contiguous().view(torch.int16).numpy())


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def edge_rows(N, Nv, bq, n_random, seed, n_blocks=6, layout_to_frame_major=None):
    """Rows every parity check covers: both ends, the video/text boundary, the last
    query block's first and last row, plus seeded random rows drawn from a few
    seeded random query blocks (the oracle's cost grows with distinct blocks).

    Rows are chosen in the head's layout; `layout_to_frame_major` (an index
    array) maps them back to frame-major rows for position-major heads."""
    last_blk = ((N - 1) // bq) * bq
    rows = {0, 1, Nv - 1, N - 1, last_blk, min(last_blk + bq - 1, N - 1)}
    if Nv < N:
        rows.add(Nv)
    rng = np.random.default_rng(seed)
    nqb = -(-N // bq)
    blocks = rng.choice(nqb, size=min(n_blocks, nqb), replace=False)
    per = max(1, n_random // len(blocks))
    for b in blocks:
        lo, hi = b * bq, min(N, (b + 1) * bq)
        rows.update(rng.choice(np.arange(lo, hi), size=min(per, hi - lo), replace=False).tolist())
    out = np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)
    if layout_to_frame_major is not None:
        out = np.sort(layout_to_frame_major[out])
    return out


def assert_close(got: np.ndarray, want: np.ndarray, what: str, rel_l2: float = REL_L2,
                 atol_max: float = ATOL_MAX, atol_mean: float = ATOL_MEAN):
    """Element-wise comparison of one head's compared rows with the oracle.

    Gates: max-abs, mean-abs and the relative L2 error ||got - want|| / ||want||
    (skipped only when the reference is all zeros). Prints one PARITY line."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    norm = float(np.sqrt(np.sum(want * want)))
    rel = float(np.sqrt(np.sum(err * err)) / norm) if norm > 0 else 0.0
    print(f"PARITY {what}: max_abs {err.max():.3e} mean_abs {err.mean():.3e} rel_l2 {rel:.3e}")
    assert err.max() <= atol_max, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= atol_mean, f"{what}: mean abs err {err.mean():.3e}"
    assert rel <= rel_l2, f"{what}: relative L2 err {rel:.3e}"
    return float(err.max()), float(err.mean()), rel


def status_clean():
    import video_dit_spatial_b200 as svg
    st, bits = svg.svg_get_device_status()
    assert st == svg.SVG_OK and bits == 0, (st, bits)


# ---------------------------------------------------------------------------
# profiling: the oracle's errors and labels, with the tolerance the kernel's
# arithmetic allows
# ---------------------------------------------------------------------------
# The profiling kernel rounds every probability it feeds to the tensor core
# to bf16 (relative error delta_j, |delta_j| <= 2^-8, independent from key to
# key); everything else is fp32 (accumulators, row sums) or exact. An output
# element therefore carries e = sum_j delta_j p_j v_j / l, of variance at most
# u2 * sum_j (p_j / l)^2 v_j^2 with u2 = (2^-8)^2 / 3 (delta uniform in
# +-2^-8). The kernel's difference d + Delta of a masked and the full output
# has Var(Delta) <= 2 (Var e_X + Var e_F), so its MSE differs from the exact
# one by mean(2 d Delta + Delta^2): a bias of at most mean(Var Delta) and a
# spread whose 6-sigma bound is 6 sqrt(sum 4 d^2 Var Delta) / n plus
# 6 sqrt(sum 2 Var Delta^2) / n. That sum is the tolerance of each MSE; a
# head whose two MSEs are closer than the sum of their tolerances is a near
# tie, whose label either side may take.
_U2 = (2.0 ** -8) ** 2 / 3.0
_CHUNK = 128


def profile_reference(qn, kn, vn, rows, T, P, L, s, w, scale):
    """(mse_s, mse_t, label, tol_s, tol_t) of one head.

    The errors and the label are the oracle's (oracle.profile_head); the two
    tolerances follow the rounding model above, from the oracle's softmax
    weights of the full and the two masked attentions."""
    ms, mt, label = O.profile_head(qn, kn, vn, rows, T, P, L, s, w, scale)
    N = kn.shape[0]
    cols = np.arange(N)
    masks = (lambda rr: O.spatial_allowed(rr[:, None], cols[None, :], T, P, L, s),
             lambda rr: O.temporal_allowed(rr[:, None], cols[None, :], T, P, L, w))
    v2 = vn * vn
    acc = np.zeros((2, 3))  # per mask: sum VarDelta, sum 4 d^2 VarDelta, sum 2 VarDelta^2
    n = 0
    rows = np.asarray(rows, dtype=np.int64)
    for c0 in range(0, rows.size, _CHUNK):
        rr = rows[c0:c0 + _CHUNK]
        wf = O.attention_weights_rows(qn, kn, rr, None, scale)
        of, var_f = wf @ vn, (wf * wf) @ v2
        del wf
        for x, fn in enumerate(masks):
            wx = O.attention_weights_rows(qn, kn, rr, fn, scale)
            d = wx @ vn - of
            vd = 2.0 * _U2 * ((wx * wx) @ v2 + var_f)
            acc[x] += (vd.sum(), np.sum(4.0 * d * d * vd), np.sum(2.0 * vd * vd))
        n += rr.size * vn.shape[1]
    tol = [acc[x, 0] / n + 6.0 * np.sqrt(acc[x, 1]) / n + 6.0 * np.sqrt(acc[x, 2]) / n
           for x in range(2)]
    return ms, mt, label, float(tol[0]), float(tol[1])


def is_near_tie(ms, mt, tol_s, tol_t) -> bool:
    return abs(ms - mt) <= tol_s + tol_t
