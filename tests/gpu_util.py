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


# ---------------------------------------------------------------------------
# FP8 PV: the tolerance the e4m3 rounding of P and V allows
# ---------------------------------------------------------------------------
# The FP8 product rounds every probability p_j = exp(s_j - m) (scaled by 2^6,
# at a running base at most 2^2 below the row's maximum) and every V element
# to E4M3. A rounding moves a value by at most half a grid step h: 2^-4 of it
# for normal values, and 2^-9 / 2 = 2^-10 (in the rounded value's units) below
# 2^-6. In the units of the exact computation that is
#   h_p(p_j)   = max(2^-4 p_j, 2^-10 * 2^-6)       (a lower running base only
#                                                    shrinks the subnormal part)
#   h_v(v_jc)  = max(2^-4 |v_jc|, 2^-10 * scale_c)
# and an output element O_ic = sum_j w_j v_jc (w = p / l, l = sum p in fp32,
# not rounded) moves by sum_j (w_j dv_jc + dp_j v_jc / l). Taking each rounding
# error as an independent zero-mean variable of variance at most h^2 (the
# worst case of any distribution on [-h, h]) gives
#   sigma_ic^2 = sum_j w_j^2 h_v(v_jc)^2 + sum_j (h_p(p_j) / l)^2 v_jc^2,
# and the element-wise bar |O - O*| <= 6 sigma_ic + 2^-8 |O*_ic| (the bf16
# rounding of the output) + 1e-6.
def fp8_reference(qn, kn, vn, label, T, P, L, s, w, bq, bk, scale, rows):
    """(O* [r, d], tol [r, d]) at frame-major `rows` of one head: the oracle's
    block-sparse attention (oracle.layer_rows) and the FP8 tolerance above."""
    N = qn.shape[0]
    want, _ = O.layer_rows(qn, kn, vn, label, T, P, L, s, w, bq, bk, scale, rows=rows)
    kind = O.MASK_TEMPORAL if label == O.HEAD_TEMPORAL else O.MASK_SPATIAL
    rows = np.asarray(rows, dtype=np.int64)
    if kind == O.MASK_TEMPORAL:
        pi = O.permutation(T, P, L)
        lrows = pi[rows]
        ql, kl, vl = (O.permute(x, T, P, L) for x in (qn, kn, vn))
    else:
        lrows, ql, kl, vl = rows, qn, kn, vn
    needed = np.unique(lrows // bq)
    bm = np.zeros((O.n_blocks(N, bq), O.n_blocks(N, bk)), dtype=bool)
    bm[needed] = O.block_mask_rows(kind, needed, T, P, L, s, w, bq, bk)
    _, vscale = O.quantize_v_e4m3(vl)
    sc = vscale.astype(np.float64)
    xv = np.abs(vl) / np.where(sc > 0, sc, 1.0)[None, :]
    hv2 = np.where(xv >= 2.0 ** -6, 2.0 ** -4 * np.abs(vl), 2.0 ** -10 * sc[None, :]) ** 2
    v2 = vl * vl
    tol = np.zeros((rows.size, vn.shape[1]))
    for c0 in range(0, rows.size, _CHUNK):
        rr = lrows[c0:c0 + _CHUNK]
        wts = O.attention_weights_rows(ql, kl, rr, O.block_allowed_fn(bm, bq, bk, N), scale)
        wmax = wts.max(axis=1, keepdims=True)  # = 1 / l
        p = wts / wmax
        hp = np.maximum(2.0 ** -4 * p, 2.0 ** -16)
        hp = np.where(wts > 0, hp, 0.0)  # keys outside the computed blocks take no part
        var = (wts * wts) @ hv2 + ((hp * wmax) ** 2) @ v2
        tol[c0:c0 + rr.size] = 6.0 * np.sqrt(var)
    tol += 2.0 ** -8 * np.abs(want) + 1e-6
    return want, tol


def assert_within(got, want, tol, what):
    """Element-wise |got - want| <= tol; prints the FP8 PARITY line."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    norm = float(np.sqrt(np.sum(want * want)))
    rel = float(np.sqrt(np.sum(err * err)) / norm) if norm > 0 else 0.0
    ratio = float(np.max(err / tol))
    print(f"PARITY-FP8 {what}: max_abs {err.max():.3e} mean_abs {err.mean():.3e} "
          f"rel_l2 {rel:.3e} max err/tol {ratio:.3f}")
    assert ratio <= 1.0, f"{what}: error exceeds the e4m3 bound by {ratio:.3f}x"
    return float(err.max()), float(err.mean()), rel
