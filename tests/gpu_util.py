"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import oracle as O

# bf16-in / fp32-accumulate attention outputs vs the fp64 oracle
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3


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


def assert_close(got: np.ndarray, want: np.ndarray, what: str):
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= ATOL_MAX, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= ATOL_MEAN, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def status_clean():
    import video_dit_spatial_b200 as svg
    st, bits = svg.svg_get_device_status()
    assert st == svg.SVG_OK and bits == 0, (st, bits)
