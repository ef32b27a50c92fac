"""svg_profile_heads_noalloc: online profiling without a caller-provided workspace.

Some callers of this library cannot allocate device memory when they call it
(an inference-engine plugin whose buffers are all planned up front, a
latency-critical loop that cannot take cudaMalloc's implicit synchronisation,
code with no allocator at hand). For them, svg_profile_heads_noalloc keeps the
MSE partial sums in a fixed 256 KiB array inside the library. This test calls
it through the C ABI twice in a row and checks both results against the
workspace-taking svg_profile_heads on the same inputs (equal labels, MSE equal
up to the rounding of a different summation order). The file is named so
that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import svg_inputs as SI

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svg():
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _profile_both(svg, wl, seed_salt):
    g = svg.Geom.from_workload(wl)
    q, k, v = (t.cuda() for t in SI.make_qkv(wl.replace(seed=wl.seed + seed_salt)))
    rows = SI.sample_rows(wl, seed_salt=seed_salt).cuda()
    BH = wl.B * wl.H
    ws = torch.empty(svg.svg_profile_workspace_bytes(g, rows.numel()) // 4 + 64,
                     dtype=torch.float32, device="cuda")
    lab_ref = torch.full((BH,), -1, dtype=torch.int8, device="cuda")
    mse_ref = torch.full((BH * 2,), float("nan"), device="cuda")
    svg.svg_profile_heads(g, q, k, v, rows, lab_ref, mse_ref, ws)
    lab = torch.full((BH,), -1, dtype=torch.int8, device="cuda")
    mse = torch.full((BH * 2,), float("nan"), device="cuda")
    svg.svg_profile_heads_noalloc(g, q, k, v, rows, lab, mse)
    st, bits = svg.svg_get_device_status()
    assert st == svg.SVG_OK and bits == 0, (st, bits)
    return lab_ref.cpu(), mse_ref.cpu(), lab.cpu(), mse.cpu()


def test_noalloc_matches_workspace_entry_point_twice(svg):
    wl = SI.TINY.replace(name="noalloc", d=128, T=5, P=300, n_text=77, H=4, n_spatial=2,
                         n_samples_fixed=300, spatial_band=1, temporal_width=20,
                         block_q=128, block_k=128, seed=4100)
    for call in range(2):  # the second call reuses the array the first one left behind
        lab_ref, mse_ref, lab, mse = _profile_both(svg, wl, seed_salt=call)
        assert torch.equal(lab, lab_ref)
        assert torch.all(torch.isfinite(mse))
        # The workspace entry point may split each tile's key range over several
        # CTAs to fill the GPU (the no-alloc one never does), so the fp32 sums
        # are added in another order: equal labels, MSE equal to rounding.
        np.testing.assert_allclose(mse.numpy(), mse_ref.numpy(), rtol=1e-3, atol=1e-9)
        assert list(lab.numpy()) == SI.planted_head_kinds(wl.replace(seed=wl.seed + call))


def test_noalloc_rejects_sizes_beyond_its_scratch(svg):
    # B*H*ceil(S/128) > 32768 needs more than the 256 KiB array: refused on the
    # host before any launch, outputs untouched.
    g = svg.Geom(1, 300, 64, 256, 0, 64, 64, 64, 1, 4, 0.125)  # 16384 video rows
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    rows = torch.zeros(128 * 110, dtype=torch.int32, device="cuda")
    lab = torch.full((300,), -1, dtype=torch.int8, device="cuda")
    with pytest.raises(svg.SvgError) as ei:
        svg.svg_profile_heads_noalloc(g, dummy, dummy, dummy, rows, lab)
    assert ei.value.status == svg.SVG_ERR_CAPACITY
    assert torch.all(lab == -1)
