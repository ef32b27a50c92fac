"""Host-side checks of the C ABI (no GPU kernel launches).

The library builds and loads, exports every symbol include/svg.h declares,
validates arguments before touching the device, and its host-only nnz count
equals the oracle's brute-force block count.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def svg():
    from video_dit_spatial_b200 import _build
    _build.build()
    import video_dit_spatial_b200 as m
    m.load()
    return m


def _header_symbols():
    text = open(os.path.join(ROOT, "include", "svg.h")).read()
    return sorted(set(re.findall(r"^\s*(?:svg_status|const char\*|int32_t)\s+(svg2?_\w+)\s*\(",
                                 text, flags=re.M)))


def test_exports_every_declared_symbol(svg):
    syms = _header_symbols()
    assert len(syms) >= 12
    lib = ctypes.CDLL(svg.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(svg.EXPORTED)


def test_status_strings(svg):
    for code, name in svg.STATUS_NAMES.items():
        assert svg.svg_status_string(code) == name
    assert svg.svg_version() == 100


def _geom(svg, T=4, P=64, L=0, d=64, bq=64, bk=64, s=1, w=4, B=1, H=2):
    return svg.Geom(B, H, T, P, L, d, bq, bk, s, w, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("T,P,L,bq,bk,s,w", [
    (4, 64, 0, 64, 64, 1, 4), (3, 5, 2, 4, 4, 0, 1), (5, 7, 3, 8, 3, 1, 2),
    (9, 9, 5, 2, 8, 2, 0), (11, 40, 7, 128, 64, 2, 12), (1, 13, 0, 4, 4, 0, 0),
    (6, 1, 4, 2, 2, 1, 0)])
def test_mask_nnz_equals_brute_force(svg, T, P, L, bq, bk, s, w):
    g = _geom(svg, T, P, L, 64, bq, bk, s, w)
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL, O.MASK_DENSE):
        want = int(O.block_mask(kind, T, P, L, s, w, bq, bk).sum())
        assert svg.svg_mask_nnz(g, kind) == want


def test_mask_nnz_large_workloads_row_sample(svg):
    # The full workloads are too large for a brute-force count, but the nnz must
    # equal the sum over rows; check rows sampled with the oracle add up with the
    # dense count as an upper bound and the tiny-case identity above.
    import svg_inputs as SI
    wl = SI.HUNYUAN
    g = svg.Geom.from_workload(wl)
    nqb = g.n_qblocks
    assert svg.svg_mask_nnz(g, O.MASK_DENSE) == nqb * g.n_kblocks
    for kind in (O.MASK_SPATIAL, O.MASK_TEMPORAL):
        nnz = svg.svg_mask_nnz(g, kind)
        assert 0 < nnz < nqb * g.n_kblocks


def test_invalid_arguments_are_rejected_before_launch(svg):
    g = _geom(svg)
    out = ctypes.c_int64()
    lib = svg.load()
    assert lib.svg_mask_nnz(None, 0, ctypes.byref(out)) == svg.SVG_ERR_INVALID_ARG
    assert lib.svg_mask_nnz(ctypes.byref(g), 3, ctypes.byref(out)) == svg.SVG_ERR_INVALID_ARG
    bad = _geom(svg, T=0)
    assert lib.svg_mask_nnz(ctypes.byref(bad), 0, ctypes.byref(out)) == svg.SVG_ERR_INVALID_ARG
    bad = _geom(svg, s=-1)
    assert lib.svg_mask_nnz(ctypes.byref(bad), 0, ctypes.byref(out)) == svg.SVG_ERR_INVALID_ARG
    # capacity is checked before the device
    assert lib.svg_build_block_mask(ctypes.byref(g), 0, 16, 16, 3, None) == svg.SVG_ERR_CAPACITY
    assert lib.svg_build_block_mask(ctypes.byref(g), 0, None, 16, 100, None) == \
        svg.SVG_ERR_INVALID_ARG
    # unsupported head dim / block size for the attention and profiling kernels
    g96 = _geom(svg, d=96)
    assert lib.svg_sparse_attention(ctypes.byref(g96), *([256] * 3), None, None, None, None,
                                    256, 256, None, None, 256, None, None, None) == \
        svg.SVG_ERR_UNSUPPORTED
    # misaligned tensor
    assert lib.svg_sparse_attention(ctypes.byref(g), 258, 256, 256, None, None, None, None,
                                    256, 256, None, None, 256, None, None, None) == \
        svg.SVG_ERR_INVALID_ARG
    # partial set of permuted tensors
    assert lib.svg_sparse_attention(ctypes.byref(g), 256, 256, 256, 256, None, None, None,
                                    256, 256, 256, 256, 256, None, None, None) == \
        svg.SVG_ERR_INVALID_ARG
    # fused layout path: labels and both CSRs required; kp/vp both or neither;
    # 128-row query blocks only
    f = lib.svg_sparse_attention_fused
    g128 = _geom(svg, bq=128)
    assert f(ctypes.byref(g128), 256, 256, 256, None, None, None, 256, 256, 256, 256, 256,
             None, None) == svg.SVG_ERR_INVALID_ARG
    assert f(ctypes.byref(g128), 256, 256, 256, None, None, 256, 256, 256, None, 256, 256,
             None, None) == svg.SVG_ERR_INVALID_ARG
    assert f(ctypes.byref(g128), 256, 264, 256, None, None, 256, 256, 256, 256, 256, 256,
             None, None) == svg.SVG_ERR_INVALID_ARG
    assert f(ctypes.byref(g128), 256, 256, 256, 256, None, 256, 256, 256, 256, 256, 256,
             None, None) == svg.SVG_ERR_INVALID_ARG
    g64 = _geom(svg, bq=64)
    assert f(ctypes.byref(g64), 256, 256, 256, None, None, 256, 256, 256, 256, 256, 256,
             None, None) == svg.SVG_ERR_UNSUPPORTED
    huge = _geom(svg, bq=128, T=1 << 15, P=1 << 14, B=1, H=4)  # 4 * 2^29 rows >= 2^31
    assert f(ctypes.byref(huge), 256, 256, 256, None, None, 256, 256, 256, 256, 256, 256,
             None, None) == svg.SVG_ERR_UNSUPPORTED
    # permute of K and V only: q and qp both NULL or both given
    assert lib.svg_permute_qkv(ctypes.byref(g), 256, 4096, 8192, None, 1 << 20, 1 << 21,
                               None, None) == svg.SVG_ERR_INVALID_ARG
    # overlapping permute buffers
    assert lib.svg_permute(ctypes.byref(g), 4096, 4096 + 256, None, None) == \
        svg.SVG_ERR_INVALID_ARG
    # profiling: too many samples, misaligned workspace, small workspace
    ws = ctypes.c_size_t()
    assert lib.svg_profile_workspace_bytes(ctypes.byref(g), 16, ctypes.byref(ws)) == svg.SVG_OK
    # 2 CTAs (B*H = 2, one tile of samples) fill 148 SMs best with 4 key-range
    # splits: per-tile errors (padded to 256 B), then the split partials
    ctas, splits, d = 2, 4, 64
    assert ws.value == 256 + ctas * splits * 3 * (d + 2) * 128 * 4
    assert lib.svg_profile_heads(ctypes.byref(g), 256, 256, 256, 256, 257, 256, None, 256,
                                 1 << 20, None) == svg.SVG_ERR_INVALID_ARG
    assert lib.svg_profile_heads(ctypes.byref(g), 256, 256, 256, 256, 16, 256, None, 260,
                                 1 << 20, None) == svg.SVG_ERR_INVALID_ARG
    assert lib.svg_profile_heads(ctypes.byref(g), 256, 256, 256, 256, 16, 256, None, 256,
                                 4, None) == svg.SVG_ERR_CAPACITY
    assert lib.svg_selftest_wait_timeout(0, None) == svg.SVG_ERR_INVALID_ARG


def _expected_splits(ctas, nkt, sms=148):
    """The documented rule: the split count in 1..4 (at most the key tiles) whose
    CTAs fill the last wave of 148 SMs best; ties go to fewer splits."""
    best, best_fill = 1, 0.0
    for sp in range(1, min(4, nkt) + 1):
        c = ctas * sp
        fill = c / (-(-c // sms) * sms)
        if fill > best_fill + 1e-9:
            best, best_fill = sp, fill
    return best


@pytest.mark.parametrize("name", ["cogvideox15_B1_H48_d64_T11_P4080_L226",
                                  "hunyuan_B1_H24_d128_T33_P3600_L256",
                                  "long_B2_H8_d128_T64_P3600_L256", "sweep_s2_w256",
                                  "tiny_B1_H2_d64_T4_P64"])
def test_profile_workspace_follows_the_split_rule(svg, name):
    import svg_inputs as SI
    wl = SI.WORKLOADS[name]
    g = svg.Geom.from_workload(wl)
    S = wl.n_samples
    tiles = -(-S // 128)
    ctas = wl.B * wl.H * tiles
    nkt = -(-wl.N // 64)
    sp = _expected_splits(ctas, nkt)
    want = ctas * 2 * 4
    if sp > 1:
        want = -(-want // 256) * 256 + ctas * sp * 3 * (wl.d + 2) * 128 * 4
    assert svg.svg_profile_workspace_bytes(g, S) == want
    # the configurations the benchmark runs split as documented
    expected = {"hunyuan_B1_H24_d128_T33_P3600_L256": 3, "long_B2_H8_d128_T64_P3600_L256": 4,
                "cogvideox15_B1_H48_d64_T11_P4080_L226": 3}
    if name in expected:
        assert sp == expected[name]


def test_no_device_reports_cuda_error(svg):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    g = _geom(svg)
    lib = svg.load()
    st = lib.svg_build_block_mask(ctypes.byref(g), 0, 256, 256, 1 << 20, None)
    assert st in (svg.SVG_ERR_CUDA, svg.SVG_ERR_UNSUPPORTED)


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import video_dit_spatial_b200 as m
    monkeypatch.setattr(m, "_lib", None)
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(OSError):
        m.load()


def test_python_binding_rejects_host_tensors():
    # A host address handed to a kernel would fault on the device: the binding
    # refuses CPU tensors before anything reaches the library.
    import torch
    import video_dit_spatial_b200 as m
    g = m.Geom(1, 1, 2, 4, 0, 64, 64, 64, 0, 0, 0.125)
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="device buffers"):
        m.svg_permute(g, x, torch.zeros_like(x))
    with pytest.raises(ValueError, match="device buffers"):
        m._ptr(x.transpose(2, 3))
    assert m._ptr(None) is None and m._ptr(1234) == 1234


def test_fp8_and_svg2_arguments_are_rejected_before_launch(svg):
    """Host-side validation of the FP8, SVG2 and SVG-EAR entry points: every
    case below is refused before any device call (no GPU needed)."""
    lib = svg.load()
    g64 = _geom(svg, d=64, bq=128, bk=128)
    g128 = _geom(svg, d=128, bq=128, bk=128)
    gq64 = _geom(svg, d=128, bq=64, bk=128)
    # FP8: d = 128 only; block_q = 128 only; labels need vp; misaligned codes
    assert lib.svg_quantize_v_e4m3(ctypes.byref(g64), 256, None, None, 256, 256, None) == \
        svg.SVG_ERR_UNSUPPORTED
    assert lib.svg_quantize_v_e4m3(ctypes.byref(g128), 256, None, 256, 256, 256, None) == \
        svg.SVG_ERR_INVALID_ARG
    assert lib.svg_quantize_v_e4m3(ctypes.byref(g128), 256, None, None, 264, 256, None) == \
        svg.SVG_ERR_INVALID_ARG
    fa = lib.svg_sparse_attention_fp8pv
    assert fa(ctypes.byref(gq64), 256, 256, None, None, 256, 256, None, 256, 256, None, None,
              256, None, None, None) == svg.SVG_ERR_UNSUPPORTED
    assert fa(ctypes.byref(g128), 256, 256, 256, None, 256, 256, None, 256, 256, None, None,
              256, None, None, None) == svg.SVG_ERR_INVALID_ARG  # qp without kp/op
    # SVG2 k-means: C a multiple of 16 in [16, 256], d 64 or 128
    ws = ctypes.c_size_t()
    assert lib.svg2_kmeans_workspace_bytes(2, 1000, 128, 17, ctypes.byref(ws)) == \
        svg.SVG_ERR_UNSUPPORTED
    assert lib.svg2_kmeans_workspace_bytes(2, 1000, 128, 272, ctypes.byref(ws)) == \
        svg.SVG_ERR_UNSUPPORTED
    assert lib.svg2_kmeans_workspace_bytes(2, 1000, 96, 32, ctypes.byref(ws)) == \
        svg.SVG_ERR_UNSUPPORTED
    assert lib.svg2_kmeans_workspace_bytes(2, 1000, 128, 32, ctypes.byref(ws)) == svg.SVG_OK
    need = ws.value
    assert lib.svg2_kmeans(2, 1000, 128, 32, 3, 256, 256, 256, 256, 256, 256, need - 1,
                           None) == svg.SVG_ERR_CAPACITY
    assert lib.svg2_kmeans(2, 1000, 128, 32, 3, 256, 256, 256, 256, 256, 264, need,
                           None) == svg.SVG_ERR_INVALID_ARG  # workspace not 256-aligned
    assert lib.svg2_kmeans_step(2, 1000, 128, 32, 256, 512, 512, 256, 256, 256, 256, need,
                                None) == svg.SVG_ERR_INVALID_ARG  # in place
    # selection: Ck <= 1024, 0 < top_p <= 1, tau >= 0 when routing
    sel = lib.svg2_select_clusters
    assert sel(1, 128, 8, 1025, ctypes.c_float(0.1), ctypes.c_float(0.9), 256, 256, 256, None,
               ctypes.c_float(0.0), 256, None) == svg.SVG_ERR_INVALID_ARG
    assert sel(1, 128, 8, 64, ctypes.c_float(0.1), ctypes.c_float(1.5), 256, 256, 256, None,
               ctypes.c_float(0.0), 256, None) == svg.SVG_ERR_INVALID_ARG
    assert sel(1, 128, 8, 64, ctypes.c_float(0.1), ctypes.c_float(0.9), 256, 256, 256, 256,
               ctypes.c_float(-1.0), 256, None) == svg.SVG_ERR_INVALID_ARG
    # tile CSR: blocks 64 or 128; at most 4096 key tiles
    csr = lib.svg2_build_tile_csr
    assert csr(1, 1000, 8, 8, 96, 128, 256, 256, 256, 256, 256, 100, 256, None) == \
        svg.SVG_ERR_UNSUPPORTED
    assert csr(1, 4097 * 64, 8, 8, 128, 64, 256, 256, 256, 256, 256, 100, 256, None) == \
        svg.SVG_ERR_UNSUPPORTED
    # row permutation: overlapping buffers, d
    assert lib.svg2_gather_rows(1, 100, 128, 4096, 256, 4096 + 256, None) == \
        svg.SVG_ERR_INVALID_ARG
    assert lib.svg2_scatter_rows(1, 100, 96, 4096, 256, 1 << 20, None) == \
        svg.SVG_ERR_UNSUPPORTED
    # attention on sorted layouts: d and block_k
    assert lib.svg2_sparse_attention(1, 1000, 96, 128, ctypes.c_float(0.1), *([256] * 6), None,
                                     None) == svg.SVG_ERR_UNSUPPORTED
    # SVG-EAR: Ck a multiple of 16 in [16, 256]; workspace size
    ews = ctypes.c_size_t()
    assert lib.svg2_ear_workspace_bytes(2, 128, 64, ctypes.byref(ews)) == svg.SVG_OK
    assert ews.value >= 2 * 64 * 128 * 2 * 2
    comp = lib.svg2_ear_compensate
    assert comp(2, 1000, 128, 40, 128, ctypes.c_float(0.1), *([256] * 9), ews.value, None) == \
        svg.SVG_ERR_UNSUPPORTED
    assert comp(2, 1000, 128, 64, 128, ctypes.c_float(0.1), *([256] * 9), ews.value - 1,
                None) == svg.SVG_ERR_CAPACITY
