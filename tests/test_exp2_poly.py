"""The FMA-pipe exp2 used by the attention softmax.

CPU: the committed coefficients are what the Remez fit script produces, and
their fp32 Horner evaluation meets the stated relative-error bound.
GPU: the device routine (range reduction + cubic + exponent scaling) against
exact 2^y over the range the kernels use.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_dit_spatial_b200", "csrc")


def _header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly_coeffs.h")).read()
    c = [float(v) for _, v in sorted(re.findall(r"kExp2Poly(\d) = ([0-9.e+-]+)f;", text))]
    bound = float(re.search(r"kExp2PolyMaxRelErr = ([0-9.e+-]+)f;", text).group(1))
    return np.array(c, dtype=np.float32), bound


def test_coefficients_reproduce_from_the_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c = fit.remez(fit.DEGREE).astype(np.float32)
    got, bound = _header_coeffs()
    assert np.array_equal(c, got)
    assert fit.fp32_error(got) <= bound * 1.0001
    assert bound < 1e-4  # far below bf16's relative spacing (2^-8)


def test_cubic_is_close_to_the_taylor_series():
    # a plausible mix-up (wrong order of coefficients, ln 2 missing) fails this
    c, _ = _header_coeffs()
    ln2 = np.log(2.0)
    np.testing.assert_allclose(c, [1.0, ln2, ln2 ** 2 / 2, ln2 ** 3 / 6], rtol=0.02)


@pytest.mark.gpu
def test_device_exp2_against_exact():
    import torch
    import video_dit_spatial_b200 as svg
    svg.load()
    _, bound = _header_coeffs()
    g = torch.Generator().manual_seed(3)
    y = torch.cat([torch.rand(1 << 20, generator=g) * 133.0 - 125.0,
                   torch.tensor([-125.0, -124.5, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0, 7.99, 8.0]),
                   torch.arange(-125, 8, dtype=torch.float32) + 0.5])
    low = torch.tensor([-1e30, -1000.0, -200.0, -126.0, -125.01])
    yd = torch.cat([y, low]).cuda()
    out = torch.empty_like(yd)
    svg.svg_selftest_exp2(yd, out)
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    exact = np.exp2(y.double().numpy())
    rel = np.abs(got[:y.numel()] / exact - 1.0)
    assert rel.max() <= bound + 4 * 2.0 ** -24, rel.max()
    tail = got[y.numel():]
    assert np.all(tail > 0) and np.all(tail <= 2.0 ** -124)
