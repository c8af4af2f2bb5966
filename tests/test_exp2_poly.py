"""The FMA-pipe 2^x building block (csrc/exp2_poly.cuh), which no shipped
kernel calls; it is kept with its device self test.

CPU: the header's coefficients are the ones the Remez fit in csrc/exp2_fit.py
derives, and a bit-exact numpy model of the device routine (same fp32
operations, same exponent-field addition) stays within the stated relative
error against exact 2^x.  GPU: the device routine against exact 2^x and
against the hardware ex2.approx, through bsa_selftest_exp2."""
import importlib.util
import math
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_variable_b200", "csrc")
BOUND = 7.5e-5  # the fit's relative error in fp32 Horner evaluation, rounded up


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_fit", os.path.join(CSRC, "exp2_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coefficients():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return [float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f;", text).group(1)) for k in range(4)]


def _model(x):
    """numpy model of exp2_poly: fp32 throughout, exponent added as bits."""
    c = [np.float32(v) for v in _header_coefficients()]
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)  # fmaf rounds once; these round twice, so
    p = (p * f + c[1]).astype(np.float32)     # the model's error is a slight upper bound
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return np.where(x >= np.float32(128.0), np.float32(np.inf), bits.view(np.float32))


def test_header_coefficients_are_the_remez_fit():
    fit = _fit_module()
    assert _header_coefficients() == fit.fp32_coefficients()
    assert fit.max_rel_error(fit.fp32_coefficients()) <= BOUND


def test_model_relative_error_over_the_softmax_range():
    # the softmax arguments: scale*log2(e)*s - m, at most the rescale threshold
    # (8) above 0, and anything below
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001, dtype=np.float32),
                        np.float32([0.0, -0.5, 0.5, -1.5, 8.0, -125.0])])
    y = _model(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert float(rel.max()) <= BOUND + 2e-7  # + the model's extra fp32 roundings
    # exact powers of two of the integer part: 2^n * p(0)
    assert _model(np.float32([3.0]))[0] == np.float32(8.0 * np.float32(_header_coefficients()[0]))


def test_model_overflow_is_inf_and_top_range_is_accurate():
    """x >= 128 overflows to +inf (as the hardware exponential does); just
    below, the exponent field still holds the exact power of two."""
    with np.errstate(over="ignore"):
        y = _model(np.float32([128.0, 128.5, 200.0, np.inf]))
    assert np.all(np.isposinf(y))
    x = np.linspace(120.0, 127.99, 10001, dtype=np.float32)
    rel = np.abs(_model(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert float(rel.max()) <= BOUND + 2e-7


def test_model_underflow_is_tiny_and_positive():
    y = _model(np.float32([-126.0, -127.0, -200.0, -np.inf]))
    assert np.all(y > 0) and np.all(y < 2.0 ** -125)


@pytest.mark.gpu
def test_device_exp2_poly_against_exact_and_mufu():
    import block_sparse_variable_b200 as bsa
    x = torch.cat([torch.linspace(-125.0, 9.0, 1_000_001), torch.tensor([0.0, 0.5, -0.5, 8.0])])
    xd = x.cuda()
    yp, ym = bsa.bsa_selftest_exp2(xd)
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel_poly = float((yp.cpu().double() / exact - 1).abs().max())
    rel_mufu = float((ym.cpu().double() / exact - 1).abs().max())
    assert rel_poly <= BOUND, rel_poly
    assert rel_mufu <= 1e-6, rel_mufu
    # the device routine is the numpy model up to fmaf's single rounding
    model = torch.from_numpy(_model(x.numpy()))
    assert float((yp.cpu() / model - 1).abs().max()) <= 4 * 2.0 ** -24
    tails = bsa.bsa_selftest_exp2(torch.tensor([-126.0, -300.0, -math.inf], device="cuda"))
    torch.cuda.synchronize()
    assert bool((tails[0] > 0).all()) and bool((tails[0] < 2.0 ** -125).all())
    assert float(tails[1][2]) == 0.0
    top = bsa.bsa_selftest_exp2(torch.tensor([127.9, 128.0, 129.5, math.inf], device="cuda"))
    torch.cuda.synchronize()
    assert math.isfinite(float(top[0][0])) and bool(torch.isposinf(top[0][1:]).all())
