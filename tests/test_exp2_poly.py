"""The FMA-pipe 2^x used for part of the attention softmax's exponentials
(range reduction by the 1.5 * 2^23 rounding trick, cubic from ot_exp2_poly.h,
exponent-field add), evaluated bit for bit as the kernel does in fp32 and
checked against 2^x."""

import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "unified_transformer_recommender_onetrans_b200", "csrc", "ot_exp2_poly.h")


def _coeffs():
    txt = open(HDR).read()
    return [np.float32(float(re.search(rf"OT_EXP2_C{k} ([0-9.eE+-]+)f", txt).group(1)))
            for k in range(4)]


def poly_exp2(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    M = np.float32(12582912.0)
    t = (x + M).astype(np.float32)
    f = (x - (t - M)).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (f * p + c1).astype(np.float32)
    p = (f * p + c0).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_on_softmax_range():
    # the softmax passes x = s*c - m <= 2^8 above the reference max, and
    # anything down to where p underflows
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 8e-5


def test_integers_and_halves():
    x = np.arange(-120, 9).astype(np.float32)
    rel = poly_exp2(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0
    assert np.max(np.abs(rel)) < 8e-5          # n exact, f = 0
    h = (np.arange(-120, 8) + 0.5).astype(np.float32)  # ties: n rounds to even
    rel = poly_exp2(h).astype(np.float64) / np.exp2(h.astype(np.float64)) - 1.0
    assert np.max(np.abs(rel)) < 8e-5


def test_clamped_tail_is_tiny_and_positive():
    x = np.array([-126.0, -200.0, -1e30], dtype=np.float32)
    y = poly_exp2(x)
    assert np.all(y > 0) and np.all(y < 2e-38)
