"""The GELU compiled into the tensor-core GEMM epilogues (ot_gelu_fit.h),
z * (1/2 + 1/2 tanh(z (A + B z^2))), checked against the exact-erf GELU,
z * Phi(z), evaluated in fp32 the way the kernel evaluates it.  The hardware
tanh is modelled as an exact tanh perturbed by its documented relative error
(about 2^-11), in both directions."""

import os
import re

import numpy as np
from scipy.special import erf

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "unified_transformer_recommender_onetrans_b200", "csrc", "ot_gelu_fit.h")
TANH_REL = 2.0 ** -10.9


def _coeffs():
    txt = open(HDR).read()
    a = float(re.search(r"OT_GELU_A ([0-9.eE+-]+)f", txt).group(1))
    b = float(re.search(r"OT_GELU_B ([0-9.eE+-]+)f", txt).group(1))
    return np.float32(a), np.float32(b)


def _gelu_kernel_form(z, tanh_scale=1.0):
    a, b = _coeffs()
    z = z.astype(np.float32)
    u = z * (b * (z * z) + a)
    t = (np.tanh(u) * np.float32(tanh_scale)).astype(np.float32)
    hz = np.float32(0.5) * z
    return hz * t + hz


def _exact(z):
    z = z.astype(np.float64)
    return z * 0.5 * (1 + erf(z / np.sqrt(2)))


def test_gelu_fit_within_bf16_resolution():
    z = np.linspace(-20, 20, 800001).astype(np.float32)
    ex = _exact(z)
    for sc in (1.0, 1.0 + TANH_REL, 1.0 - TANH_REL):
        g = _gelu_kernel_form(z, sc).astype(np.float64)
        # Phi error: fit (1.4e-4) + hardware tanh (half of 2^-10.9)
        err_phi = np.abs(g - ex) / np.maximum(np.abs(z.astype(np.float64)), 1e-30)
        assert err_phi[np.abs(z) > 1e-3].max() < 1.4e-4 + 0.5 * TANH_REL + 1e-6
        # positive side: relative error below half a bf16 ulp (2^-9)
        pos = z > 0.05
        assert (np.abs(g - ex)[pos] / ex[pos]).max() < 2.0 ** -9


def test_gelu_fit_special_values():
    z = np.array([0.0, 30.0, -30.0, 1e-6], dtype=np.float32)
    g = _gelu_kernel_form(z)
    assert g[0] == 0.0                      # GELU(0) = 0
    assert g[1] == np.float32(30.0)         # saturates to z for large z
    assert g[2] == 0.0                      # and to 0 for very negative z
    assert abs(g[3] - 0.5e-6) < 1e-12       # slope 1/2 at the origin


def test_gelu_fit_is_odd_symmetric_part():
    # GELU(z) - GELU(-z) = z holds exactly for the form (tanh is odd)
    z = np.linspace(-8, 8, 10001).astype(np.float32)
    d = _gelu_kernel_form(z).astype(np.float64) - _gelu_kernel_form(-z).astype(np.float64)
    assert np.max(np.abs(d - z)) < 4 * np.finfo(np.float32).eps * 8
