"""The GELU polynomial compiled into the GEMM epilogues (ot_gelu_poly.h) is
checked here against the exact-erf GELU, z * Phi(z), evaluated in fp32 the
way the kernel evaluates it (clamp, Horner, one FMA, one multiply)."""

import os
import re

import numpy as np
from scipy.special import erf

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "unified_transformer_recommender_onetrans_b200", "csrc", "ot_gelu_poly.h")


def _coeffs():
    txt = open(HDR).read()
    zc = float(re.search(r"OT_GELU_ZC ([0-9.]+)f", txt).group(1))
    body = txt[txt.index("{") + 1: txt.index("}")]
    c = [np.float32(float(x.strip().rstrip("f"))) for x in body.split(",") if x.strip()]
    return zc, c


def test_gelu_polynomial_error_below_bf16_resolution():
    zc, c = _coeffs()
    z = np.linspace(-20, 20, 800001).astype(np.float32)
    zcl = np.clip(z, -zc, zc)
    v = (zcl * zcl) * np.float32(1.0 / (zc * zc))
    p = np.full_like(z, c[-1])
    for ck in c[-2::-1]:
        p = (p * v + ck).astype(np.float32)
    g = z * (zcl * p + np.float32(0.5))
    exact = z.astype(np.float64) * 0.5 * (1 + erf(z.astype(np.float64) / np.sqrt(2)))
    assert np.max(np.abs(g - exact)) < 1e-4
    # and the special values: GELU(0) = 0, odd part symmetry Phi(z) + Phi(-z) = 1
    assert g[np.argmin(np.abs(z))] == 0.0
