"""Small seeded model/input builders shared by the tests (no block arithmetic)."""

from __future__ import annotations

import numpy as np
import torch


def rand_weights(layers, d, ffn, N, seed=0, dtype=torch.float32, gain_std=0.1, experts=0):
    """Random weights in the library's layout, ~N(0, 1/fan_in), gains 1+0.1N(0,1);
    with experts = E > 0 also a sparse-MoE S-side FFN: router [layers][E][d],
    expert W1 [layers][E][ffn][d] and W2 [layers][E][d][ffn]."""
    g = torch.Generator().manual_seed(seed)

    def m(shape, fan):
        return (torch.randn(shape, generator=g) * fan ** -0.5).to(dtype)

    def gain(shape):
        return (1.0 + gain_std * torch.randn(shape, generator=g)).to(dtype)

    w = {
        "Wqkv_s": m((layers, 3 * d, d), d), "Wo_s": m((layers, d, d), d),
        "W1_s": m((layers, ffn, d), d), "W2_s": m((layers, d, ffn), ffn),
        "g1_s": gain((layers, d)), "g2_s": gain((layers, d)),
        "Wqkv_ns": m((layers, N, 3 * d, d), d), "Wo_ns": m((layers, N, d, d), d),
        "W1_ns": m((layers, N, ffn, d), d), "W2_ns": m((layers, N, d, ffn), ffn),
        "g1_ns": gain((layers, N, d)), "g2_ns": gain((layers, N, d)),
    }
    if experts:
        w["W_router"] = m((layers, experts, d), d)
        w["W1_moe"] = m((layers, experts, ffn, d), d)
        w["W2_moe"] = m((layers, experts, d, ffn), ffn)
    return w


def rand_inputs(U, C, L0, N, d, seed=1, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    S = torch.randn((U, L0, d), generator=g).to(dtype)
    ns = torch.randn((U, C, N, d), generator=g).to(dtype)
    return S, ns


def to_lists(w):
    return {k: v.double().tolist() for k, v in w.items()}


def f64(t):
    return t.double().numpy() if hasattr(t, "double") else np.asarray(t, dtype=np.float64)
