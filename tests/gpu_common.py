"""Shared helpers of the GPU parity tests: build a library model from CPU
weights, run the oracle on the same inputs, compare per output tensor."""

from __future__ import annotations

import numpy as np
import torch

import unified_transformer_recommender_onetrans_b200 as ot
from oracle import oracle as O
from unified_transformer_recommender_onetrans_b200.binding import MOE_WEIGHT_NAMES, WEIGHT_NAMES

# Max relative L2 error per output tensor (stated workload tolerances).
TOL = {"f32": 1e-5, "bf16": 2e-2, "fp8": 6e-2}


def make_model(w, *, layers, d, heads, ffn, n_ns, L0, q, F=0, dtype="bf16", eps=1e-6,
               full_attn=False, moe_experts=0, moe_topk=1):
    dev = {k: w[k].cuda() for k in WEIGHT_NAMES + MOE_WEIGHT_NAMES if k in w and w[k] is not None}
    return ot.Model(layers=layers, d=d, heads=heads, ffn=ffn, n_ns=n_ns, L0=L0, q=q, F=F,
                    eps=eps, dtype=dtype, weights=dev, full_attn=full_attn,
                    moe_experts=moe_experts, moe_topk=moe_topk)


def model_of(wl, w, q=None):
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers) if q is None else q
    return make_model(w, layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                      L0=wl.L0, q=q, F=wl.F, dtype=wl.dtype, eps=wl.eps)


def oracle_cfg(m: ot.Model, fp8=False):
    c = O.Config(m.layers, m.d, m.heads, m.ffn, m.n_ns, m.L0, list(m.q), m.eps, fp8)
    c.full_attn = m.full_attn
    c.moe_experts, c.moe_topk = m.moe_experts, m.moe_topk
    return c


def kv_errors(m, kv_gpu_users, kv_oracle_users, cfg):
    """Relative L2 per layer for K and V of every given user."""
    errs = {}
    for l in range(m.layers):
        Kg = torch.stack([m.kv_layer(kv_gpu_users[i], l)[0] for i in range(len(kv_gpu_users))])
        Vg = torch.stack([m.kv_layer(kv_gpu_users[i], l)[1] for i in range(len(kv_gpu_users))])
        Ko = np.stack([O.kv_layer(cfg, kv_oracle_users[i], l)[0] for i in range(len(kv_gpu_users))])
        Vo = np.stack([O.kv_layer(cfg, kv_oracle_users[i], l)[1] for i in range(len(kv_gpu_users))])
        errs[f"K{l}"] = O.rel_l2(Kg.double().cpu().numpy(), Ko)
        errs[f"V{l}"] = O.rel_l2(Vg.double().cpu().numpy(), Vo)
    return errs


def assert_within(errs: dict, tol: float):
    worst = max(errs.values())
    assert worst <= tol, {k: f"{v:.3e}" for k, v in errs.items() if v > tol} or worst
