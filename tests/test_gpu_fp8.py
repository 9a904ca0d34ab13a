"""GPU parity of the FP8 (e4m3) projection path against the oracle's FP8 mode
(same quantisation rule applied to the oracle's own fp64 values; tolerance
6e-2 max relative L2 per output tensor), plus the long-sequence serving
workload with its embedding gather."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import unified_transformer_recommender_onetrans_b200 as ot
from gpu_common import TOL, assert_within, kv_errors, make_model, oracle_cfg
from helpers import rand_inputs, rand_weights
from oracle import oracle as O
from synth import WORKLOADS, gen_auto_split_features, gen_embedding_table, gen_weights, gen_zipf_ids

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()


def test_fp8_small_parity_and_drift():
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=201, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 7, 300, 5, 128, seed=202, dtype=torch.bfloat16)
    m = make_model(w, dtype="fp8", **shapes)
    kv = m.new_kv_cache(3)
    s_tail, ns_out = m.full_forward(S.cuda(), ns.cuda(), kv=kv)
    m.poll()
    cfg8 = oracle_cfg(m, fp8=True)
    kv_o, s_o = O.encode_user(cfg8, w, S)
    ns_o = O.score_candidates(cfg8, w, kv_o, ns)
    errs = {"s_tail": O.rel_l2(s_tail.double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(ns_out.double().cpu().numpy(), ns_o)}
    errs.update(kv_errors(m, kv, kv_o, cfg8))
    assert_within(errs, TOL["fp8"])
    # diagnostic: drift against the unquantised oracle stays inside the format's bound
    cfg64 = oracle_cfg(m, fp8=False)
    kv64, s64 = O.encode_user(cfg64, w, S)
    drift = O.rel_l2(s_tail.double().cpu().numpy(), s64)
    assert drift < 2 * 2.0 ** -4, drift


def test_fp8_rejects_cuda_core_path():
    w = rand_weights(1, 128, 256, 2, seed=3, dtype=torch.bfloat16)
    m = make_model(w, layers=1, d=128, heads=2, ffn=256, n_ns=2, L0=64, q=[64], dtype="fp8")
    with pytest.raises(ot.OtError):
        m.set_kernel_path(1)


def test_long_fp8_serving_sampled():
    """8192-token users gathered from a Zipf-sampled 2^20-row table, encoded
    once, 256 candidates scored per user; oracle on 1 user x 4 candidates."""
    wl = WORKLOADS["long_fp8"]
    w = gen_weights(wl)
    table = gen_embedding_table(wl)
    ids = gen_zipf_ids(wl)
    x = gen_auto_split_features(wl)
    m = make_model(w, layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                   L0=wl.L0, q=ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers), F=wl.F,
                   dtype="fp8")
    tdev = table.cuda()
    S = ot.embed_gather(tdev, ids.cuda())
    kv, _ = m.encode_user(S, want_s_tail=False)
    ns = m.auto_split(x.cuda())
    out = m.score_candidates(kv, ns)
    m.poll()
    u, cands = 5, [0, 77, 128, 255]
    S_u = table[ids[u]][None]
    assert torch.equal(S[u].cpu(), S_u[0])
    cfg8 = oracle_cfg(m, fp8=True)
    kv_o, _ = O.encode_user(cfg8, w, S_u)
    ns_o = O.auto_split(x[u:u + 1, cands], w["W_split"], wl.n_ns, wl.d)
    out_o = O.score_candidates(cfg8, w, kv_o, ns_o)
    errs = {"ns_out": O.rel_l2(out[u, cands].double().cpu().numpy(), out_o[0])}
    errs.update(kv_errors(m, kv[u:u + 1], kv_o, cfg8))
    assert_within(errs, TOL["fp8"])
