"""GPU parity of the FP8 (e4m3) projection path against the oracle's FP8
modes: per-tensor scales (the product rule, scales from the oracle's own
calibration) and per-row scales (the calibration pass), tolerance 6e-2 max
relative L2 per output tensor; the calibration's amax against the oracle's;
and the long-sequence serving workload with its embedding gather."""

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

SMALL = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()


@pytest.fixture(scope="module")
def small():
    w = rand_weights(3, 128, 256, 5, seed=201, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 7, 300, 5, 128, seed=202, dtype=torch.bfloat16)
    return w, S, ns


def _run(m, S, ns):
    kv = m.new_kv_cache(S.shape[0])
    s_tail, ns_out = m.full_forward(S.cuda(), ns.cuda(), kv=kv)
    m.poll()
    return s_tail, ns_out, kv


def _errs(m, cfg, w, S, ns, s_tail, ns_out, kv):
    kv_o, s_o = O.encode_user(cfg, w, S)
    ns_o = O.score_candidates(cfg, w, kv_o, ns)
    errs = {"s_tail": O.rel_l2(s_tail.double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(ns_out.double().cpu().numpy(), ns_o)}
    errs.update(kv_errors(m, kv, kv_o, cfg))
    return errs


def test_fp8_per_row_parity_and_drift(small):
    """No scales set: every projection input row is quantised with its own
    scale, against the oracle's per-row mode."""
    w, S, ns = small
    m = make_model(w, dtype="fp8", **SMALL)
    s_tail, ns_out, kv = _run(m, S, ns)
    assert_within(_errs(m, oracle_cfg(m, fp8=O.FP8_ROW), w, S, ns, s_tail, ns_out, kv), TOL["fp8"])
    # diagnostic: drift against the unquantised oracle stays inside the format's bound
    kv64, s64 = O.encode_user(oracle_cfg(m), w, S)
    drift = O.rel_l2(s_tail.double().cpu().numpy(), s64)
    assert drift < 2 * 2.0 ** -4, drift


def test_fp8_per_tensor_parity_and_drift(small):
    """Per-tensor scales from the oracle's calibration on two of the users:
    the GPU model with those scales against the oracle's per-tensor mode with
    the same scales (values beyond a calibrated amax saturate on both)."""
    w, S, ns = small
    m = make_model(w, dtype="fp8", **SMALL)
    scales, _ = O.calibrate(oracle_cfg(m), w, S[:2], ns[:2])
    m.set_act_scales(scales)
    s_tail, ns_out, kv = _run(m, S, ns)
    cfg = oracle_cfg(m, fp8=O.FP8_TENSOR)
    cfg.act_scale = scales
    assert_within(_errs(m, cfg, w, S, ns, s_tail, ns_out, kv), TOL["fp8"])
    kv64, s64 = O.encode_user(oracle_cfg(m), w, S)
    drift = O.rel_l2(s_tail.double().cpu().numpy(), s64)
    assert drift < 2 * 2.0 ** -4, drift
    # cached scoring with the same scales gives the full forward's NS outputs
    sc = m.score_candidates(kv, ns.cuda())
    m.poll()
    assert torch.equal(sc, ns_out)
    # back to per-row scales: the per-row result again
    m.set_act_scales(None)
    s_row, _, _ = _run(m, S, ns)
    m2 = make_model(w, dtype="fp8", **SMALL)
    s_row2, _, _ = _run(m2, S, ns)
    assert torch.equal(s_row, s_row2)


def test_fp8_calibrate_matches_oracle(small):
    """ot_fp8_calibrate's per-tensor amax (per-row FP8 forward of the sample,
    max |x| of every projection input) against the oracle's calibration of
    the same sample: the maxima of values that agree within the FP8
    tolerance, so within it too."""
    w, S, ns = small
    m = make_model(w, dtype="fp8", **SMALL)
    amax = m.fp8_calibrate(S[:2].cuda(), ns[:2].cuda())
    m.poll()
    g = amax.double().cpu().numpy()
    _, want = O.calibrate(oracle_cfg(m), w, S[:2], ns[:2])
    assert np.all(g > 0)
    rel = np.abs(g - want) / want
    assert rel.max() <= TOL["fp8"], rel.max()
    # accumulating a second batch only raises the maxima
    amax2 = m.fp8_calibrate(S[2:].cuda(), ns[2:].cuda(), amax=amax.clone())
    m.poll()
    assert torch.all(amax2 >= amax)
    with pytest.raises(ot.OtError):
        make_model(w, **SMALL).set_act_scales(np.ones((3, 6, 4)))   # not an fp8 model


def test_fp8_rejects_cuda_core_path():
    w = rand_weights(1, 128, 256, 2, seed=3, dtype=torch.bfloat16)
    m = make_model(w, layers=1, d=128, heads=2, ffn=256, n_ns=2, L0=64, q=[64], dtype="fp8")
    with pytest.raises(ot.OtError):
        m.set_kernel_path(1)


def test_long_fp8_serving_sampled():
    """8192-token users gathered from a Zipf-sampled 2^20-row table, encoded
    once, 256 candidates scored per user with per-tensor scales; the scales
    come from the oracle's calibration of a shorter sample (the first 2048
    rows of one user, pyramid 2048 -> 16, four candidates); oracle on 1 user
    x 4 candidates at full length with the same scales."""
    wl = WORKLOADS["long_fp8"]
    w = gen_weights(wl)
    table = gen_embedding_table(wl)
    ids = gen_zipf_ids(wl)
    x = gen_auto_split_features(wl)
    m = make_model(w, layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                   L0=wl.L0, q=ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers), F=wl.F,
                   dtype="fp8")
    u, cands = 5, [0, 77, 128, 255]
    S_u = table[ids[u]][None]
    ns_u = O.auto_split(x[u:u + 1, cands], w["W_split"], wl.n_ns, wl.d)
    cal = O.Config(wl.layers, wl.d, wl.heads, wl.ffn, wl.n_ns, 2048,
                   ot.pyramid_schedule(2048, wl.q_end, wl.layers), wl.eps)
    scales, _ = O.calibrate(cal, w, S_u[:, :2048], ns_u)
    m.set_act_scales(scales)
    tdev = table.cuda()
    S = ot.embed_gather(tdev, ids.cuda())
    kv, _ = m.encode_user(S, want_s_tail=False)
    ns = m.auto_split(x.cuda())
    out = m.score_candidates(kv, ns)
    m.poll()
    assert torch.equal(S[u].cpu(), S_u[0])
    cfg8 = oracle_cfg(m, fp8=O.FP8_TENSOR)
    cfg8.act_scale = scales
    kv_o, _ = O.encode_user(cfg8, w, S_u)
    out_o = O.score_candidates(cfg8, w, kv_o, ns_u)
    errs = {"ns_out": O.rel_l2(out[u, cands].double().cpu().numpy(), out_o[0])}
    errs.update(kv_errors(m, kv[u:u + 1], kv_o, cfg8))
    assert_within(errs, TOL["fp8"])
