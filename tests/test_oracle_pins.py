"""Pins of the CPU oracle to things other than itself (no GPU needed).

* brute force: an independent pure-Python token-by-token implementation;
* textbook reduction: with every NS parameter set equal to the S set the S/NS
  mask is the plain causal mask over [S; NS], so each block must equal a
  pre-norm causal Transformer layer built from torch's library routines
  (scaled_dot_product_attention(is_causal=True), rms_norm, gelu) in fp64;
* closed forms: uniform attention, identity blocks, single-key attention,
  RMSNorm scale invariance;
* the invariants the pages' design rests on: causality, pyramid
  consistency, KV-cache equivalence, candidate independence, S-side
  independence from NS input;
* e4m3 rounding against torch's float8_e4m3fn cast; both FP8 rules (per-row
  and per-tensor scales) against the brute force, exact results on
  representable operands, a hand-worked row, the scale granularity and the
  calibration amax;
* Auto-Split and embedding gather against numpy;
* the brute force again on random tiny shapes (hypothesis, derandomized):
  causal, full attention, the mixture of experts, both FP8 rules and the
  sequence append; the textbook reduction on random shapes; and the
  gradient oracle against finite differences.
"""

from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

from brute_force import run_candidate
from helpers import rand_inputs, rand_weights, to_lists
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def cfg_of(layers, d, heads, ffn, N, L0, q, eps=1e-6, fp8=O.FP8_OFF, act_scale=None):
    return O.Config(layers, d, heads, ffn, N, L0, list(q), eps, fp8, act_scale)


TINY_CASES = [
    # layers, d, heads, ffn, N, L0, q schedule, U, C
    (1, 8, 1, 16, 1, 1, [1], 1, 1),
    (1, 8, 2, 12, 3, 2, [2], 1, 2),
    (2, 8, 2, 16, 3, 7, [5, 2], 2, 2),
    (3, 12, 2, 20, 1, 33, [33, 9, 1], 1, 2),
    (2, 16, 1, 32, 3, 33, [7, 7], 1, 1),
]


@pytest.mark.parametrize("case", TINY_CASES)
def test_brute_force_matches_oracle(case):
    layers, d, H, f, N, L0, q, U, Cn = case
    w = rand_weights(layers, d, f, N, seed=L0 + d)
    S, ns = rand_inputs(U, Cn, L0, N, d, seed=7 * L0 + N)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns)
    wl = to_lists(w)
    for u in range(U):
        for c in range(Cn):
            bs, bns, bkv = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                         q, H, 1e-6)
            np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(js[u, c], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)
            np.testing.assert_allclose(jns[u, c], np.array(bns), rtol=0, atol=1e-12)
            for l, (K, V) in enumerate(bkv):
                Ko, Vo = O.kv_layer(cfg, kv[u], l)
                np.testing.assert_allclose(Ko, np.array(K), rtol=0, atol=1e-12)
                np.testing.assert_allclose(Vo, np.array(V), rtol=0, atol=1e-12)


def _torch_causal_layer(x, Wqkv, Wo, W1, W2, g1, g2, H, eps, causal=True):
    """Pre-norm causal (or, causal=False, bidirectional) Transformer layer from
    torch library routines (fp64)."""
    T, d = x.shape
    hd = d // H
    xn = Fnn.rms_norm(x, (d,), weight=g1, eps=eps)
    qkv = xn @ Wqkv.T
    q, k, v = qkv.split(d, dim=-1)
    heads = lambda t: t.view(T, H, hd).transpose(0, 1)  # noqa: E731
    a = Fnn.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=causal)
    h = x + a.transpose(0, 1).reshape(T, d) @ Wo.T
    return h + Fnn.gelu(Fnn.rms_norm(h, (d,), weight=g2, eps=eps) @ W1.T) @ W2.T


@pytest.mark.parametrize("pyramid", [False, True])
def test_textbook_reduction_causal_transformer(pyramid):
    layers, d, H, f, N, L0 = 2, 16, 2, 32, 3, 11
    q = [7, 3] if pyramid else [L0, L0]
    w = rand_weights(layers, d, f, N, seed=3, dtype=torch.float64)
    for name in ("Wqkv", "Wo", "W1", "W2", "g1", "g2"):
        w[name + "_ns"] = w[name + "_s"][:, None].expand(-1, N, *w[name + "_s"].shape[1:]).clone()
    S, ns = rand_inputs(1, 2, L0, N, d, seed=5, dtype=torch.float64)
    # float32-representable inputs: the oracle stores inputs as float32
    w = {k: v.float().double() for k, v in w.items()}
    S, ns = S.float().double(), ns.float().double()
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    for c in range(2):
        x = torch.cat([S[0], ns[0, c]])
        L = L0
        for l in range(layers):
            y = _torch_causal_layer(x, w["Wqkv_s"][l], w["Wo_s"][l], w["W1_s"][l], w["W2_s"][l],
                                    w["g1_s"][l], w["g2_s"][l], H, 1e-6)
            # bottom-right alignment: keep the last q S rows, then all NS rows
            x = torch.cat([y[L - q[l]:L], y[L:]])
            L = q[l]
        np.testing.assert_allclose(s_out[0], x[:L].numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(ns_out[0, c], x[L:].numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("pyramid", [False, True])
def test_textbook_reduction_full_attention(pyramid):
    """Full attention with every NS parameter set equal to the S set: each
    block is a plain bidirectional pre-norm Transformer layer over [S; NS]
    (scaled_dot_product_attention with is_causal=False), and with a pyramid
    the kept rows are the tail S rows and the NS rows of that layer."""
    layers, d, H, f, N, L0 = 2, 16, 2, 32, 3, 11
    q = [7, 3] if pyramid else [L0, L0]
    w = rand_weights(layers, d, f, N, seed=4, dtype=torch.float64)
    for name in ("Wqkv", "Wo", "W1", "W2", "g1", "g2"):
        w[name + "_ns"] = w[name + "_s"][:, None].expand(-1, N, *w[name + "_s"].shape[1:]).clone()
    S, ns = rand_inputs(1, 2, L0, N, d, seed=6, dtype=torch.float64)
    w = {k: v.float().double() for k, v in w.items()}
    S, ns = S.float().double(), ns.float().double()
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.full_attn = True
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns)
    for c in range(2):
        x = torch.cat([S[0], ns[0, c]])
        L = L0
        for l in range(layers):
            y = _torch_causal_layer(x, w["Wqkv_s"][l], w["Wo_s"][l], w["W1_s"][l], w["W2_s"][l],
                                    w["g1_s"][l], w["g2_s"][l], H, 1e-6, causal=False)
            x = torch.cat([y[L - q[l]:L], y[L:]])
            L = q[l]
        np.testing.assert_allclose(js[0, c], x[:L].numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(jns[0, c], x[L:].numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("case", TINY_CASES[1:4])
def test_brute_force_matches_oracle_full_attention(case):
    """Full attention: the joint oracle against the brute-force token loop
    with its every-key visibility; the split (cached) form refuses it."""
    layers, d, H, f, N, L0, q, U, Cn = case
    w = rand_weights(layers, d, f, N, seed=L0 + d + 2)
    S, ns = rand_inputs(U, Cn, L0, N, d, seed=7 * L0 + N + 2)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.full_attn = True
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns)
    wl = to_lists(w)
    for u in range(U):
        for c in range(Cn):
            bs, bns, bkv = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                         q, H, 1e-6, full=True)
            np.testing.assert_allclose(js[u, c], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(jns[u, c], np.array(bns), rtol=0, atol=1e-12)
            for l, (K, V) in enumerate(bkv):
                Ko, Vo = O.kv_layer(cfg, jkv[u, c], l)
                np.testing.assert_allclose(Ko, np.array(K), rtol=0, atol=1e-12)
                np.testing.assert_allclose(Vo, np.array(V), rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        O.encode_user(cfg, w, S)


def test_full_attention_breaks_the_cache_invariants():
    """What makes full attention uncacheable: S outputs change with the
    candidate's NS input and with later S rows (both are fixed under the
    causal mask); with a single layer and no pyramid the layer-0 K / V still
    do not (they come before any attention)."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=93)
    S, ns = rand_inputs(1, 1, L0, N, d, seed=94)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.full_attn = True
    s1, kv1, n1 = O.full_forward_joint(cfg, w, S, ns)
    ns2 = ns.clone()
    ns2[0, 0, N - 1] += 1.0
    s2, kv2, n2 = O.full_forward_joint(cfg, w, S, ns2)
    assert not np.allclose(s1, s2)
    K1, _ = O.kv_layer(cfg, kv1[0, 0], 0)
    K2, _ = O.kv_layer(cfg, kv2[0, 0], 0)
    assert np.array_equal(K1, K2)
    K1b, _ = O.kv_layer(cfg, kv1[0, 0], 1)
    K2b, _ = O.kv_layer(cfg, kv2[0, 0], 1)
    assert not np.allclose(K1b, K2b)
    S3 = S.clone()
    S3[0, L0 - 1] += 1.0
    s3, _, _ = O.full_forward_joint(cfg, w, S3, ns)
    assert not np.allclose(s1[0, 0, 0], s3[0, 0, 0])


# ----------------------------------------------------------------- sparse MoE
@pytest.mark.parametrize("topk", [1, 2])
@pytest.mark.parametrize("case", TINY_CASES[2:5])
def test_brute_force_matches_oracle_moe(case, topk):
    """The sparse-MoE S-side FFN (router top-k, softmax gates, gated expert
    sum) against the brute-force token loop: split and joint forms."""
    layers, d, H, f, N, L0, q, U, Cn = case
    w = rand_weights(layers, d, f, N, seed=L0 + d + 3, experts=4)
    S, ns = rand_inputs(U, Cn, L0, N, d, seed=7 * L0 + N + 3)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.moe_experts, cfg.moe_topk = 4, topk
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns)
    wl = to_lists(w)
    for u in range(U):
        for c in range(Cn):
            bs, bns, bkv = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                         q, H, 1e-6, moe_topk=topk)
            np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(js[u, c], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)
            for l, (K, V) in enumerate(bkv):
                Ko, Vo = O.kv_layer(cfg, kv[u], l)
                np.testing.assert_allclose(Ko, np.array(K), rtol=0, atol=1e-12)


@pytest.mark.parametrize("topk", [1, 2])
def test_moe_identical_experts_equal_the_dense_ffn(topk):
    """Closed form: with every expert equal to the dense FFN the gates sum to
    one, so the mixture is the dense block whatever the router says."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=101, experts=3)
    w["W1_moe"] = w["W1_s"][:, None].expand(-1, 3, -1, -1).clone()
    w["W2_moe"] = w["W2_s"][:, None].expand(-1, 3, -1, -1).clone()
    S, ns = rand_inputs(1, 2, L0, N, d, seed=102)
    dense = cfg_of(layers, d, H, f, N, L0, q)
    moe = cfg_of(layers, d, H, f, N, L0, q)
    moe.moe_experts, moe.moe_topk = 3, topk
    kv_d, s_d = O.encode_user(dense, w, S)
    kv_m, s_m = O.encode_user(moe, w, S)
    np.testing.assert_allclose(s_m, s_d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(kv_m, kv_d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.score_candidates(moe, w, kv_m, ns),
                               O.score_candidates(dense, w, kv_d, ns), rtol=0, atol=1e-12)


def test_moe_zero_router_picks_the_lowest_experts():
    """Closed form: a zero router ties every logit, so the top-1 expert is
    expert 0 (gate 1) and the top-2 are experts 0 and 1 (gates 1/2 each)."""
    layers, d, H, f, N, L0 = 1, 16, 2, 32, 2, 9
    w = rand_weights(layers, d, f, N, seed=103, experts=4)
    w["W_router"] = torch.zeros_like(w["W_router"])
    S, _ = rand_inputs(1, 1, L0, N, d, seed=104)
    moe1 = cfg_of(layers, d, H, f, N, L0, [L0])
    moe1.moe_experts, moe1.moe_topk = 4, 1
    dense = cfg_of(layers, d, H, f, N, L0, [L0])
    w0 = dict(w, W1_s=w["W1_moe"][:, 0].clone(), W2_s=w["W2_moe"][:, 0].clone())
    np.testing.assert_array_equal(O.encode_user(moe1, w, S)[1], O.encode_user(dense, w0, S)[1])
    moe2 = cfg_of(layers, d, H, f, N, L0, [L0])
    moe2.moe_experts, moe2.moe_topk = 4, 2
    w1 = dict(w, W1_s=w["W1_moe"][:, 1].clone(), W2_s=w["W2_moe"][:, 1].clone())
    y0, y1, y2 = (O.encode_user(c, ww, S)[1] for c, ww in ((dense, w0), (dense, w1), (moe2, w)))
    # y = h + (f0 + f1) / 2 = (y0 + y1) / 2 (both share h)
    np.testing.assert_allclose(y2, (y0 + y1) / 2, rtol=0, atol=1e-12)


def _zero_rows(w, key, rows):
    w[key] = w[key].clone()
    w[key][..., rows, :] = 0


def test_closed_form_uniform_attention_means():
    """W_Q = W_K = 0: every score is 0, so attention is the mean of the visible
    V rows.  With W_O = I and W_2 = 0 each output row is x + that mean."""
    layers, d, H, f, N, L0 = 1, 8, 2, 16, 3, 9
    w = rand_weights(layers, d, f, N, seed=11)
    for key in ("Wqkv_s", "Wqkv_ns"):
        _zero_rows(w, key, slice(0, 2 * d))
    w["Wo_s"] = torch.eye(d).expand(layers, d, d).clone()
    w["Wo_ns"] = torch.eye(d).expand(layers, N, d, d).clone()
    w["W2_s"] = torch.zeros_like(w["W2_s"])
    w["W2_ns"] = torch.zeros_like(w["W2_ns"])
    S, ns = rand_inputs(1, 1, L0, N, d, seed=12)
    cfg = cfg_of(layers, d, H, f, N, L0, [L0])
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    K, V = O.kv_layer(cfg, kv[0], 0)
    assert np.all(K == 0.0)
    Sd = S[0].double().numpy()
    for t in range(L0):
        np.testing.assert_allclose(s_out[0, t], Sd[t] + V[: t + 1].mean(0), atol=1e-13)
    # NS: V_N rows from the private V projection of the normalised NS rows
    x = ns[0, 0].double().numpy()
    VN = []
    for n in range(N):
        xn = x[n] / np.sqrt((x[n] ** 2).mean() + 1e-6) * w["g1_ns"][0, n].double().numpy()
        VN.append(w["Wqkv_ns"][0, n, 2 * d:].double().numpy() @ xn)
    VN = np.array(VN)
    for n in range(N):
        mean = (V.sum(0) + VN[: n + 1].sum(0)) / (L0 + n + 1)
        np.testing.assert_allclose(ns_out[0, 0, n], x[n] + mean, atol=1e-13)


def test_closed_form_identity_blocks_pyramid():
    """W_O = W_2 = 0: every block is the identity on the rows it keeps, so the
    stack returns input rows L0-q_last .. L0-1 exactly and the NS rows
    unchanged."""
    layers, d, H, f, N, L0 = 3, 8, 2, 16, 2, 20
    q = [14, 6, 4]
    w = rand_weights(layers, d, f, N, seed=21)
    for k in ("Wo_s", "Wo_ns", "W2_s", "W2_ns"):
        w[k] = torch.zeros_like(w[k])
    S, ns = rand_inputs(2, 3, L0, N, d, seed=22)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    assert np.array_equal(s_out, S[:, L0 - q[-1]:].double().numpy())
    assert np.array_equal(ns_out, ns.double().numpy())


def test_closed_form_first_query_returns_v0():
    """An S query at t = 0 sees only key 0: its attention output is v_0."""
    layers, d, H, f, N, L0 = 1, 8, 2, 16, 1, 5
    w = rand_weights(layers, d, f, N, seed=31)
    w["Wo_s"] = torch.eye(d).expand(layers, d, d).clone()
    w["W2_s"] = torch.zeros_like(w["W2_s"])
    S, ns = rand_inputs(1, 1, L0, N, d, seed=32)
    cfg = cfg_of(layers, d, H, f, N, L0, [L0])
    kv, s_out = O.encode_user(cfg, w, S)
    K, V = O.kv_layer(cfg, kv[0], 0)
    np.testing.assert_allclose(s_out[0, 0], S[0, 0].double().numpy() + V[0], atol=1e-14)


def test_closed_form_rmsnorm_scale_invariance():
    """K/V of layer 0 are projections of RMSNorm(x), which ignores a positive
    scale of x up to eps."""
    layers, d, H, f, N, L0 = 1, 16, 2, 32, 1, 6
    w = rand_weights(layers, d, f, N, seed=41)
    S, _ = rand_inputs(1, 1, L0, N, d, seed=42)
    cfg = cfg_of(layers, d, H, f, N, L0, [L0], eps=1e-30)
    kv1, _ = O.encode_user(cfg, w, S)
    kv2, _ = O.encode_user(cfg, w, S * 4.0)
    np.testing.assert_allclose(kv1, kv2, rtol=1e-13, atol=1e-14)


def _small():
    layers, d, H, f, N, L0 = 2, 16, 2, 32, 3, 13
    return layers, d, H, f, N, L0, [9, 4]


def test_invariant_causal():
    """Perturbing S row j leaves S K/V rows < j of layer 0 and the S outputs
    of rows < j (no pyramid) unchanged; rows >= j do change."""
    layers, d, H, f, N, L0, _ = _small()
    q = [L0, L0]
    w = rand_weights(layers, d, f, N, seed=51)
    S, _ = rand_inputs(1, 1, L0, N, d, seed=52)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, s_out = O.encode_user(cfg, w, S)
    j = 6
    S2 = S.clone()
    S2[0, j] += 1.0
    kv2, s_out2 = O.encode_user(cfg, w, S2)
    assert np.array_equal(s_out[0, :j], s_out2[0, :j])
    assert not np.allclose(s_out[0, j:], s_out2[0, j:])
    for l in range(layers):
        K1, V1 = O.kv_layer(cfg, kv[0], l)
        K2, V2 = O.kv_layer(cfg, kv2[0], l)
        assert np.array_equal(K1[:j], K2[:j]) and np.array_equal(V1[:j], V2[:j])


def test_invariant_pyramid_consistency():
    """A layer with query tail q equals the matching rows of the same layer
    with every row as a query, on the same input."""
    layers, d, H, f, N, L0, _ = _small()
    w = rand_weights(1, d, f, N, seed=61)
    S, ns = rand_inputs(1, 2, L0, N, d, seed=62)
    full = cfg_of(1, d, H, f, N, L0, [L0])
    kvf, sf = O.encode_user(full, w, S)
    nsf = O.score_candidates(full, w, kvf, ns)
    for q in (1, 5, L0 - 1):
        part = cfg_of(1, d, H, f, N, L0, [q])
        kvp, sp = O.encode_user(part, w, S)
        nsp = O.score_candidates(part, w, kvp, ns)
        assert np.array_equal(sp[0], sf[0, L0 - q:])
        assert np.array_equal(kvp, kvf)
        assert np.array_equal(nsp, nsf)


def test_invariant_kv_cache_equivalence_and_s_independence():
    """Encode-once + score-per-candidate equals the no-cache joint run of each
    candidate; the joint run's S outputs and K/V are the same for every
    candidate (S never sees NS)."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=71)
    S, ns = rand_inputs(2, 3, L0, N, d, seed=72)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, s_out = O.encode_user(cfg, w, S)
    ns_out = O.score_candidates(cfg, w, kv, ns)
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns)
    np.testing.assert_allclose(jns, ns_out, rtol=0, atol=1e-12)
    for c in range(3):
        np.testing.assert_allclose(js[:, c], s_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(jkv[:, c], kv, rtol=0, atol=1e-12)


@pytest.mark.parametrize("fp8", [False, True], ids=["fp64", "e4m3"])
def test_append_equals_encode_of_grown_sequence(fp8):
    """Appending delta S rows (incremental: only the new rows run, against the
    cached K/V) equals encoding the concatenated sequence with every pyramid
    window grown by delta; the grown S output is the old output followed by
    the new rows' outputs, and the old rows' K/V are unchanged.  Checked
    against the brute-force token loop on the concatenated sequence too, and
    twice in a row (append to an appended cache)."""
    layers, d, H, f, N = 3, 16, 2, 24, 2
    L0, q = 14, [14, 9, 4]
    w = rand_weights(layers, d, f, N, seed=81)
    S_all, _ = rand_inputs(2, 1, L0 + 5 + 3, N, d, seed=82)
    cfg0 = cfg_of(layers, d, H, f, N, L0, q, fp8=fp8)
    kv0, s0 = O.encode_user(cfg0, w, S_all[:, :L0])
    cfg1 = cfg0.grown(5)
    kv1, new1 = O.encode_append(cfg1, w, kv0, S_all[:, L0:L0 + 5])
    kvf, sf = O.encode_user(cfg1, w, S_all[:, :L0 + 5])
    np.testing.assert_allclose(kv1, kvf, rtol=0, atol=1e-12)
    np.testing.assert_allclose(new1, sf[:, -5:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s0, sf[:, :-5], rtol=0, atol=1e-12)
    for l in range(layers):  # the old rows' K/V moved unchanged into the grown layout
        K0, V0 = O.kv_layer(cfg0, kv0[0], l)
        K1, V1 = O.kv_layer(cfg1, kv1[0], l)
        assert np.array_equal(K1[:K0.shape[0]], K0) and np.array_equal(V1[:V0.shape[0]], V0)
    cfg2 = cfg1.grown(3)
    kv2, new2 = O.encode_append(cfg2, w, kv1, S_all[:, L0 + 5:])
    kvg, sg = O.encode_user(cfg2, w, S_all)
    np.testing.assert_allclose(kv2, kvg, rtol=0, atol=1e-12)
    np.testing.assert_allclose(new2, sg[:, -3:], rtol=0, atol=1e-12)
    if not fp8:
        wl = to_lists(w)
        bs, _, bkv = run_candidate(wl, S_all[1].double().tolist(), [[0.0] * d] * N, cfg2.q, H, 1e-6)
        np.testing.assert_allclose(new2[1], np.array(bs)[-3:], rtol=0, atol=1e-12)
        for l, (K, V) in enumerate(bkv):
            Ko, Vo = O.kv_layer(cfg2, kv2[1], l)
            np.testing.assert_allclose(Ko, np.array(K), rtol=0, atol=1e-12)
            np.testing.assert_allclose(Vo, np.array(V), rtol=0, atol=1e-12)


def test_append_needs_anchored_windows():
    """The reading the append rests on matters: re-deriving a shrinking
    pyramid for the longer sequence (windows that slide) changes the old
    rows' outputs, so the incremental result would not be a re-encode."""
    layers, d, H, f, N = 2, 16, 2, 24, 1
    w = rand_weights(layers, d, f, N, seed=83)
    S_all, _ = rand_inputs(1, 1, 16, N, d, seed=84)
    cfg0 = cfg_of(layers, d, H, f, N, 12, [12, 4])
    kv0, _ = O.encode_user(cfg0, w, S_all[:, :12])
    kv1, new1 = O.encode_append(cfg0.grown(4), w, kv0, S_all[:, 12:])
    sliding = cfg_of(layers, d, H, f, N, 16, [12, 4])   # layer 1 keeps only the last 12 rows
    _, ss = O.encode_user(sliding, w, S_all)
    assert not np.allclose(new1[0], ss[0])
    # the schedule the cache came from must be valid: every q[l] > delta
    grown = cfg_of(layers, d, H, f, N, 12, [12, 4])
    with pytest.raises(ValueError):
        O.encode_append(grown, w, np.zeros((1, grown.grown(-4).kv_user_elems())), S_all[:, :4])


def test_invariant_candidate_independence():
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=81)
    S, ns = rand_inputs(1, 5, L0, N, d, seed=82)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, _ = O.encode_user(cfg, w, S)
    batch = O.score_candidates(cfg, w, kv, ns)
    for c in range(5):
        alone = O.score_candidates(cfg, w, kv, ns[:, c:c + 1])
        assert np.array_equal(alone[:, 0], batch[:, c])


def test_ns_mask_excludes_later_ns_and_other_candidates():
    """Changing NS token m of a candidate leaves NS outputs n < m of that
    candidate unchanged and changes n >= m."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=91)
    S, ns = rand_inputs(1, 2, L0, N, d, seed=92)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    kv, _ = O.encode_user(cfg, w, S)
    a = O.score_candidates(cfg, w, kv, ns)
    ns2 = ns.clone()
    ns2[0, 0, 1] += 1.0
    b = O.score_candidates(cfg, w, kv, ns2)
    assert np.array_equal(a[0, 0, :1], b[0, 0, :1])
    assert not np.allclose(a[0, 0, 1:], b[0, 0, 1:])
    assert np.array_equal(a[0, 1], b[0, 1])


def test_pyramid_schedule_golden():
    with open(os.path.join(GOLDEN, "pyramid_schedules.json")) as fh:
        gold = json.load(fh)
    for case in gold["cases"]:
        assert O.pyramid_schedule(case["L0"], case["q_end"], case["layers"]) == case["q"]


def test_e4m3_round_matches_torch_cast():
    """Every in-range value rounds like torch's float8_e4m3fn cast (RNE)."""
    fp8 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    finite = fp8[torch.isfinite(fp8)]
    for v in finite.tolist():
        assert O.e4m3_round(v) == v
    g = torch.Generator().manual_seed(5)
    xs = torch.cat([torch.randn(4000, generator=g) * s for s in (1e-3, 0.05, 1, 30, 150)])
    xs = xs[xs.abs() < 440]
    # midpoints between neighbours are ties: they must go to the even code
    pos = finite[finite > 0].sort().values
    mids = (pos[:-1].double() + pos[1:].double()) / 2
    xs = torch.cat([xs.double(), mids, -mids])
    want = xs.float().to(torch.float8_e4m3fn).double()
    got = torch.tensor([O.e4m3_round(v) for v in xs.tolist()], dtype=torch.float64)
    assert torch.equal(got, want)
    assert O.e4m3_round(1e6) == 448.0 and O.e4m3_round(-500.0) == -448.0


def test_fp8_mode_quantises_and_stays_close():
    """Both FP8 rules really quantise (results move) and stay inside the
    format's bound: e4m3 keeps 3 mantissa bits, so each operand carries at
    most 2^-4 relative rounding error and a product of two at most about
    2 * 2^-4."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=95)
    S, ns = rand_inputs(1, 2, L0, N, d, seed=96)
    c64 = cfg_of(layers, d, H, f, N, L0, q)
    kv, s = O.encode_user(c64, w, S)
    n64 = O.score_candidates(c64, w, kv, ns)
    scales, _ = O.calibrate(c64, w, S, ns)
    for c8 in (cfg_of(layers, d, H, f, N, L0, q, fp8=O.FP8_ROW),
               cfg_of(layers, d, H, f, N, L0, q, fp8=O.FP8_TENSOR, act_scale=scales)):
        kv8, s8 = O.encode_user(c8, w, S)
        n8 = O.score_candidates(c8, w, kv8, ns)
        for a, b in ((s8, s), (kv8, kv), (n8, n64)):
            err = O.rel_l2(a, b)
            assert 1e-4 < err < 2 * 2.0 ** -4, err


def _fp8_scales(cfg, seed, lo=0.002, hi=0.01):
    """Seeded per-tensor scales small enough that the larger inputs saturate."""
    g = torch.Generator().manual_seed(seed)
    return (lo + (hi - lo) * torch.rand(cfg.scale_shape(), generator=g)).double().numpy()


@pytest.mark.parametrize("case", TINY_CASES[1:4])
@pytest.mark.parametrize("rule", [O.FP8_ROW, O.FP8_TENSOR], ids=["per_row", "per_tensor"])
def test_brute_force_matches_oracle_fp8(case, rule):
    """Both FP8 rules against the brute-force token loop, whose e4m3 rounding
    is torch's float8_e4m3fn cast: outputs, every layer's K / V, and the
    calibration amax of every projection input tensor."""
    from brute_force import Fp8
    layers, d, H, f, N, L0, q, U, Cn = case
    w = rand_weights(layers, d, f, N, seed=L0 + d + 1)
    S, ns = rand_inputs(U, Cn, L0, N, d, seed=7 * L0 + N + 1)
    cfg = cfg_of(layers, d, H, f, N, L0, q, fp8=rule)
    if rule == O.FP8_TENSOR:
        cfg.act_scale = _fp8_scales(cfg, seed=L0)
    amax = np.zeros(cfg.scale_shape())
    kv, s_out = O.encode_user(cfg, w, S, amax=amax)
    ns_out = O.score_candidates(cfg, w, kv, ns, amax=amax)
    wl = to_lists(w)
    bam = np.zeros(cfg.scale_shape()).tolist()
    st = Fp8(rule, None if cfg.act_scale is None else cfg.act_scale.tolist(), bam)
    for u in range(U):
        for c in range(Cn):
            bs, bns, bkv = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                         q, H, 1e-6, fp8=st)
            np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
            np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)
            for l, (K, V) in enumerate(bkv):
                Ko, Vo = O.kv_layer(cfg, kv[u], l)
                np.testing.assert_allclose(Ko, np.array(K), rtol=0, atol=1e-12)
                np.testing.assert_allclose(Vo, np.array(V), rtol=0, atol=1e-12)
    np.testing.assert_allclose(amax, np.array(bam), rtol=0, atol=1e-12)
    assert np.all(amax > 0)


def _e4m3_grid(g, shape, exp2):
    """Random e4m3 values times 2^exp2, each row holding one +-448 entry."""
    codes = torch.randint(0, 256, shape, generator=g, dtype=torch.uint8).view(torch.float8_e4m3fn)
    v = codes.double()
    v[~torch.isfinite(v)] = 0.0
    v[:, 0] = 448.0 * torch.where(torch.rand(shape[0], generator=g) < 0.5, 1.0, -1.0).double()
    return (v * 2.0 ** exp2).numpy()


def test_fp8_exact_when_operands_are_representable():
    """Inputs that are e4m3 values times the scale, weights likewise: both
    rules must then reproduce the fp64 product bit for bit (every operand is
    exact in e4m3 and every sum is exact in fp64)."""
    g = torch.Generator().manual_seed(11)
    x = _e4m3_grid(g, (9, 32), -3)       # per-row amax 448 * 2^-3: scale 2^-3
    W = _e4m3_grid(g, (24, 32), -5)      # amax 448 * 2^-5: scale 2^-5
    exact = x @ W.T
    for rule in (O.FP8_ROW, O.FP8_TENSOR):
        y = O.project_rows(x, W, fp8=rule, xs=2.0 ** -3)
        assert np.array_equal(y, exact), rule
    assert np.array_equal(O.project_rows(x, W), exact)


def test_fp8_scale_constant_hand_worked():
    """One row through an identity weight (exact in e4m3 after its scale
    1/448): per row, y = e4m3(x / (amax/448)) * amax/448 with torch's cast;
    per tensor with scale 0.01, the values above 4.48 saturate at 4.48."""
    x = np.array([[0.3, -1.7, 2.9, 0.01, 5.5, -5.25, 1e-3, 0.0]])
    W = np.eye(8)
    s = 5.5 / 448.0
    want = (torch.tensor(x / s).float().to(torch.float8_e4m3fn).double() * s).numpy()
    # (the scale products are rounded in another order: equal to the last bits)
    np.testing.assert_allclose(O.project_rows(x, W, fp8=O.FP8_ROW), want, rtol=1e-15, atol=0)
    assert not np.allclose(want, x, rtol=1e-3)   # it did quantise
    xs = 0.01
    q = torch.tensor(x / xs).clamp(-448, 448).float().to(torch.float8_e4m3fn).double()
    want2 = (q * xs).numpy()
    np.testing.assert_allclose(O.project_rows(x, W, fp8=O.FP8_TENSOR, xs=xs), want2, rtol=1e-15,
                               atol=0)
    assert want2[0, 4] == pytest.approx(4.48) and want2[0, 5] == pytest.approx(-4.48)


def test_fp8_scale_granularity():
    """Per row: scaling one row by 2 scales exactly its own output by 2 and
    leaves the other rows alone.  Per tensor: the other rows are unchanged
    too, but the scaled row is quantised on the tensor's fixed grid, so its
    output is not three times the old one when the row is scaled by 3."""
    g = torch.Generator().manual_seed(12)
    x = torch.randn(6, 40, generator=g).double().numpy()
    W = (torch.randn(16, 40, generator=g) / 6).numpy()
    y = O.project_rows(x, W, fp8=O.FP8_ROW)
    x2 = x.copy()
    x2[3] *= 2.0
    y2 = O.project_rows(x2, W, fp8=O.FP8_ROW)
    assert np.array_equal(np.delete(y2, 3, 0), np.delete(y, 3, 0))
    assert np.array_equal(y2[3], 2.0 * y[3])
    xs = 0.02
    t = O.project_rows(x, W, fp8=O.FP8_TENSOR, xs=xs)
    x3 = x.copy()
    x3[3] *= 3.0
    t3 = O.project_rows(x3, W, fp8=O.FP8_TENSOR, xs=xs)
    assert np.array_equal(np.delete(t3, 3, 0), np.delete(t, 3, 0))
    assert not np.allclose(t3[3], 3.0 * t[3], rtol=1e-4, atol=0)
    # the same projection with per-row scales gives 3x exactly up to fp64 rounding
    r3 = O.project_rows(x3, W, fp8=O.FP8_ROW)
    np.testing.assert_allclose(r3[3], 3.0 * y[3], rtol=1e-14, atol=1e-14)
    # amax accumulates max |x| over all rows of the tensor
    am = np.zeros(1)
    O.project_rows(x3, W, fp8=O.FP8_TENSOR, xs=xs, amax=am)
    assert am[0] == np.abs(x3).max()


def test_fp8_calibration_amax_of_first_projection():
    """The calibration's amax slot of layer 0's QKV input is max |RMSNorm(x)
    * g| over the rows that entered it: torch's rms_norm over the S rows (S
    set) and over each NS position's rows of every candidate (NS sets)."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=97)
    S, ns = rand_inputs(2, 3, L0, N, d, seed=98)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    scales, amax = O.calibrate(cfg, w, S, ns)
    want_s = Fnn.rms_norm(S.double(), (d,), weight=w["g1_s"][0].double(), eps=1e-6).abs().max()
    assert amax[0, 0, 0] == pytest.approx(float(want_s), rel=1e-12)
    for n in range(N):
        xn = Fnn.rms_norm(ns[:, :, n].double(), (d,), weight=w["g1_ns"][0, n].double(), eps=1e-6)
        assert amax[0, 1 + n, 0] == pytest.approx(float(xn.abs().max()), rel=1e-12)
    np.testing.assert_allclose(scales, np.float32(amax / 448.0), rtol=0, atol=0)


def test_fp8_per_tensor_candidate_independence():
    """Fixed per-tensor scales keep a candidate's result independent of the
    other candidates in the call."""
    layers, d, H, f, N, L0, q = _small()
    w = rand_weights(layers, d, f, N, seed=99)
    S, ns = rand_inputs(1, 4, L0, N, d, seed=100)
    cfg = cfg_of(layers, d, H, f, N, L0, q, fp8=O.FP8_TENSOR)
    cfg.act_scale = _fp8_scales(cfg, seed=3)
    kv, _ = O.encode_user(cfg, w, S)
    batch = O.score_candidates(cfg, w, kv, ns)
    for c in range(4):
        alone = O.score_candidates(cfg, w, kv, ns[:, c:c + 1])
        assert np.array_equal(alone[:, 0], batch[:, c])


def test_auto_split_matches_numpy():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(5, 32, generator=g)
    Wsp = torch.randn(4 * 8, 32, generator=g)
    ns = O.auto_split(x, Wsp, 4, 8)
    ref = (x.double().numpy() @ Wsp.double().numpy().T).reshape(5, 4, 8)
    np.testing.assert_allclose(ns, ref, rtol=1e-13, atol=1e-13)


def test_embed_gather_matches_numpy():
    g = torch.Generator().manual_seed(4)
    table = torch.randn(50, 8, generator=g)
    ids = torch.randint(0, 50, (3, 7), generator=g)
    out = O.embed_gather(table, ids)
    assert np.array_equal(out, table.double().numpy()[ids.numpy()])
    with pytest.raises(IndexError):
        O.embed_gather(table, np.array([50]))


# ----------------------------------------------------------------- backward
def _bw_case(seed=150):
    layers, d, H, f, N, L0, q = 2, 8, 2, 12, 2, 7, [5, 3]
    w = rand_weights(layers, d, f, N, seed=seed, dtype=torch.float64)
    w = {k: v.float().double() for k, v in w.items()}
    S, ns = rand_inputs(2, 2, L0, N, d, seed=seed + 1, dtype=torch.float64)
    S, ns = S.float().double(), ns.float().double()
    g = torch.Generator().manual_seed(seed + 2)
    G_s = torch.randn(2, q[-1], d, generator=g, dtype=torch.float64)
    G_ns = torch.randn(2, 2, N, d, generator=g, dtype=torch.float64)
    return cfg_of(layers, d, H, f, N, L0, q), w, S, ns, G_s, G_ns


def test_backward_oracle_forward_matches_c_oracle():
    """The PyTorch restatement the gradients come from computes what the
    pinned C oracle computes (the S tails and the NS outputs)."""
    from oracle import backward as OB
    cfg, w, S, ns, _, _ = _bw_case()
    s_t, ns_t = OB.forward(cfg, w, S, ns)
    kv, s_c = O.encode_user(cfg, w, S)
    ns_c = O.score_candidates(cfg, w, kv, ns)
    np.testing.assert_allclose(s_t.detach().numpy(), s_c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ns_t.detach().numpy(), ns_c, rtol=0, atol=1e-12)


def test_backward_oracle_matches_finite_differences():
    """Every gradient along random directions against central differences of
    the C oracle's loss: (L(p + e v) - L(p - e v)) / 2e = grad . v."""
    from oracle import backward as OB
    cfg, w, S, ns, G_s, G_ns = _bw_case()
    _, grads = OB.gradients(cfg, w, S, ns, G_s, G_ns)

    def loss(w_, S_, ns_):
        kv, s_c = O.encode_user(cfg, w_, S_.float())
        return float((s_c * G_s.numpy()).sum() +
                     (O.score_candidates(cfg, w_, kv, ns_) * G_ns.numpy()).sum())

    g = torch.Generator().manual_seed(7)
    eps = 1e-3
    for name in ["S", "ns"] + list(OB.W_NAMES):
        base = {"S": S, "ns": ns}.get(name, w.get(name))
        v = torch.randn(base.shape, generator=g, dtype=torch.float64)
        # float32-representable probes (the C oracle reads its inputs as float32)
        p_plus, p_minus = (base + eps * v).float().double(), (base - eps * v).float().double()
        step = (p_plus - p_minus).double() / 2

        def with_(p):
            if name == "S":
                return w, p, ns
            if name == "ns":
                return w, S, p
            return dict(w, **{name: p}), S, ns
        fd = (loss(*with_(p_plus)) - loss(*with_(p_minus)))
        an = 2.0 * float((grads[name] * step).sum())
        assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)), (name, fd, an)


def _bw_full_case(seed=160):
    layers, d, H, f, N, L0, q = 2, 8, 2, 12, 3, 7, [5, 3]
    w = rand_weights(layers, d, f, N, seed=seed, dtype=torch.float64)
    w = {k: v.float().double() for k, v in w.items()}
    S, ns = rand_inputs(2, 1, L0, N, d, seed=seed + 1, dtype=torch.float64)
    S, ns = S.float().double(), ns.float().double()
    g = torch.Generator().manual_seed(seed + 2)
    G_s = torch.randn(2, q[-1], d, generator=g, dtype=torch.float64)
    G_ns = torch.randn(2, 1, N, d, generator=g, dtype=torch.float64)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.full_attn = True
    return cfg, w, S, ns, G_s, G_ns


def test_backward_oracle_full_attention_forward_matches_c_oracle():
    """Full attention: the restated forward equals the C oracle's joint form
    (its every-key visibility pinned by the brute force) to 1e-12."""
    from oracle import backward as OB
    cfg, w, S, ns, _, _ = _bw_full_case()
    s_t, ns_t = OB.forward(cfg, w, S, ns)
    s_c, _, ns_c = O.full_forward_joint(cfg, w, S, ns)
    np.testing.assert_allclose(s_t.detach().numpy(), s_c[:, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ns_t.detach().numpy(), ns_c, rtol=0, atol=1e-12)


def test_backward_oracle_full_attention_matches_finite_differences():
    """Full attention: every gradient along a random direction against the
    central difference of the C oracle's joint-form loss."""
    from oracle import backward as OB
    cfg, w, S, ns, G_s, G_ns = _bw_full_case()
    _, grads = OB.gradients(cfg, w, S, ns, G_s, G_ns)

    def loss(w_, S_, ns_):
        s_c, _, ns_c = O.full_forward_joint(cfg, w_, S_.float(), ns_)
        return float((s_c[:, 0] * G_s.numpy()).sum() + (ns_c * G_ns.numpy()).sum())

    g = torch.Generator().manual_seed(9)
    eps = 1e-3
    for name in ["S", "ns"] + list(OB.W_NAMES):
        base = {"S": S, "ns": ns}.get(name, w.get(name))
        v = torch.randn(base.shape, generator=g, dtype=torch.float64)
        p_plus, p_minus = (base + eps * v).float().double(), (base - eps * v).float().double()
        step = (p_plus - p_minus).double() / 2

        def with_(p):
            if name == "S":
                return w, p, ns
            if name == "ns":
                return w, S, p
            return dict(w, **{name: p}), S, ns
        fd = loss(*with_(p_plus)) - loss(*with_(p_minus))
        an = 2.0 * float((grads[name] * step).sum())
        assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)), (name, fd, an)


def test_backward_oracle_full_attention_differs_from_causal():
    """The switch is live: the same inputs give other gradients under the
    causal mask (S rows then see neither later S rows nor NS rows)."""
    from oracle import backward as OB
    cfg, w, S, ns, G_s, G_ns = _bw_full_case()
    _, g_full = OB.gradients(cfg, w, S, ns, G_s, G_ns)
    cfg.full_attn = False
    _, g_causal = OB.gradients(cfg, w, S, ns, G_s, G_ns)
    assert float((g_full["Wqkv_s"] - g_causal["Wqkv_s"]).abs().max()) > 1e-6
    assert float((g_full["S"] - g_causal["S"]).abs().max()) > 1e-6


def _bw_moe_case(topk, seed=170):
    layers, d, H, f, N, L0, q = 2, 8, 2, 12, 2, 9, [6, 3]
    w = rand_weights(layers, d, f, N, seed=seed, dtype=torch.float64, experts=3)
    w = {k: v.float().double() for k, v in w.items()}
    S, ns = rand_inputs(2, 2, L0, N, d, seed=seed + 1, dtype=torch.float64)
    S, ns = S.float().double(), ns.float().double()
    g = torch.Generator().manual_seed(seed + 2)
    G_s = torch.randn(2, q[-1], d, generator=g, dtype=torch.float64)
    G_ns = torch.randn(2, 2, N, d, generator=g, dtype=torch.float64)
    cfg = cfg_of(layers, d, H, f, N, L0, q)
    cfg.moe_experts, cfg.moe_topk = 3, topk
    return cfg, w, S, ns, G_s, G_ns


def _moe_margins(cfg, w, S, ns, monkeypatch):
    """Smallest gap, over every S row of every layer, between the k-th and
    the (k+1)-th router logit: the room a perturbation has before the
    selection changes."""
    from oracle import backward as OB
    seen = []
    orig = OB._s_ffn

    def spy(cfg_, w_, l, h):
        seen.append((l, h.detach()))
        return orig(cfg_, w_, l, h)
    monkeypatch.setattr(OB, "_s_ffn", spy)
    OB.forward(cfg, {k: torch.as_tensor(v) for k, v in w.items()}, S, ns)
    gaps = []
    for l, h in seen:
        z = OB._rms(h, w["g2_s"][l], cfg.eps)
        lg = torch.sort(z @ w["W_router"][l].T, dim=-1, descending=True).values
        gaps.append(float((lg[:, cfg.moe_topk - 1] - lg[:, cfg.moe_topk]).min()))
    return min(gaps)


@pytest.mark.parametrize("topk", [1, 2])
def test_backward_oracle_moe_forward_matches_c_oracle(topk):
    """The restated mixture (stable-sort top-k, softmax gates over the chosen
    logits) equals the C oracle's (pinned by the brute force) to 1e-12."""
    from oracle import backward as OB
    cfg, w, S, ns, _, _ = _bw_moe_case(topk)
    s_t, ns_t = OB.forward(cfg, w, S, ns)
    kv, s_c = O.encode_user(cfg, w, S)
    ns_c = O.score_candidates(cfg, w, kv, ns)
    np.testing.assert_allclose(s_t.detach().numpy(), s_c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ns_t.detach().numpy(), ns_c, rtol=0, atol=1e-12)


@pytest.mark.parametrize("topk", [1, 2])
def test_backward_oracle_moe_matches_finite_differences(topk, monkeypatch):
    """Gradients of a mixture (router, experts, every other tensor) against
    central differences of the C oracle's loss; the routing margins are
    checked to be far above what the perturbations can move a logit by, so
    no selection changes between the two evaluations."""
    from oracle import backward as OB
    cfg, w, S, ns, G_s, G_ns = _bw_moe_case(topk)
    assert _moe_margins(cfg, w, S, ns, monkeypatch) > 2e-2
    _, grads = OB.gradients(cfg, w, S, ns, G_s, G_ns)
    assert float(grads["W1_s"].abs().max()) == 0.0  # the dense S FFN is unused

    def loss(w_, S_, ns_):
        kv, s_c = O.encode_user(cfg, w_, S_.float())
        return float((s_c * G_s.numpy()).sum() +
                     (O.score_candidates(cfg, w_, kv, ns_) * G_ns.numpy()).sum())

    g = torch.Generator().manual_seed(11)
    eps = 1e-4
    for name in ["S", "ns"] + list(OB.names(cfg)):
        base = {"S": S, "ns": ns}.get(name, w.get(name))
        v = torch.randn(base.shape, generator=g, dtype=torch.float64)
        p_plus, p_minus = (base + eps * v).float().double(), (base - eps * v).float().double()
        step = (p_plus - p_minus).double() / 2

        def with_(p):
            if name == "S":
                return w, p, ns
            if name == "ns":
                return w, S, p
            return dict(w, **{name: p}), S, ns
        fd = loss(*with_(p_plus)) - loss(*with_(p_minus))
        an = 2.0 * float((grads[name] * step).sum())
        assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)) + 1e-9, (name, fd, an)


# ------------------------------------------------------------- random small shapes
try:
    from hypothesis import given, settings
    from hypothesis import strategies as st
except ImportError:  # pragma: no cover - hypothesis is in the image
    given = None


if given is not None:
    @st.composite
    def _tiny_stack(draw):
        """A random tiny configuration: any layer count, width, head split,
        FFN width, NS count, sequence length, monotone pyramid, users and
        candidates the brute force finishes in milliseconds."""
        layers = draw(st.integers(1, 3))
        H = draw(st.sampled_from([1, 2]))
        d = H * draw(st.sampled_from([2, 4, 6]))
        f = draw(st.integers(1, 3)) * 4
        N = draw(st.integers(1, 3))
        L0 = draw(st.integers(1, 12))
        q, prev = [], L0
        for _ in range(layers):
            prev = draw(st.integers(1, prev))
            q.append(prev)
        U = draw(st.integers(1, 2))
        C = draw(st.integers(1, 2))
        seed = draw(st.integers(0, 10_000))
        return layers, d, H, f, N, L0, q, U, C, seed

    @settings(max_examples=25, deadline=None, derandomize=True)
    @given(_tiny_stack())
    def test_brute_force_matches_oracle_random_shapes(case):
        """The C oracle's split (encode + score) and joint forms against the
        token-by-token brute force on random tiny shapes (one-row tails,
        one-token sequences, heads of width 1 to 6, pyramids that keep or cut
        every row)."""
        layers, d, H, f, N, L0, q, U, Cn, seed = case
        w = rand_weights(layers, d, f, N, seed=seed)
        S, ns = rand_inputs(U, Cn, L0, N, d, seed=seed + 1)
        cfg = cfg_of(layers, d, H, f, N, L0, q)
        kv, s_out = O.encode_user(cfg, w, S)
        ns_out = O.score_candidates(cfg, w, kv, ns)
        js, _, jns = O.full_forward_joint(cfg, w, S, ns)
        wl = to_lists(w)
        for u in range(U):
            for c in range(Cn):
                bs, bns, _ = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                           q, H, 1e-6)
                np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
                np.testing.assert_allclose(js[u, c], np.array(bs), rtol=0, atol=1e-12)
                np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)
                np.testing.assert_allclose(jns[u, c], np.array(bns), rtol=0, atol=1e-12)

    @settings(max_examples=15, deadline=None, derandomize=True)
    @given(_tiny_stack())
    def test_brute_force_matches_oracle_random_shapes_full_attention(case):
        """Full attention (joint form) against the brute force's every-key
        visibility on random tiny shapes."""
        layers, d, H, f, N, L0, q, U, Cn, seed = case
        w = rand_weights(layers, d, f, N, seed=seed + 2)
        S, ns = rand_inputs(U, Cn, L0, N, d, seed=seed + 3)
        cfg = cfg_of(layers, d, H, f, N, L0, q)
        cfg.full_attn = True
        js, _, jns = O.full_forward_joint(cfg, w, S, ns)
        wl = to_lists(w)
        for u in range(U):
            for c in range(Cn):
                bs, bns, _ = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                           q, H, 1e-6, full=True)
                np.testing.assert_allclose(js[u, c], np.array(bs), rtol=0, atol=1e-12)
                np.testing.assert_allclose(jns[u, c], np.array(bns), rtol=0, atol=1e-12)

    @settings(max_examples=15, deadline=None, derandomize=True)
    @given(_tiny_stack(), st.integers(1, 5), st.integers(1, 2))
    def test_brute_force_matches_oracle_random_shapes_moe(case, experts, topk):
        """The sparse-MoE S-side FFN against the brute force on random tiny
        shapes, expert counts and top-k (k <= E)."""
        layers, d, H, f, N, L0, q, U, Cn, seed = case
        topk = min(topk, experts)
        w = rand_weights(layers, d, f, N, seed=seed + 4, experts=experts)
        S, ns = rand_inputs(U, Cn, L0, N, d, seed=seed + 5)
        cfg = cfg_of(layers, d, H, f, N, L0, q)
        cfg.moe_experts, cfg.moe_topk = experts, topk
        kv, s_out = O.encode_user(cfg, w, S)
        ns_out = O.score_candidates(cfg, w, kv, ns)
        wl = to_lists(w)
        for u in range(U):
            for c in range(Cn):
                bs, bns, _ = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                           q, H, 1e-6, moe_topk=topk)
                np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
                np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)

    @settings(max_examples=6, deadline=None, derandomize=True)
    @given(_tiny_stack())
    def test_backward_oracle_random_shapes(case):
        """The gradient oracle on random tiny shapes: its forward equals the C
        oracle's, and every gradient along a random direction equals the
        central difference of the C oracle's loss (as the fixed-shape pin)."""
        from oracle import backward as OB
        layers, d, H, f, N, L0, q, U, Cn, seed = case
        w = rand_weights(layers, d, f, N, seed=seed + 6, dtype=torch.float64)
        w = {k: v.float().double() for k, v in w.items()}
        S, ns = rand_inputs(U, Cn, L0, N, d, seed=seed + 7, dtype=torch.float64)
        S, ns = S.float().double(), ns.float().double()
        g = torch.Generator().manual_seed(seed + 8)
        G_s = torch.randn(U, q[-1], d, generator=g, dtype=torch.float64)
        G_ns = torch.randn(U, Cn, N, d, generator=g, dtype=torch.float64)
        cfg = cfg_of(layers, d, H, f, N, L0, q)
        s_t, ns_t = OB.forward(cfg, w, S, ns)
        kv, s_c = O.encode_user(cfg, w, S)
        ns_c = O.score_candidates(cfg, w, kv, ns)
        np.testing.assert_allclose(s_t.detach().numpy(), s_c, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ns_t.detach().numpy(), ns_c, rtol=0, atol=1e-12)
        _, grads = OB.gradients(cfg, w, S, ns, G_s, G_ns)

        def loss(w_, S_, ns_):
            kv_, s_ = O.encode_user(cfg, w_, S_.float())
            return float((s_ * G_s.numpy()).sum() +
                         (O.score_candidates(cfg, w_, kv_, ns_) * G_ns.numpy()).sum())

        eps = 1e-3
        for name in ["S", "ns"] + list(OB.W_NAMES):
            base = {"S": S, "ns": ns}.get(name, w.get(name))
            v = torch.randn(base.shape, generator=g, dtype=torch.float64)
            p_plus, p_minus = (base + eps * v).float().double(), (base - eps * v).float().double()
            step = (p_plus - p_minus).double() / 2

            def with_(p):
                if name == "S":
                    return w, p, ns
                if name == "ns":
                    return w, S, p
                return dict(w, **{name: p}), S, ns
            fd = loss(*with_(p_plus)) - loss(*with_(p_minus))
            an = 2.0 * float((grads[name] * step).sum())
            assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)), (name, fd, an)

    @settings(max_examples=12, deadline=None, derandomize=True)
    @given(_tiny_stack(), st.sampled_from([O.FP8_ROW, O.FP8_TENSOR]))
    def test_brute_force_matches_oracle_random_shapes_fp8(case, rule):
        """Both FP8 rules against the brute force (torch's e4m3 cast) on
        random tiny shapes: outputs and the calibration maxima."""
        from brute_force import Fp8
        layers, d, H, f, N, L0, q, U, Cn, seed = case
        w = rand_weights(layers, d, f, N, seed=seed + 9)
        S, ns = rand_inputs(U, Cn, L0, N, d, seed=seed + 10)
        cfg = cfg_of(layers, d, H, f, N, L0, q, fp8=rule)
        if rule == O.FP8_TENSOR:
            cfg.act_scale = _fp8_scales(cfg, seed=seed)
        amax = np.zeros(cfg.scale_shape())
        kv, s_out = O.encode_user(cfg, w, S, amax=amax)
        ns_out = O.score_candidates(cfg, w, kv, ns, amax=amax)
        wl = to_lists(w)
        bam = np.zeros(cfg.scale_shape()).tolist()
        fp8 = Fp8(rule, None if cfg.act_scale is None else cfg.act_scale.tolist(), bam)
        for u in range(U):
            for c in range(Cn):
                bs, bns, _ = run_candidate(wl, S[u].double().tolist(), ns[u, c].double().tolist(),
                                           q, H, 1e-6, fp8=fp8)
                np.testing.assert_allclose(s_out[u], np.array(bs), rtol=0, atol=1e-12)
                np.testing.assert_allclose(ns_out[u, c], np.array(bns), rtol=0, atol=1e-12)
        np.testing.assert_allclose(amax, np.array(bam), rtol=0, atol=1e-12)

    @settings(max_examples=12, deadline=None, derandomize=True)
    @given(_tiny_stack(), st.integers(1, 4))
    def test_append_equals_reencode_random_shapes(case, delta):
        """Appending delta rows to an encoded cache equals encoding the grown
        sequence (cache and the new rows' outputs), and the new rows' outputs
        equal the brute force's, on random tiny shapes."""
        layers, d, H, f, N, L0, q, U, _, seed = case
        w = rand_weights(layers, d, f, N, seed=seed + 11)
        S_all, _ = rand_inputs(U, 1, L0 + delta, N, d, seed=seed + 12)
        cfg0 = cfg_of(layers, d, H, f, N, L0, q)
        kv0, _ = O.encode_user(cfg0, w, S_all[:, :L0])
        cfg1 = cfg0.grown(delta)
        kv1, new1 = O.encode_append(cfg1, w, kv0, S_all[:, L0:])
        kvf, sf = O.encode_user(cfg1, w, S_all)
        np.testing.assert_allclose(kv1, kvf, rtol=0, atol=1e-12)
        np.testing.assert_allclose(new1, sf[:, -delta:], rtol=0, atol=1e-12)
        wl = to_lists(w)
        for u in range(U):
            bs, _, _ = run_candidate(wl, S_all[u].double().tolist(), [[0.0] * d] * N, cfg1.q, H, 1e-6)
            np.testing.assert_allclose(new1[u], np.array(bs)[-delta:], rtol=0, atol=1e-12)

    @settings(max_examples=16, deadline=None, derandomize=True)
    @given(_tiny_stack(), st.booleans())
    def test_textbook_reduction_random_shapes(case, full):
        """With every NS parameter set equal to the S set, each block is a
        pre-norm Transformer layer over [S; NS] from torch's library routines
        (causal, or bidirectional for full attention), on random tiny shapes."""
        layers, d, H, f, N, L0, q, _, Cn, seed = case
        w = rand_weights(layers, d, f, N, seed=seed + 13, dtype=torch.float64)
        for name in ("Wqkv", "Wo", "W1", "W2", "g1", "g2"):
            w[name + "_ns"] = w[name + "_s"][:, None].expand(-1, N, *w[name + "_s"].shape[1:]).clone()
        S, ns = rand_inputs(1, Cn, L0, N, d, seed=seed + 14, dtype=torch.float64)
        w = {k: v.float().double() for k, v in w.items()}
        S, ns = S.float().double(), ns.float().double()
        cfg = cfg_of(layers, d, H, f, N, L0, q)
        cfg.full_attn = full
        js, _, jns = O.full_forward_joint(cfg, w, S, ns)
        for c in range(Cn):
            x = torch.cat([S[0], ns[0, c]])
            L = L0
            for l in range(layers):
                y = _torch_causal_layer(x, w["Wqkv_s"][l], w["Wo_s"][l], w["W1_s"][l], w["W2_s"][l],
                                        w["g1_s"][l], w["g2_s"][l], H, 1e-6, causal=not full)
                x = torch.cat([y[L - q[l]:L], y[L:]])
                L = q[l]
            np.testing.assert_allclose(js[0, c], x[:L].numpy(), rtol=0, atol=1e-11)
            np.testing.assert_allclose(jns[0, c], x[L:].numpy(), rtol=0, atol=1e-11)
