"""GPU parity: the CUDA path through the C ABI against the CPU fp64 oracle.

Tolerances are the stated maximum relative L2 error per output tensor: 1e-5
(fp32 path), 2e-2 (bf16), 6e-2 (fp8); the mask and the pyramid indexing are
checked bit-exactly.  Output tensors: the final S tail rows, the NS outputs,
and every layer's K and V in the cache.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import unified_transformer_recommender_onetrans_b200 as ot
from gpu_common import TOL, assert_within, kv_errors, make_model, model_of, oracle_cfg
from helpers import rand_inputs, rand_weights
from oracle import oracle as O
from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights

pytestmark = pytest.mark.gpu

TEST_WAIT = 1 << 22


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()
    assert torch.cuda.is_available()


def _run_full(m, S, ns):
    kv = m.new_kv_cache(S.shape[0])
    s_tail, ns_out = m.full_forward(S, ns, kv=kv)
    m.poll()
    return s_tail, ns_out, kv


def _errors_vs_oracle(m, w, S_cpu, ns_cpu, s_tail, ns_out, kv, users):
    cfg = oracle_cfg(m)
    kv_o, s_o = O.encode_user(cfg, w, S_cpu[users])
    ns_o = O.score_candidates(cfg, w, kv_o, ns_cpu[users])
    errs = {"s_tail": O.rel_l2(s_tail[users].double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(ns_out[users].double().cpu().numpy(), ns_o)}
    errs.update(kv_errors(m, kv[users], kv_o, cfg))
    return errs


# ----------------------------------------------------------------- fp32 path
def test_tiny_fp32_block_parity():
    wl = WORKLOADS["tiny_fp32"]
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)                       # [1, 4, 256]
    m = model_of(wl, w)
    m.set_wait_limit(TEST_WAIT)
    ns = m.auto_split(x.cuda())                           # [1, 4, 8, 64]
    ns_o = O.auto_split(x, w["W_split"], wl.n_ns, wl.d)
    assert O.rel_l2(ns.double().cpu().numpy(), ns_o) <= TOL["f32"]
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns)
    # the oracle starts from its own fp64 Auto-Split output
    cfg = oracle_cfg(m)
    kv_o, s_o = O.encode_user(cfg, w, S)
    nso = O.score_candidates(cfg, w, kv_o, ns_o)
    errs = {"s_tail": O.rel_l2(s_tail.double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(ns_out.double().cpu().numpy(), nso)}
    errs.update(kv_errors(m, kv, kv_o, cfg))
    assert_within(errs, TOL["f32"])


# ----------------------------------------------------------------- bf16, small
SMALL = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])


@pytest.fixture(scope="module")
def small_case():
    w = rand_weights(3, 128, 256, 5, seed=101, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 7, 300, 5, 128, seed=102, dtype=torch.bfloat16)
    return w, S, ns


@pytest.mark.parametrize("path", [0, 1], ids=["tcgen05", "cuda_core"])
def test_bf16_small_parity(small_case, path):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    m.set_wait_limit(TEST_WAIT)
    m.set_kernel_path(path)
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns.cuda())
    errs = _errors_vs_oracle(m, w, S, ns, s_tail, ns_out, kv, [0, 1, 2])
    assert_within(errs, TOL["bf16"])


def test_bf16_tcgen05_matches_cuda_core_path(small_case):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    m.set_wait_limit(TEST_WAIT)
    a = _run_full(m, S.cuda(), ns.cuda())
    m.set_kernel_path(1)
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert O.rel_l2(x.double().cpu().numpy(), y.double().cpu().numpy()) < 1e-2


def test_bf16_deterministic(small_case):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    a = _run_full(m, S.cuda(), ns.cuda())
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_kv_cache_equivalence_and_candidate_independence(small_case):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    Sd, nsd = S.cuda(), ns.cuda()
    s_tail, ns_out, kv = _run_full(m, Sd, nsd)
    kv2, s2 = m.encode_user(Sd)
    sc = m.score_candidates(kv2, nsd)
    m.poll()
    assert torch.equal(kv2, kv) and torch.equal(s2, s_tail) and torch.equal(sc, ns_out)
    # a candidate scored alone matches the same candidate inside the batch, up
    # to the bf16 rounding of values whose summation order depends on how the
    # candidate's NS keys fall into key blocks (two bf16 ulps, 2 * 2^-8)
    for c in (0, 3, 6):
        alone = m.score_candidates(kv2, nsd[:, c:c + 1].contiguous())
        m.poll()
        err = O.rel_l2(alone[:, 0].double().cpu().numpy(), ns_out[:, c].double().cpu().numpy())
        assert err < 2 * 2.0 ** -8, (c, err)


def test_encode_without_tail_writes_same_cache(small_case):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    kv_a, _ = m.encode_user(S.cuda())
    kv_b, none = m.encode_user(S.cuda(), want_s_tail=False)
    m.poll()
    assert none is None and torch.equal(kv_a, kv_b)


# ----------------------------------------------------------------- bit-exact probes
def test_mask_probe_bitexact():
    """W_Q = W_K = 0 makes every score 0; with one-hot S / NS rows, gain 1,
    W_V = I, W_O = I and W_2 = 0, output row i has a non-zero in column j
    exactly when key j is visible to query i (plus its own one-hot)."""
    L0, N, d, q = 100, 8, 128, 60
    w = rand_weights(1, d, 256, N, seed=5, dtype=torch.bfloat16)
    eye = torch.eye(d, dtype=torch.bfloat16)
    for k, shape in (("Wqkv_s", (1, 3 * d, d)), ("Wqkv_ns", (1, N, 3 * d, d))):
        t = torch.zeros(shape, dtype=torch.bfloat16)
        t[..., 2 * d:, :] = eye
        w[k] = t
    w["g1_s"] = torch.ones_like(w["g1_s"])
    w["g1_ns"] = torch.ones_like(w["g1_ns"])
    w["Wo_s"] = eye.expand(1, d, d).clone()
    w["Wo_ns"] = eye.expand(1, N, d, d).clone()
    w["W2_s"] = torch.zeros_like(w["W2_s"])
    w["W2_ns"] = torch.zeros_like(w["W2_ns"])
    S = torch.zeros(1, L0, d, dtype=torch.bfloat16)
    S[0, torch.arange(L0), torch.arange(L0)] = 1
    ns = torch.zeros(1, 2, N, d, dtype=torch.bfloat16)
    for c in range(2):
        ns[0, c, torch.arange(N), L0 + torch.arange(N)] = 1
    for path in (0, 1):
        m = make_model(w, layers=1, d=d, heads=2, ffn=256, n_ns=N, L0=L0, q=[q])
        m.set_kernel_path(path)
        s_tail, ns_out, _ = _run_full(m, S.cuda(), ns.cuda())
        nz_s = (s_tail[0].float().cpu() != 0)
        want = torch.zeros(q, d, dtype=torch.bool)
        for i in range(q):
            t = L0 - q + i
            want[i, : t + 1] = True
        assert torch.equal(nz_s, want), path
        for c in range(2):
            nz = ns_out[0, c].float().cpu() != 0
            want = torch.zeros(N, d, dtype=torch.bool)
            for n in range(N):
                want[n, :L0] = True
                want[n, L0: L0 + n + 1] = True
            assert torch.equal(nz, want), (path, c)


def test_pyramid_identity_bitexact():
    """W_O = W_2 = 0: every block is the identity on its kept rows, so the
    final S rows are exactly input rows L0 - q_last .. L0 - 1."""
    w = rand_weights(4, 128, 256, 3, seed=9, dtype=torch.bfloat16)
    for k in ("Wo_s", "Wo_ns", "W2_s", "W2_ns"):
        w[k] = torch.zeros_like(w[k])
    q = [250, 131, 60, 7]
    S, ns = rand_inputs(3, 2, 250, 3, 128, seed=10, dtype=torch.bfloat16)
    m = make_model(w, layers=4, d=128, heads=2, ffn=256, n_ns=3, L0=250, q=q)
    s_tail, ns_out, _ = _run_full(m, S.cuda(), ns.cuda())
    assert torch.equal(s_tail.cpu(), S[:, 250 - 7:])
    assert torch.equal(ns_out.cpu(), ns)


# ----------------------------------------------------------------- errors on the device
def test_device_wait_timeout_is_reported_and_context_survives(small_case):
    w, S, ns = small_case
    m = make_model(w, **SMALL)
    m.set_wait_limit(1)  # a wait that runs out: kernels record it and return
    m.full_forward(S.cuda(), ns.cuda())
    with pytest.raises(ot.OtError) as e:
        m.poll()
    assert e.value.code == 8
    m.set_wait_limit(TEST_WAIT)
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns.cuda())
    errs = _errors_vs_oracle(m, w, S, ns, s_tail, ns_out, kv, [1])
    assert_within(errs, TOL["bf16"])


def test_embed_gather_and_bounds_flag():
    g = torch.Generator().manual_seed(0)
    table = torch.randn(1000, 384, generator=g).to(torch.bfloat16).cuda()
    ids = torch.randint(0, 1000, (3, 77), generator=g).cuda()
    out = ot.embed_gather(table, ids)
    torch.cuda.synchronize()
    assert torch.equal(out, table[ids])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = ids.clone()
    bad[1, 5] = 1000
    out = ot.embed_gather(table, bad, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 9
    assert torch.all(out[1, 5] == 0) and torch.equal(out[0], table[ids[0]])


# ----------------------------------------------------------------- full-size workloads
def _full_size(name, users_checked):
    wl = WORKLOADS[name]
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)
    m = model_of(wl, w)
    m.set_wait_limit(TEST_WAIT)
    ns = m.auto_split(x.cuda())
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns)
    cfg = oracle_cfg(m)
    ns_o = O.auto_split(x[users_checked], w["W_split"], wl.n_ns, wl.d)
    kv_o, s_o = O.encode_user(cfg, w, S[users_checked])
    nso = O.score_candidates(cfg, w, kv_o, ns_o)
    errs = {"s_tail": O.rel_l2(s_tail[users_checked].double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(ns_out[users_checked].double().cpu().numpy(), nso)}
    errs.update(kv_errors(m, kv[users_checked], kv_o, cfg))
    return errs


def test_onetrans_s_full_forward_sampled_users():
    assert_within(_full_size("onetrans_s_full", [0, 37]), TOL["bf16"])


def test_onetrans_l_full_forward_sampled_users():
    assert_within(_full_size("onetrans_l_full", [5]), TOL["bf16"])


def test_onetrans_l_cached_scoring_sampled():
    """OneTransL serving with the cross-request cache at the cached-candidate
    shape: all 32 users (1500 S tokens, d = 384) encoded once, 8 candidates
    per user scored against the cache (24 NS tokens each: 192 NS rows per
    user and head, the split-key NS attention; the two-GEMM d = 384 FFN).
    Sampled users and candidates against the oracle: NS outputs and every
    layer's K / V."""
    wl = WORKLOADS["onetrans_l_full"].with_(cands=8)
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)                    # [32, 8, 1024]
    m = model_of(wl, w)
    m.set_wait_limit(TEST_WAIT)
    kv, _ = m.encode_user(S.cuda(), want_s_tail=False)
    ns = m.auto_split(x.cuda())
    out = m.score_candidates(kv, ns)
    m.poll()
    users, cands = [2, 31], [0, 3, 7]
    cfg = oracle_cfg(m)
    kv_o, _ = O.encode_user(cfg, w, S[users])
    ns_o = O.auto_split(x[users][:, cands], w["W_split"], wl.n_ns, wl.d)
    out_o = O.score_candidates(cfg, w, kv_o, ns_o)
    errs = {"ns_out": O.rel_l2(out[users][:, cands].double().cpu().numpy(), out_o)}
    errs.update(kv_errors(m, kv[users], kv_o, cfg))
    assert_within(errs, TOL["bf16"])
    # the full forward of the same batch gives the same NS outputs
    s_tail, ns_full, kv2 = _run_full(m, S.cuda(), ns)
    assert torch.equal(kv2, kv)
    assert O.rel_l2(ns_full.double().cpu().numpy(), out.double().cpu().numpy()) < 2 * 2.0 ** -8


def test_onetrans_s_serving_sampled():
    wl = WORKLOADS["onetrans_s_serve"]
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)                    # [16, 512, 1024]
    m = model_of(wl, w)
    m.set_wait_limit(TEST_WAIT)
    kv, _ = m.encode_user(S.cuda(), want_s_tail=False)
    ns = m.auto_split(x.cuda())
    out = m.score_candidates(kv, ns)
    m.poll()
    users, cands = [3, 11], [0, 1, 100, 255, 256, 300, 510, 511]
    cfg = oracle_cfg(m)
    kv_o, _ = O.encode_user(cfg, w, S[users])
    ns_o = O.auto_split(x[users][:, cands], w["W_split"], wl.n_ns, wl.d)
    out_o = O.score_candidates(cfg, w, kv_o, ns_o)
    errs = {"ns_out": O.rel_l2(out[users][:, cands].double().cpu().numpy(), out_o)}
    errs.update(kv_errors(m, kv[users], kv_o, cfg))
    assert_within(errs, TOL["bf16"])


# ----------------------------------------------------------------- many items per CTA
def test_bf16_many_items_per_cta():
    """More (user, head, query pair) items than SMs in both attention modes, a
    ragged last pair and a pyramid layer whose second query tile is empty:
    every user against the CUDA-core path, sampled users against the oracle."""
    layers, d, H, f, N, L0 = 3, 128, 2, 256, 5, 520
    q = [520, 300, 45]
    U, C = 90, 60                      # NS rows per user: 300 (two pairs)
    w = rand_weights(layers, d, f, N, seed=31, dtype=torch.bfloat16)
    S, ns = rand_inputs(U, C, L0, N, d, seed=32, dtype=torch.bfloat16)
    m = make_model(w, layers=layers, d=d, heads=H, ffn=f, n_ns=N, L0=L0, q=q)
    m.set_wait_limit(TEST_WAIT)
    a = _run_full(m, S.cuda(), ns.cuda())
    users = [0, 47, 89]
    errs = _errors_vs_oracle(m, w, S, ns, *a, users)
    assert_within(errs, TOL["bf16"])
    m.set_kernel_path(1)
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert O.rel_l2(x.double().cpu().numpy(), y.double().cpu().numpy()) < 1e-2


# ----------------------------------------------------------------- host-buffer entry point
def test_full_forward_host_matches_device_path():
    """ot_full_forward_host (pinned host in / out, inputs staged through two
    alternating workspace slots on the model's copy stream) against Auto-Split
    + ot_full_forward on device tensors, bit for bit, over three back-to-back
    calls so both slots are used and one is reused."""
    wl = WORKLOADS["onetrans_s_full"]
    w = gen_weights(wl)
    m = model_of(wl, w)
    m.set_wait_limit(TEST_WAIT)
    groups = ([0, 1, 2], [3, 4, 5], [6, 7, 8])
    B, C = len(groups[0]), wl.cands
    ws = torch.empty(m.host_workspace_bytes(B, C), dtype=torch.uint8, device="cuda")
    host_runs, dev_runs = [], []
    for users in groups:
        S = gen_s_tokens(wl, users=users, weights=w)
        x = gen_auto_split_features(wl, users=users)
        S_h, x_h = S.pin_memory(), x.pin_memory()
        tail_h = torch.empty(B, m.q[-1], wl.d, dtype=m.storage).pin_memory()
        ns_h = torch.empty(B, C, wl.n_ns, wl.d, dtype=m.storage).pin_memory()
        m.full_forward_host(S_h, x_h, tail_h, ns_h, ws=ws)
        host_runs.append((S_h, x_h, tail_h, ns_h))
    torch.cuda.synchronize()
    m.poll()
    for S_h, x_h, tail_h, ns_h in host_runs:
        ns = m.auto_split(x_h.cuda())
        tail_d, ns_d = m.full_forward(S_h.cuda(), ns)
        m.poll()
        assert torch.equal(tail_h, tail_d.cpu()) and torch.equal(ns_h, ns_d.cpu())
    assert not torch.equal(host_runs[0][2], host_runs[1][2])


# ----------------------------------------------------------------- split-key NS attention
@pytest.mark.parametrize("shape", ["nq128_odd_even_blocks", "nq1_two_blocks", "nq80_partial_tiles"])
def test_split_key_ns_attention(shape):
    """NS attention with at most 128 query rows per (user, head): 128 and 80
    rows take the tensor-memory kernel's split-key mode (the two tiles of a
    CTA take alternate key blocks and merge their softmax states; layers with
    an even and an odd number of key blocks, a partly filled tile), a single
    row the decode-shaped kernel (key splits over four warps, a layer with
    two key blocks); every user against the oracle and the CUDA-core path."""
    if shape == "nq128_odd_even_blocks":
        layers, d, H, f, N, U, C, L0, q = 3, 128, 2, 256, 16, 4, 8, 260, [260, 200, 60]
    elif shape == "nq1_two_blocks":
        layers, d, H, f, N, U, C, L0, q = 3, 128, 2, 256, 1, 5, 1, 100, [100, 64, 1]
    else:
        layers, d, H, f, N, U, C, L0, q = 3, 128, 2, 256, 16, 3, 5, 200, [200, 150, 70]
    w = rand_weights(layers, d, f, N, seed=51, dtype=torch.bfloat16)
    S, ns = rand_inputs(U, C, L0, N, d, seed=52, dtype=torch.bfloat16)
    m = make_model(w, layers=layers, d=d, heads=H, ffn=f, n_ns=N, L0=L0, q=q)
    m.set_wait_limit(TEST_WAIT)
    a = _run_full(m, S.cuda(), ns.cuda())
    errs = _errors_vs_oracle(m, w, S, ns, *a, list(range(U)))
    assert_within(errs, TOL["bf16"])
    m.set_kernel_path(1)
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert O.rel_l2(x.double().cpu().numpy(), y.double().cpu().numpy()) < 1e-2


def test_ns_attention_two_row_tiles_ragged():
    """NS attention with 190 query rows per (user, head): both row tiles of a
    CTA live, the second partly past the last row (a warp with 30 live rows,
    two warps with none); 10 NS tokens per candidate, so NS key blocks split
    candidates and some warps see no key of a block.  Full forward (NS
    attention on the side stream) against the oracle and the CUDA-core path;
    cached scoring bit-identical to it."""
    layers, d, H, f, N, U, C, L0, q = 3, 128, 2, 1024, 10, 2, 19, 850, [850, 200, 100]
    w = rand_weights(layers, d, f, N, seed=61, dtype=torch.bfloat16)
    S, ns = rand_inputs(U, C, L0, N, d, seed=62, dtype=torch.bfloat16)
    m = make_model(w, layers=layers, d=d, heads=H, ffn=f, n_ns=N, L0=L0, q=q)
    m.set_wait_limit(TEST_WAIT)
    a = _run_full(m, S.cuda(), ns.cuda())
    errs = _errors_vs_oracle(m, w, S, ns, *a, list(range(U)))
    assert_within(errs, TOL["bf16"])
    kv2, _ = m.encode_user(S.cuda(), want_s_tail=False)
    sc = m.score_candidates(kv2, ns.cuda())
    m.poll()
    assert torch.equal(sc, a[1])
    m.set_kernel_path(1)
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert O.rel_l2(x.double().cpu().numpy(), y.double().cpu().numpy()) < 1e-2


# ----------------------------------------------------------------- fused feed-forward
@pytest.mark.parametrize("shape", ["small_d128", "onetrans_s_d256"])
def test_fused_ffn_matches_two_gemm_path(shape):
    """The fused kernel (output projection, then the FFN with its hidden kept
    on chip) against the three tensor-core GEMMs it replaces (kernel path 2),
    on the S side and the grouped NS side, both within the oracle tolerance.
    The fused kernel keeps H = X + A Wo^T in fp32 (the FFN's residual and the
    source of its normed input) where the GEMM path stores H as bf16, so
    after one layer they differ by one bf16 rounding of H and what follows
    from it (below one bf16 ulp, 2^-8, relative L2); through a pyramid of
    layers that compounds, and the stack is held to two bf16 ulps."""
    if shape == "small_d128":
        w1 = rand_weights(1, 128, 256, 5, seed=40, dtype=torch.bfloat16)
        w = rand_weights(3, 128, 256, 5, seed=41, dtype=torch.bfloat16)
        S, ns = rand_inputs(5, 40, 300, 5, 128, seed=42, dtype=torch.bfloat16)
        kw1 = dict(SMALL, layers=1, q=[300])
        kw = SMALL
    else:
        wl = WORKLOADS["onetrans_s_full"]
        base = dict(d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=600)
        w1 = rand_weights(1, wl.d, wl.ffn, wl.n_ns, seed=45, dtype=torch.bfloat16)
        w = rand_weights(2, wl.d, wl.ffn, wl.n_ns, seed=43, dtype=torch.bfloat16)
        S, ns = rand_inputs(6, 3, 600, wl.n_ns, wl.d, seed=44, dtype=torch.bfloat16)
        kw1 = dict(base, layers=1, q=[600])
        kw = dict(base, layers=2, q=[600, 300])
    for weights, shapes, tol in ((w1, kw1, 2.0 ** -8), (w, kw, 2 * 2.0 ** -8)):
        m = make_model(weights, **shapes)
        m.set_wait_limit(TEST_WAIT)
        a = _run_full(m, S.cuda(), ns.cuda())
        errs = _errors_vs_oracle(m, weights, S, ns, *a, [0, S.shape[0] - 1])
        assert_within(errs, TOL["bf16"])
        m.set_kernel_path(2)
        b = _run_full(m, S.cuda(), ns.cuda())
        errs = _errors_vs_oracle(m, weights, S, ns, *b, [0, S.shape[0] - 1])
        assert_within(errs, TOL["bf16"])
        for x, y in zip(a, b):
            assert O.rel_l2(x.double().cpu().numpy(), y.double().cpu().numpy()) < tol


# ----------------------------------------------------------------- full (non-causal) attention
def _full_model(w, path=0, **shapes):
    m = make_model(w, full_attn=True, **shapes)
    m.set_wait_limit(TEST_WAIT)
    m.set_kernel_path(path)
    return m


def _full_errors(m, w, S, ns, s_tail, ns_out, kv, users):
    cfg = oracle_cfg(m)
    cfg.full_attn = True
    js, jkv, jns = O.full_forward_joint(cfg, w, S[users], ns[users])
    errs = {"s_tail": O.rel_l2(s_tail[users].double().cpu().numpy(), js[:, 0]),
            "ns_out": O.rel_l2(ns_out[users].double().cpu().numpy(), jns)}
    errs.update(kv_errors(m, kv[users], jkv[:, 0], cfg))
    return errs


@pytest.mark.parametrize("path", [0, 1, 2], ids=["tcgen05_fused", "cuda_core", "tcgen05_two_gemm"])
def test_full_attention_parity(path):
    """Full attention (every token sees its whole sequence, one candidate per
    user) against the oracle's joint form: the tensor-core path with the S and
    NS sides in shared launches, the CUDA-core path and the two-GEMM FFN path
    (layer by layer: both sides' projections, then both attentions)."""
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=111, dtype=torch.bfloat16)
    S, ns = rand_inputs(4, 1, 300, 5, 128, seed=112, dtype=torch.bfloat16)
    m = _full_model(w, path, **shapes)
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns.cuda())
    assert_within(_full_errors(m, w, S, ns, s_tail, ns_out, kv, [0, 3]), TOL["bf16"])
    # the cached calls refuse a full-attention model; several candidates per user too
    with pytest.raises(ot.OtError) as e:
        m.encode_user(S.cuda())
    assert e.value.code == 10
    with pytest.raises(ot.OtError) as e:
        m.full_forward(S.cuda(), torch.cat([ns, ns], dim=1).cuda())
    assert e.value.code == 2


def test_full_attention_onetrans_s_shapes():
    """Full attention at the OneTransS widths (d = 256, 4 heads, 16 NS tokens,
    a 600 -> 300 pyramid) on sampled users against the oracle."""
    wl = WORKLOADS["onetrans_s_full"]
    shapes = dict(layers=2, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=600, q=[600, 300])
    w = rand_weights(2, wl.d, wl.ffn, wl.n_ns, seed=113, dtype=torch.bfloat16)
    S, ns = rand_inputs(6, 1, 600, wl.n_ns, wl.d, seed=114, dtype=torch.bfloat16)
    m = _full_model(w, 0, **shapes)
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns.cuda())
    assert_within(_full_errors(m, w, S, ns, s_tail, ns_out, kv, [0, 5]), TOL["bf16"])


def test_full_attention_tiny_fp32():
    """The tiny fp32 block with full attention (CUDA-core kernels) at 1e-5."""
    wl = WORKLOADS["tiny_fp32"]
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)[:, :1]                 # one candidate
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    m = make_model(w, layers=wl.layers, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns,
                   L0=wl.L0, q=q, F=wl.F, eps=wl.eps, dtype="f32", full_attn=True)
    ns = m.auto_split(x.cuda())
    s_tail, ns_out, kv = _run_full(m, S.cuda(), ns)
    cfg = oracle_cfg(m)
    cfg.full_attn = True
    ns_o = O.auto_split(x, w["W_split"], wl.n_ns, wl.d)
    js, jkv, jns = O.full_forward_joint(cfg, w, S, ns_o)
    errs = {"s_tail": O.rel_l2(s_tail.double().cpu().numpy(), js[:, 0]),
            "ns_out": O.rel_l2(ns_out.double().cpu().numpy(), jns)}
    errs.update(kv_errors(m, kv, jkv[:, 0], cfg))
    assert_within(errs, TOL["f32"])


def test_full_attention_mask_probe_bitexact():
    """The mask probe of the causal test with full attention: every output
    row has a non-zero in every S column and every NS column of its user."""
    L0, N, d, q = 100, 8, 128, 60
    w = rand_weights(1, d, 256, N, seed=5, dtype=torch.bfloat16)
    eye = torch.eye(d, dtype=torch.bfloat16)
    for k, shape in (("Wqkv_s", (1, 3 * d, d)), ("Wqkv_ns", (1, N, 3 * d, d))):
        t = torch.zeros(shape, dtype=torch.bfloat16)
        t[..., 2 * d:, :] = eye
        w[k] = t
    w["g1_s"] = torch.ones_like(w["g1_s"])
    w["g1_ns"] = torch.ones_like(w["g1_ns"])
    w["Wo_s"] = eye.expand(1, d, d).clone()
    w["Wo_ns"] = eye.expand(1, N, d, d).clone()
    w["W2_s"] = torch.zeros_like(w["W2_s"])
    w["W2_ns"] = torch.zeros_like(w["W2_ns"])
    S = torch.zeros(2, L0, d, dtype=torch.bfloat16)
    S[:, torch.arange(L0), torch.arange(L0)] = 1
    ns = torch.zeros(2, 1, N, d, dtype=torch.bfloat16)
    ns[:, 0, torch.arange(N), L0 + torch.arange(N)] = 1
    want = torch.zeros(d, dtype=torch.bool)
    want[:L0 + N] = True
    for path in (0, 1):
        m = _full_model(w, path, layers=1, d=d, heads=2, ffn=256, n_ns=N, L0=L0, q=[q])
        s_tail, ns_out, _ = _run_full(m, S.cuda(), ns.cuda())
        assert torch.equal(s_tail.float().cpu() != 0, want.expand(2, q, d)), path
        assert torch.equal(ns_out.float().cpu() != 0, want.expand(2, 1, N, d)), path


# ----------------------------------------------------------------- sparse mixture of experts
def _moe_inputs(U, C, L0, N, d, E, seed):
    """S rows whose router logits are decisive: row t carries a large
    component on coordinate t % E (its first expert) and a smaller one on a
    second coordinate (its second expert), and the router reads those
    coordinates, so no rounding difference between the GPU and the oracle
    can swap the chosen experts (both sides decide in their own precision)."""
    S, ns = rand_inputs(U, C, L0, N, d, seed=seed, dtype=torch.float32)
    t = torch.arange(L0)
    e1 = t % E
    e2 = (t + 1 + t // E) % E
    e2 = torch.where(e2 == e1, (e1 + 1) % E, e2)
    S[:, t, e1] += 45.0
    S[:, t, e2] += 22.0
    return S.to(torch.bfloat16), ns.to(torch.bfloat16)


def _moe_weights(layers, d, f, N, E, seed):
    w = rand_weights(layers, d, f, N, seed=seed, dtype=torch.bfloat16, experts=E)
    r = torch.zeros(layers, E, d)
    r[:, torch.arange(E), torch.arange(E)] = 0.3
    w["W_router"] = r.to(torch.bfloat16)
    return w


@pytest.mark.parametrize("topk", [1, 2])
@pytest.mark.parametrize("path", [0, 1, 2], ids=["tcgen05_fused", "cuda_core", "tcgen05_two_gemm"])
def test_moe_parity(path, topk):
    """The sparse-MoE S-side FFN (router, expert-major rows, the experts' FFN,
    combine) against the oracle: the fused-FFN path computing only each
    expert's filled rows, the CUDA-core path and the two-GEMM path; the NS
    side keeps its dense private FFNs; cached scoring matches the full
    forward, and a second run is bit-identical (the slots an expert's rows
    take depend on atomic order, the results must not)."""
    E = 4
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = _moe_weights(3, 128, 256, 5, E, seed=121)
    S, ns = _moe_inputs(3, 4, 300, 5, 128, E, seed=122)
    m = make_model(w, moe_experts=E, moe_topk=topk, **shapes)
    m.set_wait_limit(TEST_WAIT)
    m.set_kernel_path(path)
    a = _run_full(m, S.cuda(), ns.cuda())
    errs = _errors_vs_oracle(m, w, S, ns, *a, [0, 2])
    assert_within(errs, TOL["bf16"])
    b = _run_full(m, S.cuda(), ns.cuda())
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    kv2, s2 = m.encode_user(S.cuda())
    sc = m.score_candidates(kv2, ns.cuda())
    m.poll()
    assert torch.equal(kv2, a[2]) and torch.equal(s2, a[0]) and torch.equal(sc, a[1])


def test_moe_onetrans_s_shapes():
    """Eight experts, top-2, at the OneTransS widths (d = 256, 4 heads, FFN
    1024, 16 NS tokens, 600 -> 300 pyramid): sampled users against the
    oracle."""
    E = 8
    wl = WORKLOADS["onetrans_s_full"]
    shapes = dict(layers=2, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=600, q=[600, 300])
    w = _moe_weights(2, wl.d, wl.ffn, wl.n_ns, E, seed=123)
    S, ns = _moe_inputs(6, 2, 600, wl.n_ns, wl.d, E, seed=124)
    m = make_model(w, moe_experts=E, moe_topk=2, **shapes)
    m.set_wait_limit(TEST_WAIT)
    a = _run_full(m, S.cuda(), ns.cuda())
    assert_within(_errors_vs_oracle(m, w, S, ns, *a, [1, 4]), TOL["bf16"])


# ----------------------------------------------------------------- paged KV cache
def _page_table(m, U, n_pages, seed, share=None):
    """A random assignment of distinct pages to every (user, layer block);
    share = (a, b): user b lists user a's pages (their rows are identical)."""
    ppu = m.kv_pages_per_user()
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[: U * ppu].view(U, ppu)
    if share:
        perm[share[1]] = perm[share[0]]
    return perm.to(torch.int32).cuda()


@pytest.mark.parametrize("shape", ["small", "onetrans_s_c1", "onetrans_s_c8"])
def test_paged_cache_matches_dense_cache(shape):
    """ot_encode_user_paged / ot_score_candidates_paged against the dense
    cache, bit for bit: the S tails, the NS outputs and every layer's K / V
    gathered from the pages (shuffled page ids in a pool with spare pages;
    layers whose last page is partly used); small-NS, split-key and
    two-tile NS attention read the pages."""
    if shape == "small":
        shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
        U, C = 3, 7
    else:
        wl = WORKLOADS["onetrans_s_full"]
        shapes = dict(layers=3, d=wl.d, heads=wl.heads, ffn=wl.ffn, n_ns=wl.n_ns, L0=700,
                      q=[700, 333, 60])
        U, C = 4, (1 if shape == "onetrans_s_c1" else 8)
    w = rand_weights(shapes["layers"], shapes["d"], shapes["ffn"], shapes["n_ns"], seed=131,
                     dtype=torch.bfloat16)
    S, ns = rand_inputs(U, C, shapes["L0"], shapes["n_ns"], shapes["d"], seed=132, dtype=torch.bfloat16)
    m = make_model(w, **shapes)
    m.set_wait_limit(TEST_WAIT)
    Sd, nsd = S.cuda(), ns.cuda()
    kv, s_dense = m.encode_user(Sd)
    out_dense = m.score_candidates(kv, nsd)
    n_pages = U * m.kv_pages_per_user() + 9
    pool = m.new_page_pool(n_pages)
    pool.fill_(float("nan"))  # stale pages: nothing unwritten may leak into the results
    pages = _page_table(m, U, n_pages, seed=133)
    s_paged = m.encode_user_paged(Sd, pool, pages)
    out_paged = m.score_candidates_paged(pool, pages, nsd)
    m.poll()
    assert torch.equal(s_paged, s_dense)
    assert torch.equal(out_paged, out_dense)
    for u in range(U):
        for l in range(m.layers):
            K, V = m.kv_from_pages(pool, pages[u].cpu(), l)
            Kd, Vd = m.kv_layer(kv[u], l)
            assert torch.equal(K, Kd) and torch.equal(V, Vd), (u, l)


def test_paged_cache_fp8_per_tensor_matches_dense_cache():
    """FP8 with per-tensor activation scales (the e4m3 hidden written by the
    first FFN projection) through the paged calls: bit for bit the dense
    cache's S tails, NS outputs and K / V."""
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=137, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 6, 300, 5, 128, seed=138, dtype=torch.bfloat16)
    m = make_model(w, dtype="fp8", **shapes)
    m.set_wait_limit(TEST_WAIT)
    scales, _ = O.calibrate(oracle_cfg(m), w, S[:1], ns[:1])
    m.set_act_scales(scales)
    Sd, nsd = S.cuda(), ns.cuda()
    kv, s_dense = m.encode_user(Sd)
    out_dense = m.score_candidates(kv, nsd)
    n_pages = 3 * m.kv_pages_per_user() + 5
    pool = m.new_page_pool(n_pages)
    pool.fill_(float("nan"))
    pages = _page_table(m, 3, n_pages, seed=139)
    s_paged = m.encode_user_paged(Sd, pool, pages)
    out_paged = m.score_candidates_paged(pool, pages, nsd)
    m.poll()
    assert torch.equal(s_paged, s_dense) and torch.equal(out_paged, out_dense)
    for u in range(3):
        for l in range(m.layers):
            K, V = m.kv_from_pages(pool, pages[u].cpu(), l)
            Kd, Vd = m.kv_layer(kv[u], l)
            assert torch.equal(K, Kd) and torch.equal(V, Vd), (u, l)


def test_paged_cache_shared_prefix_pages():
    """Users with identical S rows list the same pages (a shared prefix
    covering the whole sequence): their results equal each other and the
    dense cache's, and a third user with its own pages is unaffected."""
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=134, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 4, 300, 5, 128, seed=135, dtype=torch.bfloat16)
    S[1] = S[0]
    m = make_model(w, **shapes)
    m.set_wait_limit(TEST_WAIT)
    n_pages = 3 * m.kv_pages_per_user()
    pool = m.new_page_pool(n_pages)
    pages = _page_table(m, 3, n_pages, seed=136, share=(0, 1))
    s_paged = m.encode_user_paged(S.cuda(), pool, pages)
    out_paged = m.score_candidates_paged(pool, pages, ns.cuda())
    kv, s_dense = m.encode_user(S.cuda())
    out_dense = m.score_candidates(kv, ns.cuda())
    m.poll()
    assert torch.equal(s_paged, s_dense) and torch.equal(out_paged, out_dense)
    assert torch.equal(s_paged[0], s_paged[1])


def test_paged_cache_fp32_cuda_core_and_oracle():
    """The tiny fp32 block on the CUDA-core kernels with a paged cache,
    against the oracle at 1e-5."""
    wl = WORKLOADS["tiny_fp32"]
    w = gen_weights(wl)
    S = gen_s_tokens(wl, weights=w)
    x = gen_auto_split_features(wl)
    m = model_of(wl, w)
    ns = m.auto_split(x.cuda())
    pool = m.new_page_pool(m.kv_pages_per_user() + 2)
    pages = _page_table(m, 1, pool.shape[0], seed=137)
    s_tail = m.encode_user_paged(S.cuda(), pool, pages)
    out = m.score_candidates_paged(pool, pages, ns)
    m.poll()
    cfg = oracle_cfg(m)
    kv_o, s_o = O.encode_user(cfg, w, S)
    out_o = O.score_candidates(cfg, w, kv_o, O.auto_split(x, w["W_split"], wl.n_ns, wl.d))
    errs = {"s_tail": O.rel_l2(s_tail.double().cpu().numpy(), s_o),
            "ns_out": O.rel_l2(out.double().cpu().numpy(), out_o)}
    assert_within(errs, TOL["f32"])


def test_paged_cache_bad_page_id_is_reported():
    """A page id outside the pool is never dereferenced: the call completes,
    the device error word reports OT_ERR_DEVICE_BOUNDS, and the context is
    fine for the next call."""
    shapes = dict(layers=2, d=128, heads=2, ffn=256, n_ns=3, L0=200, q=[200, 90])
    w = rand_weights(2, 128, 256, 3, seed=138, dtype=torch.bfloat16)
    S, ns = rand_inputs(2, 2, 200, 3, 128, seed=139, dtype=torch.bfloat16)
    m = make_model(w, **shapes)
    m.set_wait_limit(TEST_WAIT)
    n_pages = 2 * m.kv_pages_per_user()
    pool = m.new_page_pool(n_pages)
    pages = _page_table(m, 2, n_pages, seed=140)
    bad = pages.clone()
    bad[1, 1] = n_pages + 5
    m.encode_user_paged(S.cuda(), pool, bad)
    with pytest.raises(ot.OtError) as e:
        m.poll()
    assert e.value.code == 9
    s_tail = m.encode_user_paged(S.cuda(), pool, pages)
    m.poll()
    kv, s_dense = m.encode_user(S.cuda())
    m.poll()
    assert torch.equal(s_tail, s_dense)
