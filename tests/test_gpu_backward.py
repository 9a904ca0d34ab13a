"""GPU parity of the backward pass (ot_full_backward, fp32, activation
checkpointing) against the oracle's gradients (fp64 restatement of the
forward + autograd, pinned to finite differences of the C oracle).

Tolerance: max relative L2 error per gradient tensor of 1e-4.  The forward's
fp32 bound is 1e-5 per output tensor; a gradient is a product of the
forward's Jacobians taken in the opposite order, over twice the chain of
rounded fp32 steps (the recomputed forward, then the backward), and the
softmax / RMSNorm backward subtract nearly equal terms (p (dp - D),
r g dz - x c), which loses about one more digit: 10x the forward's bound."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import unified_transformer_recommender_onetrans_b200 as ot
from helpers import rand_inputs, rand_weights
from oracle import backward as OB
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TOL_GRAD = 1e-4
TOL_FWD = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()


def _case(layers, d, heads, ffn, N, L0, q, U, C, seed, full=False, experts=0, topk=1):
    w = rand_weights(layers, d, ffn, N, seed=seed, experts=experts)
    S, ns = rand_inputs(U, max(C, 1), L0, N, d, seed=seed + 1)
    ns = ns[:, :C].contiguous()
    g = torch.Generator().manual_seed(seed + 2)
    G_s = torch.randn(U, q[-1], d, generator=g)
    G_ns = torch.randn(U, C, N, d, generator=g)
    cfg = ot.make_config(layers=layers, d=d, heads=heads, ffn=ffn, n_ns=N, L0=L0, q=q, full_attn=full,
                         moe_experts=experts, moe_topk=topk)
    ocfg = O.Config(layers, d, heads, ffn, N, L0, list(q), 1e-6)
    ocfg.full_attn = full
    ocfg.moe_experts, ocfg.moe_topk = experts, topk
    return cfg, ocfg, w, S, ns, G_s, G_ns


def _run(cfg, w, S, ns, G_s, G_ns):
    dw = {k: v.cuda() for k, v in w.items()}
    C = ns.shape[1]
    out = ot.full_backward(cfg, dw, S.cuda(), ns.cuda() if C else None, G_s.cuda(),
                           G_ns.cuda() if C else None)
    torch.cuda.synchronize()
    return out


def _errors(ocfg, w, S, ns, G_s, G_ns, out):
    s_tail, ns_out, grads, dS, dns = out
    C = ns.shape[1]
    w64 = {k: w[k].double() for k in OB.names(ocfg)}
    if C:
        ns_o_in, G_ns_o = ns.double(), G_ns.double()
    else:
        # no candidates: the oracle takes one with a zero upstream gradient,
        # which adds nothing to any S-side gradient (S rows never see NS rows)
        ns_o_in = torch.randn(S.shape[0], 1, ocfg.n_ns, ocfg.d, dtype=torch.float64)
        G_ns_o = torch.zeros_like(ns_o_in)
    _, want = OB.gradients(ocfg, w64, S.double(), ns_o_in, G_s.double(), G_ns_o)
    moe = getattr(ocfg, "moe_experts", 0)
    errs = {k: O.rel_l2(grads[k].double().cpu().numpy(), want[k].numpy())
            for k in OB.names(ocfg) if (C or not k.endswith("_ns")) and not (moe and k in ("W1_s", "W2_s"))}
    if moe:
        for k in ("W1_s", "W2_s"):
            assert torch.count_nonzero(grads[k]) == 0, k
    errs["S"] = O.rel_l2(dS.double().cpu().numpy(), want["S"].numpy())
    fwd = {}
    s_o, ns_o = OB.forward(ocfg, w64, S.double(), ns_o_in)
    fwd["s_tail"] = O.rel_l2(s_tail.double().cpu().numpy(), s_o.detach().numpy())
    if C:
        errs["ns"] = O.rel_l2(dns.double().cpu().numpy(), want["ns"].numpy())
        fwd["ns_out"] = O.rel_l2(ns_out.double().cpu().numpy(), ns_o.detach().numpy())
    else:
        for k in OB.W_NAMES:
            if k.endswith("_ns"):
                assert torch.count_nonzero(grads[k]) == 0, k
    return errs, fwd


CASES = {
    # several GEMM tiles with ragged tails (300 S rows, d = 128, ffn = 192),
    # head dim 64, a pyramid 150 -> 61
    "hd64_ragged": dict(layers=2, d=128, heads=2, ffn=192, N=4, L0=150, q=[150, 61], U=2, C=3),
    # head dim 32, three layers, a one-row tail
    "hd32_3layers": dict(layers=3, d=64, heads=2, ffn=96, N=3, L0=40, q=[33, 9, 1], U=2, C=2),
    # head dim 16, one candidate, one NS token
    "hd16_n1": dict(layers=1, d=64, heads=4, ffn=64, N=1, L0=70, q=[70], U=3, C=1),
}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name):
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(**CASES[name], seed=300 + len(name))
    errs, fwd = _errors(ocfg, w, S, ns, G_s, G_ns, _run(cfg, w, S, ns, G_s, G_ns))
    assert max(fwd.values()) <= TOL_FWD, fwd
    assert max(errs.values()) <= TOL_GRAD, {k: f"{v:.2e}" for k, v in errs.items()}


FULL_CASES = {
    # full attention, one candidate per user: S rows also see the NS keys
    "hd64_ragged": dict(layers=2, d=128, heads=2, ffn=192, N=4, L0=150, q=[150, 61], U=2, C=1),
    "hd16_3layers": dict(layers=3, d=64, heads=4, ffn=96, N=3, L0=70, q=[70, 33, 1], U=3, C=1),
}


@pytest.mark.parametrize("name", list(FULL_CASES))
def test_backward_full_attention_parity(name):
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(**FULL_CASES[name], seed=800 + len(name), full=True)
    errs, fwd = _errors(ocfg, w, S, ns, G_s, G_ns, _run(cfg, w, S, ns, G_s, G_ns))
    assert max(fwd.values()) <= TOL_FWD, fwd
    assert max(errs.values()) <= TOL_GRAD, {k: f"{v:.2e}" for k, v in errs.items()}


def test_backward_full_attention_matches_full_forward():
    """The backward's recomputed outputs equal what the library's own full
    forward (ot_full_forward, fp32, full attention) computes, to fp32
    rounding."""
    spec = dict(FULL_CASES["hd64_ragged"])
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(**spec, seed=901, full=True)
    s_tail, ns_out, _, _, _ = _run(cfg, w, S, ns, G_s, G_ns)
    from gpu_common import make_model
    m = make_model(w, layers=spec["layers"], d=spec["d"], heads=spec["heads"], ffn=spec["ffn"],
                   n_ns=spec["N"], L0=spec["L0"], q=spec["q"], dtype="f32", full_attn=True)
    s_f, ns_f = m.full_forward(S.cuda(), ns.cuda())
    m.poll()
    assert O.rel_l2(s_tail.double().cpu().numpy(), s_f.double().cpu().numpy()) < 1e-5
    assert O.rel_l2(ns_out.double().cpu().numpy(), ns_f.double().cpu().numpy()) < 1e-5


def _moe_decisive(w, experts, layers, d, scale=4.0):
    """Router weights that read a few coordinates strongly, so the logit gaps
    between experts are far above fp32 rounding (the GPU routes in fp32, the
    oracle in fp64: the same choices need clear margins)."""
    g = torch.Generator().manual_seed(1234)
    wr = torch.zeros(layers, experts, d)
    for l in range(layers):
        for e in range(experts):
            wr[l, e, (7 * e + l) % d] = scale * (1.0 + 0.37 * e)
            wr[l, e] += 0.05 * torch.randn(d, generator=g)
    w["W_router"] = wr
    return w


MOE_CASES = {
    "top1_e3": dict(layers=2, d=64, heads=2, ffn=96, N=3, L0=90, q=[90, 41], U=2, C=2, experts=3, topk=1),
    "top2_e4": dict(layers=2, d=128, heads=2, ffn=192, N=2, L0=150, q=[150, 61], U=2, C=2, experts=4, topk=2),
}


@pytest.mark.parametrize("name", list(MOE_CASES))
def test_backward_moe_parity(name, monkeypatch):
    """A mixture-of-experts S-side FFN: gradients of the router, the
    experts and every other tensor against the oracle (the routing margins
    are checked to be clear of fp32 rounding first)."""
    spec = MOE_CASES[name]
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(**spec, seed=950 + len(name))
    w = _moe_decisive(w, spec["experts"], spec["layers"], spec["d"])
    seen = []
    orig = OB._s_ffn

    def spy(c_, w_, l, h):
        seen.append((l, h.detach()))
        return orig(c_, w_, l, h)
    monkeypatch.setattr(OB, "_s_ffn", spy)
    OB.forward(ocfg, {k: v.double() for k, v in w.items()}, S.double(), ns.double())
    monkeypatch.setattr(OB, "_s_ffn", orig)
    for l, h in seen:
        z = OB._rms(h, w["g2_s"][l].double(), 1e-6)
        lg = torch.sort(z @ w["W_router"][l].double().T, dim=-1, descending=True).values
        assert float((lg[:, spec["topk"] - 1] - lg[:, spec["topk"]]).min()) > 1e-3
    errs, fwd = _errors(ocfg, w, S, ns, G_s, G_ns, _run(cfg, w, S, ns, G_s, G_ns))
    assert max(fwd.values()) <= TOL_FWD, fwd
    assert max(errs.values()) <= TOL_GRAD, {k: f"{v:.2e}" for k, v in errs.items()}


def test_backward_s_only():
    """C = 0: the S side alone; the NS gradients are zero."""
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(layers=2, d=64, heads=2, ffn=128, N=2, L0=90, q=[50, 20],
                                           U=2, C=0, seed=411)
    errs, fwd = _errors(ocfg, w, S, ns, G_s, G_ns, _run(cfg, w, S, ns, G_s, G_ns))
    assert max(fwd.values()) <= TOL_FWD, fwd
    assert max(errs.values()) <= TOL_GRAD, {k: f"{v:.2e}" for k, v in errs.items()}


def test_backward_deterministic_and_optional_outputs():
    """Same inputs, same bits; leaving out the forward outputs and the input
    gradients changes none of the weight gradients."""
    cfg, _, w, S, ns, G_s, G_ns = _case(**CASES["hd32_3layers"], seed=512)
    a = _run(cfg, w, S, ns, G_s, G_ns)
    b = _run(cfg, w, S, ns, G_s, G_ns)
    for k in ot.GRAD_NAMES:
        assert torch.equal(a[2][k], b[2][k]), k
    assert torch.equal(a[3], b[3]) and torch.equal(a[4], b[4])
    dw = {k: w[k].cuda() for k in ot.GRAD_NAMES}
    _, _, g2, dS2, dns2 = ot.full_backward(cfg, dw, S.cuda(), ns.cuda(), G_s.cuda(), G_ns.cuda(),
                                           want_outputs=False, want_input_grads=False)
    torch.cuda.synchronize()
    assert dS2 is None and dns2 is None
    for k in ot.GRAD_NAMES:
        assert torch.equal(a[2][k], g2[k]), k


def test_backward_rejects():
    cfg, _, w, S, ns, G_s, G_ns = _case(**CASES["hd16_n1"], seed=600)
    dw = {k: w[k].cuda() for k in ot.GRAD_NAMES}
    args = (dw, S.cuda(), ns.cuda(), G_s.cuda(), G_ns.cuda())
    bad = ot.make_config(layers=1, d=64, heads=4, ffn=64, n_ns=1, L0=70, q=[70], dtype="bf16")
    with pytest.raises(ot.OtError, match="DTYPE"):
        ot.full_backward(bad, *args)
    bad = ot.make_config(layers=1, d=64, heads=4, ffn=64, n_ns=1, L0=70, q=[70], moe_experts=2)
    with pytest.raises(ot.OtError, match="ARG"):  # a mixture without its router and experts
        ot.full_backward(bad, *args)
    bad = ot.make_config(layers=1, d=64, heads=4, ffn=64, n_ns=1, L0=70, q=[71])
    with pytest.raises(ot.OtError, match="SHAPE"):
        ot.full_backward(bad, *args)
    small = torch.empty(ot.backward_workspace_bytes(cfg, 3, 1) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ot.OtError, match="WORKSPACE"):
        ot.full_backward(cfg, *args, ws=small)
    assert ot.backward_workspace_bytes(bad, 3, 1) == 0
    assert ot.backward_launches(cfg, 3, 1) > 0


def test_backward_onetrans_s_sampled():
    """OneTransS shapes in fp32 (6 layers, d = 256, 4 heads, ffn 1024, 16 NS
    tokens, pyramid 1190 -> 12), 4 users x 2 candidates; gradients of the
    whole batch against the oracle's on the first user (the users are
    independent, so user 0's input gradients and its share of the weight
    gradients follow from user 0 alone): dS and dns of user 0 in full, the
    weight gradients as the difference of two runs, with and without user
    0's upstream gradients."""
    layers, d, H, f, N, L0 = 6, 256, 4, 1024, 16, 1190
    q = ot.pyramid_schedule(L0, 12, layers)
    cfg, ocfg, w, S, ns, G_s, G_ns = _case(layers, d, H, f, N, L0, q, U=4, C=2, seed=700)
    full = _run(cfg, w, S, ns, G_s, G_ns)
    G_s0, G_ns0 = G_s.clone(), G_ns.clone()
    G_s0[0] = 0
    G_ns0[0] = 0
    rest = _run(cfg, w, S, ns, G_s0, G_ns0)
    w64 = {k: w[k].double() for k in OB.W_NAMES}
    _, want = OB.gradients(ocfg, w64, S[:1].double(), ns[:1].double(), G_s[:1].double(),
                           G_ns[:1].double())
    errs = {"S": O.rel_l2(full[3][0:1].double().cpu().numpy(), want["S"].numpy()),
            "ns": O.rel_l2(full[4][0:1].double().cpu().numpy(), want["ns"].numpy())}
    for k in OB.W_NAMES:
        diff = (full[2][k].double() - rest[2][k].double()).cpu().numpy()
        # the difference of two fp32 sums of the whole batch: its rounding is
        # relative to the batch's gradient, not to user 0's share
        scale = np.linalg.norm(full[2][k].double().cpu().numpy()) / np.linalg.norm(want[k].numpy())
        errs[k] = O.rel_l2(diff, want[k].numpy()) / max(1.0, scale)
    assert max(errs.values()) <= TOL_GRAD, {k: f"{v:.2e}" for k, v in errs.items()}
