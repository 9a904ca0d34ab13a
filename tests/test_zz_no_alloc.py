"""ot_score_candidates_noalloc: candidate scoring for callers that cannot
allocate device memory (serving runtimes that forbid allocation on the
request path, hosts that own all GPU memory in their own pool).  It scores
into the library's fixed device scratch instead of a caller workspace; its
results must match ot_score_candidates on the same inputs, call after call,
and the oracle.

The file name sorts last, so pytest collects it after every other test file:
a -x run that stops here has already run everything else.  The tests pass
both on their own in a fresh process and after the other tests.
"""

from __future__ import annotations

import ctypes as C

import pytest
import torch

from gpu_common import TOL, make_model, oracle_cfg
from helpers import rand_inputs, rand_weights
from oracle import oracle as O
from unified_transformer_recommender_onetrans_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()


def _raw_noalloc(m, kv, ns, out, U=None, Cn=None):
    """Call the entry point through the C ABI directly."""
    stream = torch.cuda.current_stream().cuda_stream
    U = ns.shape[0] if U is None else U
    Cn = ns.shape[1] if Cn is None else Cn
    return B.lib().ot_score_candidates_noalloc(m.handle, C.c_void_p(kv.data_ptr()), U,
                                               C.c_void_p(ns.data_ptr()), Cn,
                                               C.c_void_p(out.data_ptr()), C.c_void_p(stream))


def test_noalloc_scoring_matches_workspace_scoring_twice():
    shapes = dict(layers=3, d=128, heads=2, ffn=256, n_ns=5, L0=300, q=[300, 170, 37])
    w = rand_weights(3, 128, 256, 5, seed=301, dtype=torch.bfloat16)
    S, ns = rand_inputs(3, 7, 300, 5, 128, seed=302, dtype=torch.bfloat16)
    m = make_model(w, **shapes)
    kv, _ = m.encode_user(S.cuda(), want_s_tail=False)
    nsd = ns.cuda()
    ref = m.score_candidates(kv, nsd)
    m.poll()
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the same scratch
        out = torch.full_like(nsd, float("nan"))
        assert _raw_noalloc(m, kv, nsd, out) == 0
        m.poll()
        outs.append(out)
    for out in outs:
        err = O.rel_l2(out.double().cpu().numpy(), ref.double().cpu().numpy())
        assert err <= TOL["bf16"], err
        assert torch.equal(out, ref)
    # and against the oracle directly, on two users
    cfg = oracle_cfg(m)
    users = [0, 2]
    kv_o, _ = O.encode_user(cfg, w, S[users])
    ns_o = O.score_candidates(cfg, w, kv_o, ns[users])
    err = O.rel_l2(outs[1][users].double().cpu().numpy(), ns_o)
    assert err <= TOL["bf16"], err


def test_noalloc_rejects_requests_beyond_its_scratch():
    w = rand_weights(1, 128, 256, 5, seed=303, dtype=torch.bfloat16)
    m = make_model(w, layers=1, d=128, heads=2, ffn=256, n_ns=5, L0=64, q=[64])
    S, _ = rand_inputs(1, 1, 64, 5, 128, seed=304, dtype=torch.bfloat16)
    kv, _ = m.encode_user(S.cuda(), want_s_tail=False)
    # 7 * rows * d + rows * ffn bf16 elements per call: pick C so it exceeds 16 MiB
    per_row = (7 * 128 + 256) * 2
    C_big = (16 << 20) // (per_row * 5) + 64
    ns = torch.zeros(1, C_big, 5, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(ns)
    assert _raw_noalloc(m, kv, ns, out) == 6  # OT_ERR_WORKSPACE_TOO_SMALL
    # shape and alignment are checked first, as ot_score_candidates checks them
    assert _raw_noalloc(m, kv, ns, out, Cn=(1 << 30) // 5 + 1) == 2  # OT_ERR_SHAPE
    bad = torch.empty(ns.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:]
    stream = torch.cuda.current_stream().cuda_stream
    rc = B.lib().ot_score_candidates_noalloc(m.handle, C.c_void_p(kv.data_ptr()), 1,
                                             C.c_void_p(bad.data_ptr()), C_big,
                                             C.c_void_p(out.data_ptr()), C.c_void_p(stream))
    assert rc == 4  # OT_ERR_ALIGN
    m.poll()
