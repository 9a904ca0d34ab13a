"""GPU parity of ot_encode_append (appending S rows to encoded users) against
the oracle's encode of the whole grown sequence, through the C ABI.

The grown model has L0 and every query tail longer by the appended rows (the
pyramid windows stay anchored at their first row); the old cache comes from a
model with the shorter schedule and the same weights.
"""

from __future__ import annotations

import pytest
import torch

from gpu_common import TOL, assert_within, kv_errors, make_model, oracle_cfg
from helpers import rand_inputs, rand_weights
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TEST_WAIT = 1 << 22


@pytest.fixture(scope="module", autouse=True)
def _build():
    from unified_transformer_recommender_onetrans_b200.build import build
    build()
    assert torch.cuda.is_available()


def _models(w, dtype, layers, d, H, f, N, L0, q, delta):
    kw = dict(layers=layers, d=d, heads=H, ffn=f, n_ns=N, dtype=dtype)
    old = make_model(w, L0=L0, q=q, **kw)
    new = make_model(w, L0=L0 + delta, q=[v + delta for v in q], **kw)
    for m in (old, new):
        m.set_wait_limit(TEST_WAIT)
    return old, new


CASES = {
    # dtype, layers, d, H, ffn, N, U, L0, q (old), delta
    "bf16_ragged_70": ("bf16", 3, 128, 2, 256, 4, 3, 300, [300, 180, 40], 70),
    "bf16_one_row": ("bf16", 2, 128, 2, 256, 4, 2, 257, [257, 129], 1),
    "bf16_two_tiles_of_new_rows": ("bf16", 2, 256, 4, 1024, 3, 2, 150, [150, 20], 300),
    "f32": ("f32", 2, 64, 2, 256, 3, 2, 40, [40, 12], 9),
}


@pytest.mark.parametrize("case", list(CASES))
def test_append_matches_oracle_of_grown_sequence(case):
    """Old cache (GPU encode of the first L0 rows) + append of delta rows:
    the grown cache (every layer's K and V, old rows included) and the new
    rows' final outputs against the oracle encode of all L0 + delta rows with
    the grown schedule; candidates scored against the grown cache against
    the oracle's scores; and the same against the GPU's own full encode of
    the grown sequence (close to rounding)."""
    dtype, layers, d, H, f, N, U, L0, q, delta = CASES[case]
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    w = rand_weights(layers, d, f, N, seed=91, dtype=tdt)
    S, ns = rand_inputs(U, 2, L0 + delta, N, d, seed=92, dtype=tdt)
    old, new = _models(w, dtype, layers, d, H, f, N, L0, q, delta)
    kv_old, _ = old.encode_user(S[:, :L0].contiguous().cuda(), want_s_tail=False)
    kv, out_new = new.encode_append(kv_old, S[:, L0:].contiguous().cuda())
    new.poll()
    cfg = oracle_cfg(new)
    kv_o, s_o = O.encode_user(cfg, w, S)
    errs = {"out_new": O.rel_l2(out_new.double().cpu().numpy(), s_o[:, -delta:])}
    errs.update(kv_errors(new, kv, kv_o, cfg))
    sc = new.score_candidates(kv, ns.cuda())
    new.poll()
    errs["ns_out"] = O.rel_l2(sc.double().cpu().numpy(), O.score_candidates(cfg, w, kv_o, ns))
    assert_within(errs, TOL[dtype])
    # the GPU's full encode of the grown sequence: the appended path differs
    # from it only in which rows share a tile (summation order and the
    # reference max of the softmax), so they agree to a few rounding steps
    kv_f, s_f = new.encode_user(S.cuda())
    new.poll()
    close = 1e-6 if dtype == "f32" else 4 * 2.0 ** -8
    assert O.rel_l2(kv.double().cpu().numpy(), kv_f.double().cpu().numpy()) < close
    assert O.rel_l2(out_new.double().cpu().numpy(), s_f[:, -delta:].double().cpu().numpy()) < close


def test_append_twice_and_old_rows_unchanged():
    """Two appends in a row (37 rows, then 5) give the oracle's encode of the
    whole sequence; the old rows' K/V are copied bit for bit into the grown
    layout; the CUDA-core path agrees."""
    layers, d, H, f, N, U, L0, q = 3, 128, 2, 256, 4, 2, 200, [200, 120, 50]
    w = rand_weights(layers, d, f, N, seed=93, dtype=torch.bfloat16)
    S, _ = rand_inputs(U, 1, L0 + 42, N, d, seed=94, dtype=torch.bfloat16)
    m0, m1 = _models(w, "bf16", layers, d, H, f, N, L0, q, 37)
    m2 = make_model(w, layers=layers, d=d, heads=H, ffn=f, n_ns=N, L0=L0 + 42, q=[v + 42 for v in q])
    m2.set_wait_limit(TEST_WAIT)
    kv0, _ = m0.encode_user(S[:, :L0].contiguous().cuda(), want_s_tail=False)
    kv1, _ = m1.encode_append(kv0, S[:, L0:L0 + 37].contiguous().cuda())
    kv2, out2 = m2.encode_append(kv1, S[:, L0 + 37:].contiguous().cuda())
    m2.poll()
    for u in range(U):
        for l in range(layers):
            K0, V0 = m0.kv_layer(kv0[u], l)
            K2, V2 = m2.kv_layer(kv2[u], l)
            assert torch.equal(K2[:K0.shape[0]], K0) and torch.equal(V2[:V0.shape[0]], V0)
    cfg = oracle_cfg(m2)
    kv_o, s_o = O.encode_user(cfg, w, S)
    errs = {"out_new": O.rel_l2(out2.double().cpu().numpy(), s_o[:, -5:])}
    errs.update(kv_errors(m2, kv2, kv_o, cfg))
    assert_within(errs, TOL["bf16"])
    m2.set_kernel_path(1)
    kv2c, out2c = m2.encode_append(kv1, S[:, L0 + 37:].contiguous().cuda())
    m2.poll()
    assert O.rel_l2(out2c.double().cpu().numpy(), out2.double().cpu().numpy()) < 1e-2


def test_append_rejects_bad_requests_on_host():
    """Host checks before any launch: a delta that would leave the old
    schedule empty, overlapping caches, a short workspace."""
    layers, d, H, f, N = 2, 128, 2, 256, 2
    w = rand_weights(layers, d, f, N, seed=95, dtype=torch.bfloat16)
    m = make_model(w, layers=layers, d=d, heads=H, ffn=f, n_ns=N, L0=100, q=[100, 30])
    from unified_transformer_recommender_onetrans_b200.binding import lib
    kv = m.new_kv_cache(1)
    S_new = torch.zeros(1, 30, d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(S_new)
    ws = torch.empty(m.append_workspace_bytes(1, 30), dtype=torch.uint8, device="cuda")
    p = lambda t: t.data_ptr()  # noqa: E731
    # q[last] = 30 <= delta = 30: no old schedule
    assert lib().ot_encode_append(m.handle, p(kv), 1, p(S_new), 30, p(kv) + kv.numel() * 2 + 4096,
                                  p(out), p(ws), ws.numel(), None) == 2
    # the grown cache overlapping the old one
    assert lib().ot_encode_append(m.handle, p(kv), 1, p(S_new[:, :10]), 10, p(kv), p(out), p(ws),
                                  ws.numel(), None) == 1
    # workspace too small
    kv2 = m.new_kv_cache(1)
    assert lib().ot_encode_append(m.handle, p(kv), 1, p(S_new[:, :10]), 10, p(kv2), p(out), p(ws),
                                  16, None) == 6
    m.poll()
