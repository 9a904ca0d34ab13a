"""C-ABI checks that need no GPU: the library loads, exports every function
include/onetrans.h declares, and rejects bad arguments on the host before
touching the device."""

import ctypes as C
import os
import re

import pytest

import unified_transformer_recommender_onetrans_b200 as ot
from unified_transformer_recommender_onetrans_b200 import binding as B
from unified_transformer_recommender_onetrans_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return B.lib()


def header_functions():
    txt = open(os.path.join(ROOT, "include", "onetrans.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(ot_[a-z_0-9]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.SIGNATURES), set(names) ^ set(B.SIGNATURES)


def test_status_strings(lib):
    for code in range(11):
        assert lib.ot_status_str(code)
    assert lib.ot_status_str(0) == b"ok"


def _cfg(**kw):
    c = B.OtConfig()
    base = dict(layers=2, d=128, heads=2, ffn=256, n_ns=3, L0=40, F=64, eps=1e-6, dtype=1)
    base.update(kw)
    q = base.pop("q", [40, 10])
    for k, v in base.items():
        setattr(c, k, v)
    for i, v in enumerate(q):
        c.q[i] = v
    return c


def _create(lib, cfg, weights=None):
    w = weights or B.OtWeights(**{n: 16 * (i + 1) for i, n in enumerate(B.WEIGHT_NAMES)})
    h = C.c_void_p()
    return lib.ot_model_create(C.byref(cfg), C.byref(w), C.byref(h))


def test_create_rejects_bad_config_on_host(lib):
    assert lib.ot_model_create(None, None, None) == 1
    assert _create(lib, _cfg(q=[41, 10])) == 2          # q_0 > L0
    assert _create(lib, _cfg(q=[40, 41])) == 2          # q_1 > L_1
    assert _create(lib, _cfg(q=[40, 0])) == 2
    assert _create(lib, _cfg(heads=4)) == 2             # head_dim 32 on the bf16 path
    assert _create(lib, _cfg(d=96, heads=1, q=[40, 10])) == 2
    assert _create(lib, _cfg(dtype=7)) == 3
    assert _create(lib, _cfg(layers=0)) == 1
    w = B.OtWeights(**{n: 16 * (i + 1) for i, n in enumerate(B.WEIGHT_NAMES)})
    w.Wo_s = 18                                          # misaligned
    assert _create(lib, _cfg(), w) == 4
    w.Wo_s = None
    assert _create(lib, _cfg(), w) == 1


def test_calls_reject_null_model(lib):
    assert lib.ot_encode_user(None, None, 1, None, None, None, 0, None) == 1
    assert lib.ot_score_candidates(None, None, 1, None, 1, None, None, 0, None) == 1
    assert lib.ot_full_forward(None, None, None, 1, 1, None, None, None, None, 0, None) == 1
    assert lib.ot_full_forward_host(None, None, None, 1, 1, None, None, None, None, 0, None) == 1
    assert lib.ot_host_workspace_bytes(None, 1, 1) == 0
    assert lib.ot_auto_split(None, None, 1, None, None) == 1
    assert lib.ot_embed_gather(None, 1, 8, None, 1, None, None, None) == 1
    assert lib.ot_embed_gather(16, 1, 12, 16, 1, 16, None, None) == 2
    assert lib.ot_embed_gather(16, 1, 8, 16, 1, 24, None, None) == 4
    assert lib.ot_kv_cache_bytes(None, 1) == 0
    assert lib.ot_encode_append(None, None, 1, None, 1, None, None, None, 0, None) == 1
    assert lib.ot_append_workspace_bytes(None, 1, 1) == 0
    assert lib.ot_set_wait_limit(None, 5) == 1
    assert lib.ot_launch_count(None) == -1


def test_product_pyramid_schedule_matches_golden():
    import json
    gold = json.load(open(os.path.join(ROOT, "tests", "golden", "pyramid_schedules.json")))
    for case in gold["cases"]:
        assert ot.pyramid_schedule(case["L0"], case["q_end"], case["layers"]) == case["q"]
    # ties go to even: L0=10, q_end=1, 3 layers -> 10, 5.5 -> 6? (5.5 ties to 6), 1
    assert ot.pyramid_schedule(10, 1, 3) == [10, 6, 1]
    assert ot.pyramid_schedule(9, 2, 3) == [9, 6, 2]     # 5.5 -> 6
    assert ot.pyramid_schedule(11, 2, 3) == [11, 6, 2]   # 6.5 -> 6


def test_product_path_does_not_import_oracle():
    """The product package never reaches the oracle (no CPU fallback)."""
    pkg = os.path.join(ROOT, "unified_transformer_recommender_onetrans_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.replace("oracle-free", ""), f


def _bw_args(cfg, U=2, Cn=3, misalign=None, ws_bytes=None):
    """ot_full_backward arguments with placeholder (never dereferenced)
    device addresses: the host checks return before any device work."""
    names = list(B.GRAD_NAMES)
    w = B.OtWeights(**{n: 4096 * (i + 1) for i, n in enumerate(names)})
    g = B.OtGrads(**{n: 4096 * (i + 101) for i, n in enumerate(names)})
    if misalign:
        setattr(g, misalign, getattr(g, misalign) + 4)
    nbytes = lib_bw_bytes(cfg, U, Cn) if ws_bytes is None else ws_bytes
    return (C.byref(cfg), C.byref(w), 1 << 20, 2 << 20, U, Cn, 3 << 20, 4 << 20, 0, 0, C.byref(g),
            0, 0, 5 << 20, nbytes, None)


def lib_bw_bytes(cfg, U, Cn):
    return B.lib().ot_backward_workspace_bytes(C.byref(cfg), U, Cn)


def test_backward_host_checks(lib):
    f32 = dict(dtype=0, d=64, heads=2, ffn=96, n_ns=3, L0=40, q=[40, 10])
    cfg = _cfg(**f32)
    ws = lib_bw_bytes(cfg, 2, 3)
    assert ws > 0 and ws % 256 == 0
    # the workspace grows with the batch; C = 0 needs no NS buffers
    assert lib_bw_bytes(cfg, 4, 3) > ws > lib_bw_bytes(cfg, 2, 0) > 0
    assert lib.ot_full_backward(None, None, None, None, 1, 1, None, None, None, None, None, None,
                                None, None, 0, None) == 1
    assert lib.ot_full_backward(*_bw_args(_cfg(**dict(f32, dtype=1)))) == 3          # bf16
    assert lib.ot_full_backward(*_bw_args(_cfg(**dict(f32, full_attn=1)))) == 2     # full: C must be 1
    assert lib_bw_bytes(_cfg(**dict(f32, full_attn=1)), 2, 1) > 0
    assert lib.ot_full_backward(*_bw_args(_cfg(**dict(f32, moe_experts=4, moe_topk=1)))) == 1   # no MoE tensors
    assert lib.ot_full_backward(*_bw_args(_cfg(**dict(f32, q=[41, 10])))) == 2
    assert lib.ot_full_backward(*_bw_args(cfg, misalign="W1_ns")) == 4
    assert lib.ot_full_backward(*_bw_args(cfg, ws_bytes=ws - 1)) == 6
    args = list(_bw_args(cfg))
    args[4] = 0                                                                      # U = 0
    assert lib.ot_full_backward(*args) == 1
    assert lib_bw_bytes(_cfg(**dict(f32, dtype=1)), 2, 3) == 0


def test_backward_launch_count(lib):
    """Kernel launches per call.  Per layer, with candidates: the forward is
    8 launches per side (norm, QKV, attention, O, norm, FFN1, GELU, FFN2),
    6 when only recomputed (no output GEMM; the attention's outputs are kept
    from the checkpointing pass); the backward 10 per side for the FFN and
    O projection, 4 attention kernels, 5 per side for QKV and the first
    norm, 1 residual add.  The top layer is not recomputed."""
    f32 = dict(dtype=0, d=64, heads=2, ffn=96, n_ns=3, L0=40)
    for layers, q in ((1, [40]), (2, [40, 10]), (3, [40, 20, 5])):
        c = _cfg(**dict(f32, layers=layers, q=q))
        assert lib.ot_backward_launches(C.byref(c), 2, 3) == 16 * layers + 12 * (layers - 1) + 35 * layers
        assert lib.ot_backward_launches(C.byref(c), 2, 0) == 8 * layers + 6 * (layers - 1) + 18 * layers
    assert lib.ot_backward_launches(C.byref(_cfg(**dict(f32, dtype=1, layers=1, q=[40]))), 2, 3) == 0


def test_backward_binding_checks_tensor_shapes_on_host():
    """full_backward refuses tensors that do not match an accepted
    configuration before anything reaches the device (CPU tensors here: the
    shape check comes first; a matching set then fails only on the device
    check).  An invalid configuration is left to the library's status."""
    import torch
    import unified_transformer_recommender_onetrans_b200 as ot

    L, d, H, f, N, L0, U, C = 1, 64, 2, 96, 3, 40, 2, 2
    q = [9]
    cfg = ot.make_config(layers=L, d=d, heads=H, ffn=f, n_ns=N, L0=L0, q=q)
    shapes = {"Wqkv_s": (L, 3 * d, d), "Wo_s": (L, d, d), "W1_s": (L, f, d), "W2_s": (L, d, f),
              "g1_s": (L, d), "g2_s": (L, d), "Wqkv_ns": (L, N, 3 * d, d), "Wo_ns": (L, N, d, d),
              "W1_ns": (L, N, f, d), "W2_ns": (L, N, d, f), "g1_ns": (L, N, d), "g2_ns": (L, N, d)}
    w = {k: torch.zeros(s) for k, s in shapes.items()}
    S, ns = torch.zeros(U, L0, d), torch.zeros(U, C, N, d)
    G_s, G_ns = torch.zeros(U, q[-1], d), torch.zeros(U, C, N, d)
    with pytest.raises(ValueError, match="CUDA"):  # every shape right: the device check
        ot.full_backward(cfg, w, S, ns, G_s, G_ns)
    with pytest.raises(ValueError, match="shape"):
        ot.full_backward(cfg, w, torch.zeros(U, L0 + 1, d), ns, G_s, G_ns)
    with pytest.raises(ValueError, match="G_s must have shape"):
        ot.full_backward(cfg, w, S, ns, torch.zeros(U, L0, d), G_ns)
    bad_w = dict(w, W1_ns=torch.zeros(L, N, d, f))  # transposed
    with pytest.raises(ValueError, match="W1_ns"):
        ot.full_backward(cfg, bad_w, S, ns, G_s, G_ns)
    with pytest.raises(ValueError, match="float32"):
        ot.full_backward(cfg, w, S.double(), ns, G_s, G_ns)
    with pytest.raises(ValueError, match="grads"):
        ot.full_backward(cfg, w, S, ns, G_s, G_ns, grads={"Wo_s": torch.zeros(L, d, d + 1)})
