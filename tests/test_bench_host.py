"""Host-side arithmetic of bench.py that the reported numbers rest on."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.mark.parametrize("name,per_user_gflop", [
    # whole-block FLOPs per user at C = 1 as the workload tables give them
    # (OneTransS 8.41, OneTransL 29.79 GFLOP per user, Auto-Split included)
    ("onetrans_s_full", 8.41),
    ("onetrans_l_full", 29.79),
])
def test_forward_flops_match_the_workload_tables(name, per_user_gflop):
    import bench
    from synth import WORKLOADS
    import unified_transformer_recommender_onetrans_b200 as ot
    wl = WORKLOADS[name]
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    total, attn = bench.forward_flops(wl, q, 4, 1)
    auto_split = 2.0 * wl.F * wl.n_ns * wl.d
    got = total / 4 + auto_split
    assert abs(got / 1e9 - per_user_gflop) < 0.005 * per_user_gflop, got
    assert 0 < attn < total


def test_forward_flops_attention_share_scales_with_candidates():
    import bench
    from synth import WORKLOADS
    import unified_transformer_recommender_onetrans_b200 as ot
    wl = WORKLOADS["onetrans_s_full"]
    q = ot.pyramid_schedule(wl.L0, wl.q_end, wl.layers)
    t1, a1 = bench.forward_flops(wl, q, 2, 1)
    t3, a3 = bench.forward_flops(wl, q, 2, 3)
    # the NS side (every term that grows with C) is linear in C
    ns1 = t1 - bench.forward_flops(wl, q, 2, 0)[0]
    ns3 = t3 - bench.forward_flops(wl, q, 2, 0)[0]
    assert abs(ns3 - 3 * ns1) < 1e-6 * ns3
    assert a3 > a1


def test_captured_traffic_is_tied_to_the_kernel_source():
    import hashlib
    import bench
    for kind, (src, sha, nbytes, launches) in bench.CAPTURED_TRAFFIC.items():
        path = os.path.join(ROOT, "unified_transformer_recommender_onetrans_b200", "csrc", src)
        assert os.path.exists(path), src
        assert nbytes > 0 and launches > 0
        with open(path, "rb") as fh:
            current = hashlib.sha256(fh.read()).hexdigest() == sha
        value, note = bench.captured_traffic(kind)
        # reported only while the captured source is the one in the tree
        assert (value == nbytes) == current, (kind, note)
    assert bench.captured_traffic("no_such_kernel")[0] is None


def test_metric_name_is_shared_by_both_arms():
    import bench
    from synth import WORKLOADS
    wl = WORKLOADS["onetrans_s_full"]
    assert bench.metric_name(wl) == "S-tokens/s (onetrans_s_full full forward)"
