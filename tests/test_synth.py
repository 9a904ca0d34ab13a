"""Workload generators: shapes, [SEP] placement, subset determinism, Zipf ids,
and the parameter-count consistency with the pages' OneTransS / OneTransL table."""

import torch

from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights, gen_zipf_ids
from synth.workloads import _interleave_order


def test_concat_order_places_sep_between_sequences():
    wl = WORKLOADS["onetrans_s_full"]
    order = _interleave_order(wl, None)
    assert len(order) == 1190
    assert order[600] == ("sep", 0) and order[1001] == ("sep", 1)
    assert sum(1 for a, _ in order if a == "sep") == 2


def test_interleave_order_is_time_merged_with_three_seps():
    wl = WORKLOADS["onetrans_l_full"]
    g = torch.Generator().manual_seed(0)
    order = _interleave_order(wl, g)
    assert len(order) == 1500
    seps = [i for i, (a, _) in enumerate(order) if a == "sep"]
    assert len(seps) == 3
    # each sequence's events keep their own order
    for k in range(4):
        idx = [i for a, i in order if a == k]
        assert idx == sorted(idx) and len(idx) == wl.seq_lens[k]


def test_subset_generation_is_consistent():
    wl = WORKLOADS["onetrans_s_full"].with_(users=4, L0=1190)
    w = gen_weights(wl.with_(layers=1))
    full = gen_s_tokens(wl, weights=w)
    sub = gen_s_tokens(wl, users=[2], weights=w)
    assert torch.equal(full[2:3], sub)
    x = gen_auto_split_features(wl.with_(cands=6))
    xs = gen_auto_split_features(wl.with_(cands=6), users=[1], cands=[4, 5])
    assert torch.equal(x[1:2, 4:6], xs)


def test_zipf_ids_in_range_and_skewed():
    wl = WORKLOADS["long_fp8"]
    ids = gen_zipf_ids(wl, users=[0, 1], rows=1 << 12)
    assert ids.shape == (2, wl.L0) and ids.min() >= 0 and ids.max() < (1 << 12)
    counts = torch.bincount(ids.flatten(), minlength=1 << 12).sort(descending=True).values
    assert counts[0] > 20 * counts[100]


def _params(wl):
    d, f, N, L = wl.d, wl.ffn, wl.n_ns, wl.layers
    per_set = 3 * d * d + d * d + 2 * d * f + 2 * d
    return L * per_set * (1 + N) + N * d * wl.F


def test_param_counts_match_pages_table():
    """Private QKV/O/FFN per NS position per layer reproduces the printed
    sizes (OneTrans summary page table: OneTransS 91M, OneTransL 330M) to
    within 10%."""
    s = _params(WORKLOADS["onetrans_s_full"])
    l = _params(WORKLOADS["onetrans_l_full"])
    assert abs(s / 91e6 - 1) < 0.10, s
    assert abs(l / 330e6 - 1) < 0.11, l
