"""Host logic of the N > 1 bench path, run as two gloo ranks on the CPU.

The forward shards by user with no data-path collective: each rank takes a
disjoint block of users, generates exactly those users' inputs, and the step
time of the job is the slowest rank's (one MAX all-reduce, same order on every
rank)."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, users_per_rank, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        wl = WORKLOADS["tiny_fp32"].with_(users=users_per_rank)
        shard = bench.user_shard(world, rank, users_per_rank)
        w = gen_weights(wl)
        S = gen_s_tokens(wl, users=shard, weights=w)
        x = gen_auto_split_features(wl, users=shard)
        # the slowest rank sets the step time
        t = bench.max_over_ranks(1.0 + 10.0 * rank, world, dist, torch.device("cpu"))
        shards = [None] * world
        dist.all_gather_object(shards, list(shard))
        torch.save({"S": S, "x": x, "t": t, "shards": shards},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_users_and_take_max_time(tmp_path):
    world, per = 2, 3
    mp.start_processes(_rank_main, args=(world, _free_port(), per, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sys.path.insert(0, ROOT)
    from synth import WORKLOADS, gen_auto_split_features, gen_s_tokens, gen_weights

    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    # disjoint blocks covering users 0 .. world*per - 1, seen identically by all ranks
    assert res[0]["shards"] == res[1]["shards"] == [[0, 1, 2], [3, 4, 5]]
    # both ranks report the slowest rank's time
    assert res[0]["t"] == res[1]["t"] == 11.0
    # each rank's inputs are exactly its slice of one big batch
    wl = WORKLOADS["tiny_fp32"].with_(users=world * per)
    w = gen_weights(wl)
    S_all = gen_s_tokens(wl, weights=w)
    x_all = gen_auto_split_features(wl)
    for r in range(world):
        assert torch.equal(res[r]["S"], S_all[r * per:(r + 1) * per])
        assert torch.equal(res[r]["x"], x_all[r * per:(r + 1) * per])
    assert not torch.equal(res[0]["S"], res[1]["S"])


def test_user_shard_rejects_bad_rank():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(ValueError):
        bench.user_shard(2, 2, 4)
    assert list(bench.user_shard(1, 0, 4)) == [0, 1, 2, 3]
