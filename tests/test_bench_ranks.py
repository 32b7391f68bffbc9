"""The multi-rank host logic of bench.py, as two gloo ranks on the CPU.

Tokens are independent in the layer (papernotes 整体框架: the lookup and the
mixing act per token), so a batch shards over ranks with no collective on
the data path: every rank holds the same tables and runs its own batch, and
the only cross-rank step is the reduction of the step time (max over ranks)
that turns into whole-job throughput.
"""
import dataclasses
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2
TOKENS = 96


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from static_token_routed_b200 import workloads as wl
        base = wl.with_tokens(wl.WORKLOADS["small_bf16"], TOKENS)
        w = bench.rank_workload(base, rank)
        b = wl.make_batch(w)
        # a step time that differs per rank: the job is as fast as its slowest rank
        ms_max = bench.max_over_ranks(1.5 + rank, dist, "cpu")
        value = bench.job_throughput(w.n_tokens, WORLD, ms_max)
        ids = [torch.empty(TOKENS, dtype=torch.int32) for _ in range(WORLD)]
        dist.all_gather(ids, b.ids.to(torch.int32))
        xs = [torch.empty(TOKENS, w.d_in) for _ in range(WORLD)]
        dist.all_gather(xs, b.x.float())
        same_tables = dataclasses.replace(w, batch_seed=0) == dataclasses.replace(base,
                                                                                  batch_seed=0)
        out[rank] = {"ms_max": ms_max, "value": value, "same_tables": same_tables,
                     "ids": [t.tolist() for t in ids],
                     "x_equal": bool(torch.equal(xs[0], xs[1])),
                     "in_range": bool((b.ids >= 0).all() and (b.ids < w.vocab).all())}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_batches_and_reduce_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(_free_port(), out), nprocs=WORLD, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        # max over ranks, seen identically by every rank
        assert res[r]["ms_max"] == pytest.approx(2.5)
        # whole-job throughput: all ranks' tokens over the slowest rank's time
        assert res[r]["value"] == pytest.approx(WORLD * TOKENS / 2.5e-3)
        assert res[r]["same_tables"] and res[r]["in_range"]
    # both ranks gathered the same two batches, and the batches differ
    assert res[0]["ids"] == res[1]["ids"]
    assert res[0]["ids"][0] != res[0]["ids"][1]
    assert not res[0]["x_equal"]


def test_rank_zero_runs_the_unsharded_workload():
    sys.path.insert(0, ROOT)
    import bench
    from static_token_routed_b200 import workloads as wl
    base = wl.WORKLOADS["paper_shaped"]
    assert bench.rank_workload(base, 0) is base
    w1 = bench.rank_workload(base, 1)
    assert w1.n_tokens == base.n_tokens and w1.batch_seed != base.batch_seed
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
