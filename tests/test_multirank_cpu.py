"""Multi-rank host logic of the benchmark on CPU (gloo, 2 ranks): every rank
decodes its own batch of the same shape (weak scaling, no data-path
collective), and the reported time is the slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import kin_inputs as ki


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.shard_workload(ki.WORKLOADS["qwen3_8b_32k"], rank)
        per_rank_ms = 10.0 + 5.0 * rank          # rank 1 is the slower one
        total = bench.reduce_max(per_rank_ms, "cpu")
        value = bench.whole_job_value(world, w.B * w.Hq, 20, total)
        # a shard's inputs are its own: the first rows of K differ across ranks
        lens, _, hh = ki.case_meta(w)
        k0, _ = ki.pair_rows(w, hh, 0, 0, 16)
        gathered = [None] * world
        dist.all_gather_object(gathered, (w.seed, w.B, w.Hq, total, value, k0.tobytes()))
        q.put((rank, gathered))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_weak_scaling_shards_and_max_over_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    g = results[0]
    assert g == results[1]
    seeds = [x[0] for x in g]
    assert len(set(seeds)) == world                          # independent shards
    assert len(set((x[1], x[2]) for x in g)) == 1            # same per-rank shape
    assert all(x[3] == 15.0 for x in g)                      # max over ranks
    assert g[0][4] == pytest.approx(world * 32 * 32 * 20 / 0.015)
    assert g[0][5] != g[1][5]                                # different data per rank


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.whole_job_value(1, 1024, 10, 2.0) == pytest.approx(1024 * 10 / 0.002)
