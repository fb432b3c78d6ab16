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
        total = bench.reduce_max(per_rank_ms)
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
    assert bench.reduce_max(3.5) == 3.5
    assert bench.whole_job_value(1, 1024, 10, 2.0) == pytest.approx(1024 * 10 / 0.002)


# A wrapper that runs bench.py's own entry point with the per-rank GPU
# measurement replaced by a CPU stub (three steps: rank 0 takes 5, 25 and
# 5 ms, rank 1 15 ms each), so the launcher, the process group, the
# max-over-ranks reduction and the JSON line are exercised on CPU ranks.
_STUB = """
import sys
sys.path.insert(0, {root!r})
import bench
import kin_inputs as ki


def fake_measure(args, rank, world, local):
    import torch.distributed as dist
    w0 = ki.WORKLOADS[args.workload]
    w = bench.shard_workload(w0, rank)
    lens, _, _ = ki.case_meta(w)
    dist.barrier()
    return bench.RankRecord(
        w0=w0, w=w, k=w0.k, lens_final=lens, per_step=[5.0, 25.0, 5.0] if rank == 0 else [15.0] * 3,
        parts=[("select", 269e6, "kin_select.cu"), ("attn", 538e6, "kin_attn.cu")],
        part_ms={{"select": [0.04 + 0.01 * rank], "attn": [0.09]}}, upd_ms=[],
        e2e_ms=[12.0 + rank] * args.steps, e2e={{"mode": "stub", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}},
        clocks={{"sm_mhz": 1900 + rank, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"] if rank else [],
                 "samples": 1}},
        wall=0.1, status=0, launches_per_step=3, kv_layout="stub")


bench.measure_rank = fake_measure
sys.exit(bench.main())
"""


def _stub_bench(tmp_path, args, env_extra=None):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "bench_stub.py"
    script.write_text(_STUB.format(root=root))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                          "MASTER_PORT")}
    env.update(env_extra or {})
    env["CUDA_VISIBLE_DEVICES"] = ""
    return subprocess.run([sys.executable, str(script), *args], capture_output=True, text=True, timeout=300,
                          env=env)


def test_bench_gpus_flag_launches_ranks_and_reports_the_slowest(tmp_path):
    r = _stub_bench(tmp_path, ["--gpus", "2", "--steps", "3", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    import json
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["config"]["global_batch"] == 64 and d["config"]["parallelism"] == "dp2"
    assert d["ms_per_step"] == pytest.approx(15.0)                       # the slower rank's time
    # percentiles of each step's max over ranks: 15, 25, 15 ms
    assert d["step_us"] == pytest.approx({"p10": 15e3, "p50": 15e3, "p90": 23e3})
    assert d["value"] == pytest.approx(2 * 32 * 32 * 3 / 0.045)          # both ranks' heads / max time
    assert d["e2e"]["value"] == pytest.approx(2 * 32 * 32 * 3 / 0.039)
    assert d["kernel_ms"]["select"] == pytest.approx(0.05)              # max over ranks
    assert len(d["clocks"]["per_rank"]) == 2 and d["clocks"]["reasons"] == ["sw_power_cap"]
    assert d["scaling"] == "weak" and "cpu_baseline" not in d


def test_bench_gpus_flag_must_agree_with_the_launcher(tmp_path):
    r = _stub_bench(tmp_path, ["--gpus", "2", "--steps", "1", "--warmup", "3"], {"WORLD_SIZE": "1"})
    assert r.returncode == 2 and "disagrees" in r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]
