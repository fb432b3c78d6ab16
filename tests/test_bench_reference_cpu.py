"""The benchmark's reference arm on the CPU: it times the oracle as it stands
on the host cores and prints one JSON line with the contract's keys; its
step is one pass over the sampled pairs, whose time fits inside the run;
under a multi-rank launch only rank 0 works and prints."""
import json
import pytest
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *extra):
    env = dict(os.environ, **env_extra)
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "1",
           "--ref-pairs", "2", *extra]
    return subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, check=True).stdout


def test_reference_arm_prints_the_contract_line():
    lines = [l for l in _run({}).splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "query-heads/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 1
    assert d["config"]["workload"] == "qwen3_8b_32k"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "2 of 256" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "query-heads/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    # a step is one pass over the sampled pairs (2 pairs x 4 query heads), and
    # its time follows from the rate; the claimed time fits inside the run
    assert "2 sampled" in d["step"]
    import bench
    assert d["config"] == bench.workload_config(bench.ki.WORKLOADS["qwen3_8b_32k"], 256, 1, means="dual")
    assert abs(d["ms_per_step"] - 2 * 4 / d["value"] * 1e3) < 1e-6 * d["ms_per_step"]
    assert d["steps"] * d["ms_per_step"] / 1e3 <= d["wall_s"]
    p = d["step_us"]
    assert 0 < p["p10"] <= p["p50"] <= p["p90"] <= d["wall_s"] * 1e6


def test_reference_arm_is_silent_on_other_ranks():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}, "--gpus", "2").strip() == ""


def test_default_sample_keeps_every_host_thread_busy():
    import bench
    assert bench.sample_pairs_default() >= 2 * (os.cpu_count() or 1)
    assert bench.sample_pairs_default() >= 32


def test_traffic_lookup_is_keyed_by_means_kind_and_layout():
    """A captured traffic figure is reported only for the variant it was
    captured on: the select's bytes depend on the block-means kind, and a
    paged or shared-prefix run has no capture of its own."""
    import argparse
    import bench
    base = dict(means_fp32=False, means_bf16=False, paged=False, shared_prefix=1)
    ns = lambda **kw: argparse.Namespace(**{**base, **kw})
    assert bench.traffic_key("kin_select.cu", ns()) == "kin_select.cu@dual"
    assert bench.traffic_key("kin_select.cu", ns(means_fp32=True)) == "kin_select.cu@fp32"
    assert bench.traffic_key("kin_attn.cu", ns()) == "kin_attn.cu"
    assert bench.traffic_key("kin_attn.cu", ns(paged=True)) == "kin_attn.cu@paged"
    assert bench.traffic_key("kin_attn.cu", ns(shared_prefix=4)) == "kin_attn.cu@paged"
    # every line of the table parses, and a line is read only under its own key
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows and all(len(r) == 5 for r in rows)
    for key, wl, k, digest, nbytes in rows:
        if digest == bench.kernel_source_digest(key.split("@")[0]):
            assert bench.profiled_traffic(key, wl, int(k)) == int(float(nbytes))
            assert bench.profiled_traffic(key + "@paged", wl, int(k)) is None


def test_means_kind_follows_the_flags():
    import argparse
    import bench
    base = dict(means_fp32=False, means_bf16=False, means_dual=False, shared_prefix=1)
    ns = lambda **kw: argparse.Namespace(**{**base, **kw})
    assert bench.means_kind(ns()) == "dual"
    assert bench.means_kind(ns(shared_prefix=8)) == "fp32"          # per-page means: fp32 unless asked
    assert bench.means_kind(ns(shared_prefix=8, means_dual=True)) == "dual"
    assert bench.means_kind(ns(means_fp32=True)) == "fp32"
    assert bench.means_kind(ns(means_bf16=True)) == "bf16"
    with pytest.raises(SystemExit):
        bench.means_kind(ns(means_fp32=True, means_dual=True))
