"""The eFLOPs cost model ("Kinetics: Rethinking Test-Time Scaling Law",
response Q3): T = A/C + M/B, eFLOPs = A + (C/B) M, with A and M counted from
the method's definition; M agrees with the benchmark's independent count of
algorithmic bytes."""
import math

import numpy as np
import pytest

import bench
import kin_inputs as ki
from block_top_sparse_kin_b200 import eflops as ef


def test_time_is_compute_plus_memory():
    c = ef.Cost(3.0e12, 7.0e9)
    r = ef.eflops(c, 2.0e15, 8.0e12)
    assert math.isclose(r["t_pred_us"], (3.0e12 / 2.0e15 + 7.0e9 / 8.0e12) * 1e6, rel_tol=1e-12)
    assert math.isclose(r["eflops"], 3.0e12 + 250.0 * 7.0e9, rel_tol=1e-12)
    assert math.isclose(r["t_pred_us"], r["t_compute_us"] + r["t_memory_us"], rel_tol=1e-12)


@pytest.mark.parametrize("name", sorted(n for n in ki.WORKLOADS))
def test_bytes_match_the_benchmark_count(name):
    w = ki.WORKLOADS[name]
    lens, _, _ = ki.case_meta(w)
    parts = ef.step_costs(w.B, w.Hkv, w.Hq, w.D, w.bs, lens, w.k, w.n_append)
    sel_b, attn_b = bench.algorithmic_bytes(w, w.k, lens)
    assert parts["select"].bytes == sel_b
    assert parts["attn"].bytes == attn_b


def test_dense_budget_counts_every_token_and_no_scoring():
    lens = np.array([100, 37])
    parts = ef.step_costs(2, 2, 8, 128, 16, lens, 64, 0)   # nb = 7, 3 <= k
    assert parts["select"].flops == 0
    assert parts["attn"].flops == 4 * 128 * 4 * 2 * (100 + 37)   # 4 D FLOPs x g x Hkv x tokens


def test_sparse_step_is_memory_bound_on_b200():
    """The pages' point: KV memory access dominates decode.  With the
    measured B200 peaks the step's memory time exceeds its compute time by
    far at every workload."""
    for name, w in ki.WORKLOADS.items():
        lens, _, _ = ki.case_meta(w)
        tot = sum(ef.step_costs(w.B, w.Hkv, w.Hq, w.D, w.bs, lens, w.k, w.n_append).values(), ef.Cost(0, 0))
        r = ef.eflops(tot, 1638.7e12, 6555.2e9)
        assert r["t_memory_us"] > 20 * r["t_compute_us"], name


def test_append_adds_the_touched_blocks():
    lens = np.array([33])      # 1 appended token opens block 2 of a bs-16 sequence
    p = ef.step_costs(1, 1, 1, 128, 16, lens, 2, n_append=1)["update"]
    assert p.flops == 1 * 128  # one valid row in the touched block
    assert p.bytes == 128 * 2 * 4 + 128 * 4
