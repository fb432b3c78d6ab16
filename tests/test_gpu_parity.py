"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded bf16 inputs.  Small shapes are compared on every (batch, kv
head); the five decode workloads run at full size in the same launch
configuration the benchmark times, and every (batch, kv head) of each is
compared with the oracle (every budget of the sweep).  Tolerances: see
kin_testlib.
"""
import math

import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import D, all_pairs, check_pair, check_pairs, gpu_step, make_device_case

pytestmark = pytest.mark.gpu

W = ki.Workload

SMALL = [
    # name, B, Hkv, Hq, D, bs, Lmin, Lmax, k, seed, (extra)
    W("ragged_g4_bs16", 2, 2, 8, D, 16, 700, 1000, 16, 10, Lcap=1024),
    W("ragged_g1_bs32", 3, 1, 1, D, 32, 33, 333, 5, 11, Lcap=400),
    W("ragged_g5_bs64", 2, 2, 10, D, 64, 100, 900, 6, 12, Lcap=960),
    W("len1_g8", 1, 3, 24, D, 16, 1, 1, 4, 13, Lcap=16),
    W("bs128_g8", 2, 1, 8, D, 128, 129, 1000, 3, 14, Lcap=1024),
    W("g2_many_chunks", 4, 2, 4, D, 16, 2000, 4000, 100, 15, Lcap=4096),
    # nb = k-1, k, k+1 (k = 8, bs 16) and partial / full last blocks
    W("nb_edges", 6, 1, 4, D, 16, 0, 0, 8, 16, Lcap=160, lens=(112, 113, 128, 129, 144, 1)),
    W("bs32_partial_tiles", 4, 2, 6, D, 32, 0, 0, 4, 17, Lcap=300, lens=(33, 47, 48, 290)),
    W("append_7", 2, 2, 8, D, 16, 0, 0, 6, 18, Lcap=200, n_append=7, lens=(100, 37)),
    W("append_1_full", 2, 1, 4, D, 32, 0, 0, 3, 19, Lcap=128, n_append=1, lens=(128, 65)),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_shapes_every_pair(w):
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    means = dc.means.cpu().numpy()
    assert np.array_equal(dc.seq_lens.cpu().numpy(), dc.lens_final)
    for b in range(w.B):
        for h in range(w.Hkv):
            check_pair(dc, gr, b, h, w.k, gpu_means=means)


def test_all_equal_scores_take_lowest_indices():
    """q = 0 makes every block score 0: the tie rule keeps 0..k-2 and the last
    block, and the output is the plain mean of V over those tokens."""
    w = W("zeros", 2, 2, 8, D, 16, 0, 0, 6, 20, Lcap=512, lens=(500, 257))
    dc = make_device_case(w)
    dc.q.zero_()
    dc.q_host[:] = 0
    gr = gpu_step(dc, w.k)
    for b in range(w.B):
        nb = -(-int(dc.lens_final[b]) // 16)
        for h in range(w.Hkv):
            assert list(gr.sel[b, h]) == [0, 1, 2, 3, 4, nb - 1]
            check_pair(dc, gr, b, h, w.k)


def test_update_matches_fresh_build_bitwise():
    """Means refreshed by an append equal means built from scratch on the
    updated cache, bit for bit (same fp32 token-order sums)."""
    w = W("upd", 3, 2, 4, D, 32, 0, 0, 4, 21, Lcap=256, n_append=40, lens=(200, 41, 256))
    dc = make_device_case(w)
    gpu_step(dc, w.k)
    upd = dc.means.clone()
    fresh = torch.full_like(dc.means, float("nan"))
    kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, fresh)
    torch.cuda.synchronize()
    for b in range(w.B):
        nb = -(-int(dc.lens_final[b]) // w.bs)
        assert torch.equal(upd[b, :, :nb], fresh[b, :, :nb])


def test_workspace_reuse_is_deterministic():
    w = W("reuse", 4, 2, 8, D, 16, 3000, 4000, 32, 22, Lcap=4096)
    dc = make_device_case(w)
    ws = kin.alloc_workspace(dc.dims, w.k)
    a = gpu_step(dc, w.k, ws=ws)
    b = gpu_step(dc, w.k, ws=ws, build_means=False)
    assert np.array_equal(a.sel, b.sel) and np.array_equal(a.out, b.out) and np.array_equal(a.lse, b.lse)
    # the attention's completion counters (the first 256-byte aligned region) are back at zero
    n = (w.B * w.Hkv * 4 + 255) // 256 * 256
    assert torch.count_nonzero(ws[:n]) == 0


def test_one_workspace_serves_every_budget_in_turn():
    """One zeroed workspace of the largest size the budgets need, used by a
    select and an attention per budget back to back on one stream (no
    re-zeroing, one synchronize at the end; the budgets split the pairs into
    different chunk counts and the last one is dense): every budget's
    results equal a fresh workspace's bit for bit, and the completion
    counters end at zero."""
    w = W("ws_budgets", 4, 2, 8, D, 16, 2000, 4000, 8, 26, Lcap=4096)
    dc = make_device_case(w)
    ks = (2, 8, 31, 73, 200, 256)
    fresh = [gpu_step(dc, k, build_means=i == 0) for i, k in enumerate(ks)]
    ws = torch.zeros(max(kin.kin_workspace_bytes(dc.dims, k) for k in ks), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    runs = []
    for k in ks:
        sel = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
        cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
        out = torch.empty((w.B, w.Hq, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, k, sel, cnt, ws, st)
        kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, k, 0.0,
                                   out, lse, ws, st)
        runs.append((sel, cnt, out, lse))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for k, f, (sel, cnt, out, lse) in zip(ks, fresh, runs):
        assert np.array_equal(sel.cpu().numpy(), f.sel) and np.array_equal(cnt.cpu().numpy(), f.cnt), k
        assert np.array_equal(out.float().cpu().numpy(), f.out) and np.array_equal(lse.cpu().numpy(), f.lse), k
    n = (w.B * w.Hkv * 4 + 255) // 256 * 256
    assert torch.count_nonzero(ws[:n]) == 0


def test_bad_device_lengths_are_flagged_not_fatal():
    w = W("bad", 3, 1, 4, D, 16, 0, 0, 4, 23, Lcap=128, lens=(100, 50, 80))
    dc = make_device_case(w)
    gr0 = gpu_step(dc, w.k)
    assert gr0.status == 0
    dc.seq_lens.copy_(torch.tensor([100, 129, 0], dtype=torch.int32))
    gr = gpu_step(dc, w.k, build_means=False)
    assert gr.status == 5
    assert gr.cnt[1, 0] == 0 and gr.cnt[2, 0] == 0
    assert np.all(gr.sel[1:] == -1)
    assert np.all(gr.out[1:] == 0) and np.all(np.isneginf(gr.lse[1:]))
    assert np.array_equal(gr.out[0], gr0.out[0])


def test_budget_covering_every_block_with_a_bad_length():
    """k >= ceil(Lcap / bs): the select writes every block of each sequence
    without scoring (no sequence can hold more blocks than the budget); a
    length outside [1, Lcap] gets sel_cnt 0, a row of -1 and the status;
    the outputs of the good sequences equal dense attention (oracle)."""
    w = W("dense_only", 3, 2, 4, D, 16, 0, 0, 8, 25, Lcap=100, lens=(100, 37, 1))
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    for b in range(w.B):
        nb = -(-int(dc.lens_final[b]) // w.bs)
        for h in range(w.Hkv):
            assert list(gr.sel[b, h]) == list(range(nb)) + [-1] * (w.k - nb)
            check_pair(dc, gr, b, h, w.k)
    dc.seq_lens.copy_(torch.tensor([100, 0, 1], dtype=torch.int32))
    bad = gpu_step(dc, w.k, build_means=False)
    assert bad.status == 5
    assert np.all(bad.cnt[1] == 0) and np.all(bad.sel[1] == -1)
    assert np.array_equal(bad.sel[[0, 2]], gr.sel[[0, 2]]) and np.array_equal(bad.out[0], gr.out[0])


def test_bad_block_index_is_flagged_and_skipped():
    w = W("badidx", 1, 1, 4, D, 16, 0, 0, 4, 24, Lcap=256, lens=(200,))
    dc = make_device_case(w)
    gpu_step(dc, w.k)
    sel = torch.tensor([[[0, 3, 99, 12]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[4]], dtype=torch.int32, device="cuda")
    out = torch.empty((1, 4, D), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = kin.alloc_workspace(dc.dims, 4)
    kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, 4, 0.0,
                               out, None, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    K, V = ki.pair_rows(w, dc.hh, 0, 0, 200)
    ref, _ = oracle.attend(dc.q_host[0], K, V, 200, 16, np.array([0, 3, 12]), 1 / math.sqrt(D))
    assert np.abs(out[0].float().cpu().numpy() - ref).max() <= 2e-2


def test_host_validation_errors():
    dims = kin.make_dims(2, 2, 8, D, 16, 256)
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    q = torch.zeros((2, 8, D), dtype=torch.bfloat16, device="cuda")
    means = torch.zeros((2, 2, 16, D), dtype=torch.float32, device="cuda")
    sel = torch.zeros((2, 2, 4), dtype=torch.int32, device="cuda")
    ws = kin.alloc_workspace(dims, 4)
    with pytest.raises(kin.KinError) as e:
        kin.kin_block_topk_select(dims, q, means, t, 1, sel, t, ws)
    assert e.value.status == 1
    with pytest.raises(kin.KinError) as e:
        kin.kin_block_topk_select(dims, q, means, t, 4, sel, t, ws[:64])
    assert e.value.status == 2
    with pytest.raises(kin.KinError) as e:
        kin.kin_block_topk_select(kin.make_dims(2, 2, 8, 64, 16, 256), q, means, t, 4, sel, t, ws)
    assert e.value.status == 1
    with pytest.raises(kin.KinError) as e:
        kin.kin_block_topk_select(kin.make_dims(2, 1, 16, D, 16, 256), q, means, t, 4, sel, t, ws)
    assert e.value.status == 3


def test_binding_refuses_short_or_foreign_tensors():
    """The C ABI receives bare pointers, so the binding checks every tensor
    against the dims before the call: a buffer shorter than the dims imply,
    a host tensor or a non-contiguous view raises ValueError and nothing is
    launched (the outputs keep their contents)."""
    dims = kin.make_dims(2, 2, 8, D, 16, 256)
    lens = torch.full((2,), 200, dtype=torch.int32, device="cuda")
    q = torch.zeros((2, 8, D), dtype=torch.bfloat16, device="cuda")
    means = torch.zeros((2, 2, 16, D), dtype=torch.float32, device="cuda")
    sel = torch.full((2, 2, 4), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((2, 2), -7, dtype=torch.int32, device="cuda")
    ws = kin.alloc_workspace(dims, 4)
    bad = {
        "q": (q[:1], means, sel, cnt, lens),
        "block_means": (q, means[:, :, :15].contiguous(), sel, cnt, lens),
        "sel_idx": (q, means, sel[:, :, :3].contiguous(), cnt, lens),
        "sel_cnt": (q, means, sel, cnt[:1], lens),
        "seq_lens": (q, means, sel, cnt, lens[:1]),
    }
    for name, (qq, mm, ss, cc, ll) in bad.items():
        with pytest.raises(ValueError, match=name):
            kin.kin_block_topk_select(dims, qq, mm, ll, 4, ss, cc, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kin.kin_block_topk_select(dims, q.cpu(), means, lens, 4, sel, cnt, ws)
    with pytest.raises(ValueError, match="contiguous"):
        kin.kin_block_topk_select(dims, q, means, lens, 4, sel.transpose(0, 1), cnt, ws)
    out = torch.zeros((2, 8, D), dtype=torch.bfloat16, device="cuda")
    k_cache = torch.zeros((2, 2, 256, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="v_cache"):
        kin.kin_sparse_decode_attn(dims, q, k_cache, k_cache[:1], lens, sel, cnt, 4, 0.0, out, None, ws)
    with pytest.raises(ValueError, match="lse"):
        kin.kin_sparse_decode_attn(dims, q, k_cache, k_cache, lens, sel, cnt, 4, 0.0, out,
                                   torch.zeros(3, device="cuda"), ws)
    torch.cuda.synchronize()
    assert torch.all(sel == -7) and torch.all(cnt == -7)


# ------------------------------------------------------- full-size workloads
def _full(name, ks=None):
    """A decode workload at full size, in the benchmark's launch shapes:
    properties on every pair, then every pair against the oracle (means,
    selection, outputs and lse) for every budget."""
    w = ki.WORKLOADS[name]
    dc = make_device_case(w)
    ks = ks or (w.k,)
    results = []
    for i, k in enumerate(ks):
        gr = gpu_step(dc, k, build_means=i == 0)
        assert gr.status == 0
        lens = dc.lens_final
        nb = -(-lens // w.bs)
        exp_cnt = np.minimum(nb, k)[:, None].repeat(w.Hkv, 1)
        assert np.array_equal(gr.cnt, exp_cnt)
        assert np.all(gr.sel[:, :, 0] == 0)
        last = gr.sel[np.arange(w.B)[:, None], np.arange(w.Hkv)[None, :], exp_cnt - 1]
        assert np.array_equal(last, (nb - 1)[:, None].repeat(w.Hkv, 1))
        assert np.all(np.isfinite(gr.out)) and np.all(np.isfinite(gr.lse))
        results.append((k, gr))
    means = dc.means.cpu().numpy()
    del dc.k_cache, dc.v_cache
    torch.cuda.empty_cache()
    near = check_pairs(dc, results, all_pairs(w), gpu_means=means)
    print(f"{name}: {w.B * w.Hkv} pairs x {len(ks)} budgets against the oracle, {near} near-tie selections")


def test_workload_tiny():
    _full("tiny")


def test_workload_qwen3_8b_32k():
    _full("qwen3_8b_32k")


def test_workload_qwen3_14b_ragged():
    _full("qwen3_14b_ragged")


def test_workload_qwen3_32b_128k_append():
    _full("qwen3_32b_128k_append")


def test_workload_qwen3_0p6b_sweep():
    _full("qwen3_0p6b_sweep", ks=ki.SWEEP_K)
