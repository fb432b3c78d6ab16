"""Paged KV cache on the GPU: the same decode step over a shuffled page pool
(the page is one KV block) must give the contiguous cache's results bit for
bit (means, kept blocks, outputs, lse, appended rows), and so the oracle's;
the oracle's own paged definition (a gather through the block table) is
checked against the pool directly.  A page index outside the pool is
flagged and skipped."""
import math

import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import (D, all_pairs, check_pair, check_pairs, gpu_step, gpu_step_paged, make_device_case,
                         to_pages)

pytestmark = pytest.mark.gpu
W = ki.Workload

CASES = [
    W("paged_g4_bs16", 3, 2, 8, D, 16, 300, 1000, 12, 70, Lcap=1024),
    W("paged_g1_bs32", 2, 3, 3, D, 32, 33, 500, 5, 71, Lcap=520),
    W("paged_g8_bs64", 2, 1, 8, D, 64, 100, 900, 4, 72, Lcap=960),
    W("paged_bs128", 2, 2, 4, D, 128, 129, 1000, 3, 73, Lcap=1024),
    W("paged_append_7", 2, 2, 8, D, 16, 0, 0, 6, 74, Lcap=200, n_append=7, lens=(100, 44)),
    W("paged_append_1_new_page", 2, 1, 4, D, 32, 0, 0, 3, 75, Lcap=160, n_append=1, lens=(128, 64)),
    W("paged_dense_and_len1", 3, 1, 4, D, 16, 0, 0, 8, 76, Lcap=160, lens=(112, 1, 129)),
]


def _compare_with_contiguous(w, seed):
    dc = make_device_case(w)
    pg = to_pages(dc, seed=seed)
    seq_p = dc.seq_lens.clone()
    means_p = torch.full_like(dc.means, float("nan"))
    gr = gpu_step(dc, w.k)                      # contiguous: build (+ append), select, attend
    gp = gpu_step_paged(dc, pg, w.k, seq_p, means_p)
    assert gr.status == 0 and gp.status == 0
    assert torch.equal(seq_p, dc.seq_lens)
    for b in range(w.B):
        nb = -(-int(dc.lens_final[b]) // w.bs)
        assert torch.equal(means_p[b, :, :nb], dc.means[b, :, :nb])
    assert np.array_equal(gp.sel, gr.sel) and np.array_equal(gp.cnt, gr.cnt)
    assert np.array_equal(gp.out, gr.out) and np.array_equal(gp.lse, gr.lse)
    return dc, pg, gr


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_paged_step_equals_contiguous_and_oracle(w):
    dc, pg, gr = _compare_with_contiguous(w, seed=w.seed)
    means = dc.means.cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            check_pair(dc, gr, b, h, w.k, gpu_means=means)
    if w.n_append:  # the appended rows landed in the right pages
        kp, vp = pg.k.cpu(), pg.v.cpu()
        for b in range(w.B):
            for t in range(int(dc.lens_pre[b]), int(dc.lens_final[b])):
                page, r = int(pg.table_host[b, t // w.bs]), t % w.bs
                assert torch.equal(kp[page, :, r], dc.k_cache[b, :, t].cpu())
                assert torch.equal(vp[page, :, r], dc.v_cache[b, :, t].cpu())


def test_oracle_gather_reads_the_pool_as_the_kernels_do():
    w = CASES[0]
    dc = make_device_case(w)
    pg = to_pages(dc, seed=5)
    pool = pg.k.cpu().view(torch.int16).numpy().view(np.uint16)
    for b, h in [(0, 0), (2, 1)]:
        L = int(dc.lens_final[b])
        K, _ = ki.pair_rows(w, dc.hh, b, h, L)
        assert np.array_equal(oracle.gather_paged(pool, pg.table_host[b], L, w.bs, h), K)


def test_paged_bad_page_index_is_flagged_and_skipped():
    w = W("paged_bad", 2, 2, 4, D, 16, 0, 0, 6, 77, Lcap=320, lens=(300, 250))
    dc = make_device_case(w)
    pg = to_pages(dc, seed=9)
    seq = dc.seq_lens.clone()
    means = torch.zeros_like(dc.means)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_means_build_paged(dc.dims, pg.k, pg.table, seq, means, st)
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    kin.kin_block_topk_select(dc.dims, dc.q, means, seq, w.k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    kin.kin_sparse_decode_attn_paged(dc.dims, dc.q, pg.k, pg.v, pg.table, seq, sel, cnt, w.k, 0.0, out, lse,
                                     ws, st)
    good = out.clone()
    # sequence 1's first kept block now points past the pool
    table = pg.table.clone()
    table[1, int(sel[1, 0, 0].item())] = pg.num_pages
    kin.kin_sparse_decode_attn_paged(dc.dims, dc.q, pg.k, pg.v, table, seq, sel, cnt, w.k, 0.0, out, lse, ws,
                                     st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    assert torch.equal(out[0], good[0])          # the other sequence is untouched
    assert bool(torch.isfinite(out[1].float()).all())


def test_paged_ragged_workload_full_size():
    """The ragged 64-sequence workload at full size over a shuffled pool:
    bit-identical to the contiguous cache, every pair against the oracle."""
    w = ki.WORKLOADS["qwen3_14b_ragged"]
    dc, pg, gr = _compare_with_contiguous(w, seed=11)
    check_pairs(dc, [(w.k, gr)], all_pairs(w))
