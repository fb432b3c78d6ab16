"""bf16 block means (the extended calls): each mean is the fp32 mean rounded
to bf16, bit for bit; the select over them matches the oracle scoring its
own bf16-rounded means (within the near-tie band); the update refreshes a
block exactly as a fresh build does; the paged layout gives the contiguous
results; and the 32K workload at full size passes on sampled pairs."""
import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
from kin_testlib import D, GpuResult, all_pairs, check_pair, check_pairs, make_device_case, to_pages

pytestmark = pytest.mark.gpu
W = ki.Workload


def step_bf16(dc, k, pages=None):
    """Build (+ append) bf16 means, select over them, attend."""
    w = dc.w
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    means = torch.full(dc.means.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    seq = dc.seq_lens.clone()
    k_rows, v_rows, table = (dc.k_cache, dc.v_cache, None) if pages is None else (pages.k, pages.v, pages.table)
    kin.kin_block_means_build_ex(dc.dims, k_rows, seq, means, block_table=table, dev_status=st)
    if w.n_append:
        kin.kin_block_means_update_ex(dc.dims, k_rows, v_rows, means, seq, dc.k_new, dc.v_new, w.n_append,
                                      block_table=table, dev_status=st)
    ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    kin.kin_block_topk_select_ex(dc.dims, dc.q, means, seq, k, sel, cnt, ws, st)
    if pages is None:
        kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, seq, sel, cnt, k, 0.0, out, lse, ws, st)
    else:
        kin.kin_sparse_decode_attn_paged(dc.dims, dc.q, pages.k, pages.v, pages.table, seq, sel, cnt, k, 0.0, out,
                                         lse, ws, st)
    torch.cuda.synchronize()
    return means, seq, GpuResult(sel.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy(),
                                 lse.cpu().numpy(), int(st.item()))


CASES = [
    W("bf16_g4_bs16", 3, 2, 8, D, 16, 500, 1000, 12, 80, Lcap=1024),
    W("bf16_g1_bs32", 2, 2, 2, D, 32, 40, 600, 5, 81, Lcap=640),
    W("bf16_g8_bs64", 2, 1, 8, D, 64, 200, 1000, 4, 82, Lcap=1024),
    W("bf16_append_9", 2, 2, 4, D, 16, 0, 0, 6, 83, Lcap=256, n_append=9, lens=(120, 60)),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_bf16_means_step_against_fp32_means_and_oracle(w):
    dc = make_device_case(w)
    seq0 = dc.seq_lens.clone()
    means, seq, gr = step_bf16(dc, w.k)
    assert gr.status == 0
    # the fp32 means of the default calls, rounded to bf16 by torch, bit for bit
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m32 = torch.zeros(dc.means.shape, dtype=torch.float32, device="cuda")
    kin.kin_block_means_build(dc.dims, dc.k_cache, seq0, m32, st)
    if w.n_append:
        kin.kin_block_means_update(dc.dims, dc.k_cache.clone(), dc.v_cache.clone(), m32, seq0, dc.k_new, dc.v_new,
                                   w.n_append, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.equal(seq0, seq)
    for b in range(w.B):
        nb = -(-int(dc.lens_final[b]) // w.bs)
        assert torch.equal(means[b, :, :nb], m32[b, :, :nb].to(torch.bfloat16))
    gm = means.float().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            check_pair(dc, gr, b, h, w.k, gpu_means=gm, bf16_means=True)


def test_bf16_means_paged_equals_contiguous():
    w = CASES[3]
    dc = make_device_case(w)
    m_c, _, g_c = step_bf16(dc, w.k)
    dc2 = make_device_case(w)
    m_p, _, g_p = step_bf16(dc2, w.k, pages=to_pages(dc2, seed=4))
    assert g_c.status == 0 and g_p.status == 0
    assert torch.equal(torch.nan_to_num(m_c.float()), torch.nan_to_num(m_p.float()))
    assert np.array_equal(g_c.sel, g_p.sel) and np.array_equal(g_c.out, g_p.out)


def test_bf16_means_32k_workload_every_pair():
    w = ki.WORKLOADS["qwen3_8b_32k"]
    dc = make_device_case(w)
    means, _, gr = step_bf16(dc, w.k)
    assert gr.status == 0
    gm = means.float().cpu().numpy()
    check_pairs(dc, [(w.k, gr)], all_pairs(w), gpu_means=gm, bf16_means=True)
