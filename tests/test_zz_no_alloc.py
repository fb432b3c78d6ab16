"""kin_block_topk_select_noalloc: the select for callers that may not
allocate device memory (a runtime that owns a fixed memory plan, a plugin
without allocation rights, a decode loop that must never reach the
allocator).  It must return exactly what the workspace-based
kin_block_topk_select returns, call after call, even though every call
reuses the same scratch array inside the library.  This file sorts last so a
run that stops at the first failure has run every other test first."""
import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
from kin_testlib import D, make_device_case

pytestmark = pytest.mark.gpu


def _reference(dc, k):
    ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.full((dc.w.B, dc.w.Hkv, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((dc.w.B, dc.w.Hkv), -7, dtype=torch.int32, device="cuda")
    kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, k, sel, cnt, ws)
    torch.cuda.synchronize()
    return sel.cpu().numpy(), cnt.cpu().numpy()


def _noalloc(dc, k):
    sel = torch.full((dc.w.B, dc.w.Hkv, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((dc.w.B, dc.w.Hkv), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_topk_select_noalloc(dc.dims, dc.q, dc.means, dc.seq_lens, k, sel, cnt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return sel.cpu().numpy(), cnt.cpu().numpy()


def test_noalloc_select_matches_workspace_select_on_consecutive_calls():
    cases = [
        ki.Workload("noalloc_a", 4, 4, 16, D, 16, 1500, 3000, 24, 31, Lcap=3072),
        ki.Workload("noalloc_b", 3, 2, 10, D, 32, 300, 900, 6, 32, Lcap=960),
    ]
    devs = [make_device_case(w) for w in cases]
    for dc in devs:
        kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, dc.means)
    torch.cuda.synchronize()
    refs = [_reference(dc, dc.w.k) for dc in devs]
    # two calls in a row on the same inputs, then a call on other inputs whose
    # scratch rows overlap the previous call's: indices are integer results,
    # so they must match bit for bit
    for dc, ref in ((devs[0], refs[0]), (devs[0], refs[0]), (devs[1], refs[1])):
        sel, cnt = _noalloc(dc, dc.w.k)
        assert np.array_equal(cnt, ref[1])
        assert np.array_equal(sel, ref[0])


def test_noalloc_select_takes_no_device_memory():
    """After a first call on the device (which looks up the scratch array),
    further calls leave the device's free memory unchanged: the call itself
    allocates nothing.  Outputs are allocated before the measurement."""
    w = ki.Workload("noalloc_mem", 2, 2, 8, D, 16, 900, 2000, 12, 33, Lcap=2048)
    dc = make_device_case(w)
    kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, dc.means)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_topk_select_noalloc(dc.dims, dc.q, dc.means, dc.seq_lens, w.k, sel, cnt, st)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        kin.kin_block_topk_select_noalloc(dc.dims, dc.q, dc.means, dc.seq_lens, w.k, sel, cnt, st)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert int(st.item()) == 0
    assert free1 == free0


def test_noalloc_select_at_its_scratch_capacity():
    """B * Hkv * ceil(Lcap / bs) exactly KIN_NOALLOC_SCRATCH_FLOATS (64 x 8 x
    4096 = 2^21 scores, so the last pair's row ends at the array's end), on
    seeded random means and ragged lengths that include full sequences: the
    same selection as the workspace select, bit for bit.  One block more of
    capacity is refused by the entry point before anything is launched."""
    import ctypes
    B, Hkv, Hq, bs, Lcap, k = 64, 8, 32, 16, 4096 * 16, 300
    assert B * Hkv * (Lcap // bs) == kin.NOALLOC_SCRATCH_FLOATS
    dims = kin.make_dims(B, Hkv, Hq, D, bs, Lcap)
    g = torch.Generator(device="cuda").manual_seed(33)
    means = torch.randn((B, Hkv, Lcap // bs, D), generator=g, device="cuda", dtype=torch.float32)
    q = torch.randn((B, Hq, D), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    lens = torch.randint(1, Lcap + 1, (B,), generator=g, device="cuda", dtype=torch.int32)
    lens[:4] = Lcap
    ws = kin.alloc_workspace(dims, k)
    out = []
    for noalloc in (False, True):
        sel = torch.full((B, Hkv, k), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if noalloc:
            kin.kin_block_topk_select_noalloc(dims, q, means, lens, k, sel, cnt, st)
        else:
            kin.kin_block_topk_select(dims, q, means, lens, k, sel, cnt, ws, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        out.append((sel.cpu().numpy(), cnt.cpu().numpy()))
    assert np.array_equal(out[0][1], out[1][1]) and np.array_equal(out[0][0], out[1][0])
    nb = -(-lens.cpu().numpy() // bs)
    assert np.array_equal(out[1][1], np.minimum(nb, k)[:, None].repeat(Hkv, 1))
    over = kin.make_dims(B, Hkv, Hq, D, bs, Lcap + 1)  # 4097 blocks per sequence
    p = [ctypes.c_void_p(x.data_ptr()) for x in (q, means, lens, ws, ws)]
    rc = kin.load_library().kin_block_topk_select_noalloc(ctypes.byref(over), p[0], p[1], p[2], k, p[3], p[4],
                                                          None, None)
    assert rc == 3


def test_noalloc_select_rejects_problems_beyond_its_scratch():
    # B * Hkv * ceil(Lcap / bs) = 64 * 8 * 8192 > 2^21 scores
    # (the C entry point itself, with small stand-in buffers: it refuses before
    # launching anything; the binding would refuse the short buffers first)
    import ctypes
    dims = kin.make_dims(64, 8, 32, D, 16, 8192 * 16)
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    q = torch.zeros((1, D), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros(4, device="cuda")
    p = [ctypes.c_void_p(x.data_ptr()) for x in (q, m, t, t, t)]
    rc = kin.load_library().kin_block_topk_select_noalloc(ctypes.byref(dims), p[0], p[1], p[2], 8, p[3], p[4],
                                                          None, None)
    assert rc == 3
