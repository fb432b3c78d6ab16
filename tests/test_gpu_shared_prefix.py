"""Shared-prompt (Best-of-N) reuse on the GPU: groups of samples whose block
tables map the prompt's blocks to one set of pages, with block means stored
per page.  The per-page-means select must equal the select over logical
means of the same blocks, bit for bit (and so the outputs); sampled pairs
are checked against the oracle on the logical sequences gathered through
the table; appends into a sample's own pages refresh only its page means."""
import math

import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import D, make_device_case
from kin_tiecheck import check_topk_set

pytestmark = pytest.mark.gpu
W = ki.Workload


def shared_pool(dc, n, prompt_blocks, seed):
    """Pages for groups of n consecutive sequences: the prompt blocks of every
    sample map to the group's first sample's pages; other blocks (up to the
    post-append length) get pages of their own, in shuffled order."""
    w = dc.w
    B, Hkv, cap, D_ = dc.k_cache.shape
    bs, nbcap = w.bs, w.nbcap
    nbs = [-(-int(L) // bs) for L in dc.lens_final]
    table = np.full((B, nbcap), -1, np.int64)
    owner = []  # (b, i) whose rows fill each page
    for b in range(B):
        first = b - b % n
        for i in range(nbs[b]):
            if i < prompt_blocks and b != first:
                table[b, i] = table[first, i]
            else:
                table[b, i] = len(owner)
                owner.append((b, i))
    P = len(owner)
    perm = np.random.default_rng(seed).permutation(P)
    table = np.where(table >= 0, perm[np.maximum(table, 0)], -1).astype(np.int32)
    src_b = torch.tensor([o[0] for o in owner], device="cuda")
    src_i = torch.tensor([o[1] for o in owner], device="cuda")
    dst = torch.from_numpy(perm.astype(np.int64)).cuda()
    pools = []
    for cache in (dc.k_cache, dc.v_cache):
        padded = torch.nn.functional.pad(cache, (0, 0, 0, nbcap * bs - cap))
        pool = torch.full((P, Hkv, bs, D_), float("nan"), dtype=torch.bfloat16, device="cuda")
        pool[dst] = padded.view(B, Hkv, nbcap, bs, D_)[src_b, :, src_i]
        pools.append(pool)
    return pools[0], pools[1], torch.from_numpy(table).cuda(), table


def run(dc, kpool, vpool, table, per_page, k, seq=None, bf16=False, dual=False):
    w = dc.w
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    seq = dc.seq_lens.clone() if seq is None else seq
    dt = torch.bfloat16 if bf16 else torch.float32
    shape = (kpool.shape[0], w.Hkv, w.D) if per_page else (w.B, w.Hkv, w.nbcap, w.D)
    if dual:  # fp32 means, their bf16 rounding and the radii, in one buffer
        means = kin.alloc_dual_page_means(dc.dims, kpool.shape[0]) if per_page else kin.alloc_dual_means(dc.dims)
    else:
        means = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    kin.kin_block_means_build_ex(dc.dims, kpool, seq, means, block_table=table, dev_status=st, per_page=per_page)
    if w.n_append:
        kin.kin_block_means_update_ex(dc.dims, kpool, vpool, means, seq, dc.k_new, dc.v_new, w.n_append,
                                      block_table=table, dev_status=st, per_page=per_page)
    ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    if per_page:
        kin.kin_block_topk_select_paged(dc.dims, dc.q, means, table, seq, k, sel, cnt, ws, st,
                                        num_pages=kpool.shape[0])
    else:
        kin.kin_block_topk_select_ex(dc.dims, dc.q, means, seq, k, sel, cnt, ws, st)
    kin.kin_sparse_decode_attn_paged(dc.dims, dc.q, kpool, vpool, table, seq, sel, cnt, k, 0.0, out, lse, ws, st)
    torch.cuda.synchronize()
    return sel.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


def oracle_check(dc, kpool, vpool, table_host, b, h, k, sel, cnt, out, lse):
    """The oracle on the logical sequence of (b, h) gathered through the table."""
    w = dc.w
    L = int(dc.lens_final[b])
    kp = kpool.cpu().view(torch.int16).numpy().view(np.uint16)
    vp = vpool.cpu().view(torch.int16).numpy().view(np.uint16)
    K = oracle.gather_paged(kp, table_host[b], L, w.bs, h)
    V = oracle.gather_paged(vp, table_host[b], L, w.bs, h)
    qg = dc.q_host[b, h * w.g:(h + 1) * w.g]
    means = oracle.block_means(K, L, w.bs)
    scores = oracle.block_scores(qg, means)
    rsel, rcnt = oracle.select(scores, k)
    c = int(cnt[b, h])
    assert c == rcnt
    g = sel[b, h, :c]
    nb = means.shape[0]
    forced = {0, nb - 1}
    assert np.all(np.diff(g) > 0) and forced <= set(g.tolist()), (b, h)
    qf = ki.bf16_to_f32(qg).astype(np.float64)
    eps = (np.abs(qf).sum(axis=0) @ np.abs(means).T).mean() / math.sqrt(D)
    check_topk_set(scores, np.arange(1, nb - 1), [i for i in rsel[:rcnt] if i not in forced],
                   [i for i in g if i not in forced], eps, what=(b, h))
    o_ref, lse_ref = oracle.attend(qg, K, V, L, w.bs, g, 1 / math.sqrt(D))
    err = np.abs(out[b, h * w.g:(h + 1) * w.g].astype(np.float64) - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (b, h, err.max())
    assert np.all(np.abs(lse[b, h * w.g:(h + 1) * w.g] - lse_ref) <= 1e-3 + 1e-4 * np.abs(lse_ref))


@pytest.mark.parametrize("w,n,prompt_blocks", [
    (W("bon4_bs16", 8, 2, 8, D, 16, 0, 0, 16, 100, Lcap=1200,
       lens=(1100, 1050, 1199, 1001, 900, 990, 1111, 1024)), 4, 50),
    (W("bon2_bs32_append", 4, 2, 4, D, 32, 0, 0, 6, 101, Lcap=640, n_append=3,
       lens=(600, 500, 620, 400)), 2, 12),
], ids=lambda x: getattr(x, "name", str(x)))
@pytest.mark.parametrize("bf16", [False, True], ids=["fp32_means", "bf16_means"])
def test_shared_prompt_pages_and_page_means(w, n, prompt_blocks, bf16):
    dc = make_device_case(w)
    kpool, vpool, table, table_host = shared_pool(dc, n, prompt_blocks, seed=w.seed)
    # per-page means (one mean per shared page) against logical means of the same blocks
    kp2, vp2 = kpool.clone(), vpool.clone()
    a = run(dc, kpool, vpool, table, True, w.k, bf16=bf16)
    b_ = run(dc, kp2, vp2, table, False, w.k, bf16=bf16)
    assert a[4] == 0 and b_[4] == 0
    for x, y in zip(a[:4], b_[:4]):
        assert np.array_equal(x, y)
    if not bf16:
        sel, cnt, out, lse, _ = a
        for b in range(w.B):
            for h in range(w.Hkv):
                oracle_check(dc, kpool, vpool, table_host, b, h, w.k, sel, cnt, out, lse)


def test_shared_prompt_bad_page_is_flagged():
    w = W("bon_bad", 4, 1, 4, D, 16, 0, 0, 8, 102, Lcap=320, lens=(300, 300, 280, 310))
    dc = make_device_case(w)
    kpool, vpool, table, _ = shared_pool(dc, 2, 10, seed=3)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    means = torch.zeros((kpool.shape[0], w.Hkv, w.D), dtype=torch.float32, device="cuda")
    kin.kin_block_means_build_ex(dc.dims, kpool, dc.seq_lens, means, block_table=table, dev_status=st, per_page=True)
    bad = table.clone()
    bad[3, 15] = kpool.shape[0] + 4
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    kin.kin_block_topk_select_paged(dc.dims, dc.q, means, bad, dc.seq_lens, w.k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    assert np.all(cnt.cpu().numpy() == w.k)


@pytest.mark.parametrize("w,n,prompt_blocks", [
    (W("bon4_bs16", 8, 2, 8, D, 16, 0, 0, 16, 100, Lcap=1200,
       lens=(1100, 1050, 1199, 1001, 900, 990, 1111, 1024)), 4, 50),
    (W("bon2_bs32_append", 4, 2, 4, D, 32, 0, 0, 6, 101, Lcap=640, n_append=3,
       lens=(600, 500, 620, 400)), 2, 12),
    (W("bon8_32k_like", 8, 2, 8, D, 16, 0, 0, 128, 103, Lcap=16384, n_append=1,
       lens=(16000, 15000, 16383, 12000, 9000, 16200, 14000, 16383)), 8, 512),
], ids=lambda x: getattr(x, "name", str(x)))
def test_dual_page_means_select_equals_fp32_page_means(w, n, prompt_blocks):
    """Dual means stored per page (the shared-prompt layout): the select reads
    their bf16 rows through the table and rescores the band from the fp32 rows
    through it, and must return the fp32 per-page select's blocks bit for bit
    (and so the same outputs); the logical dual means over the same pool give
    them too."""
    dc = make_device_case(w)
    kpool, vpool, table, _ = shared_pool(dc, n, prompt_blocks, seed=w.seed)
    pools = [(kpool.clone(), vpool.clone()) for _ in range(3)]
    f = run(dc, *pools[0], table, True, w.k)
    d = run(dc, *pools[1], table, True, w.k, dual=True)
    dl = run(dc, *pools[2], table, False, w.k, dual=True)
    assert f[4] == 0 and d[4] == 0 and dl[4] == 0
    for x, y, z in zip(f[:4], d[:4], dl[:4]):
        assert np.array_equal(x, y) and np.array_equal(x, z)


def test_dual_page_means_bad_page_is_flagged_and_scored_as_the_fp32_select():
    """A page index past the pool: flagged, the block scored from a zero row
    by both the fp32 and the dual per-page select, so both keep the same
    blocks."""
    w = W("bon_bad_dual", 4, 1, 4, D, 16, 0, 0, 8, 104, Lcap=320, lens=(300, 300, 280, 310))
    dc = make_device_case(w)
    kpool, vpool, table, _ = shared_pool(dc, 2, 10, seed=5)
    P = kpool.shape[0]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f32 = torch.zeros((P, w.Hkv, w.D), dtype=torch.float32, device="cuda")
    dual = kin.alloc_dual_page_means(dc.dims, P)
    kin.kin_block_means_build_ex(dc.dims, kpool, dc.seq_lens, f32, block_table=table, dev_status=st, per_page=True)
    kin.kin_block_means_build_ex(dc.dims, kpool, dc.seq_lens, dual, block_table=table, dev_status=st, per_page=True)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    bad = table.clone()
    bad[3, 15] = P + 4
    out = []
    for means in (f32, dual):
        ws = kin.alloc_workspace(dc.dims, w.k)
        sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
        cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
        st.zero_()
        kin.kin_block_topk_select_paged(dc.dims, dc.q, means, bad, dc.seq_lens, w.k, sel, cnt, ws, st, num_pages=P)
        torch.cuda.synchronize()
        assert int(st.item()) == 5
        assert np.all(cnt.cpu().numpy() == w.k)
        out.append(sel.cpu().numpy())
    assert np.array_equal(out[0], out[1])


def test_dual_page_means_buffer_needs_its_page_count():
    w = W("bon_count", 2, 1, 4, D, 16, 0, 0, 8, 105, Lcap=320, lens=(300, 300))
    dc = make_device_case(w)
    kpool, _, table, _ = shared_pool(dc, 2, 10, seed=6)
    dual = kin.alloc_dual_page_means(dc.dims, kpool.shape[0])
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        kin.kin_block_topk_select_paged(dc.dims, dc.q, dual, table, dc.seq_lens, w.k, sel, cnt, ws)
    with pytest.raises(ValueError):  # a buffer sized for fewer pages than the call names
        kin.kin_block_topk_select_paged(dc.dims, dc.q, dual, table, dc.seq_lens, w.k, sel, cnt, ws,
                                        num_pages=kpool.shape[0] + 1)

