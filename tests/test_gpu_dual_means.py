"""Dual block means (KIN_MEANS_DUAL): fp32 means, their bf16 rounding and
the row norms in one buffer; the select scans the bf16 copy and rescores
from the fp32 rows only the blocks its error bound cannot place.  It must
return exactly the fp32 select's indices, bit for bit, on every shape: the
fp32 select is itself checked against the oracle in the other GPU tests.
"""
import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
from kin_testlib import D, GpuResult, all_pairs, check_pairs, make_device_case, random_shapes, to_pages

pytestmark = pytest.mark.gpu
W = ki.Workload


def _parts(dual, dims):
    """The fp32 rows, bf16 rows and error radii of a dual buffer (views)."""
    rows = dims.batch * dims.num_kv_heads * (-(-dims.max_seq_len // dims.block_size))
    f32 = dual[:rows * D * 4].view(torch.float32).view(rows, D)
    b16 = dual[rows * D * 4:rows * D * 6].view(torch.bfloat16).view(rows, D)
    nrm = dual[rows * D * 6:rows * (D * 6 + 4)].view(torch.float32)
    return f32, b16, nrm


def _select(dc, means, k):
    w = dc.w
    ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.full((w.B, w.Hkv, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if means.dtype == torch.uint8:
        kin.kin_block_topk_select_ex(dc.dims, dc.q, means, dc.seq_lens, k, sel, cnt, ws, st)
    else:
        kin.kin_block_topk_select(dc.dims, dc.q, means, dc.seq_lens, k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return sel.cpu().numpy(), cnt.cpu().numpy()


def _build_both(w):
    """Two device cases of one workload (their caches are identical), one
    with fp32 means and one with dual means, each built and then appended to
    (when the workload appends) through its own calls."""
    a, b = make_device_case(w), make_device_case(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_means_build(a.dims, a.k_cache, a.seq_lens, a.means, st)
    dual = kin.alloc_dual_means(b.dims)
    kin.kin_block_means_build_ex(b.dims, b.k_cache, b.seq_lens, dual, dev_status=st)
    if w.n_append:
        kin.kin_block_means_update(a.dims, a.k_cache, a.v_cache, a.means, a.seq_lens, a.k_new, a.v_new,
                                   w.n_append, st)
        kin.kin_block_means_update_ex(b.dims, b.k_cache, b.v_cache, dual, b.seq_lens, b.k_new, b.v_new,
                                      w.n_append, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return a, b, dual


def _valid_rows(w, dc):
    nb = -(-dc.lens_final.astype(np.int64) // w.bs)
    nbcap = -(-w.cap // w.bs)
    return np.concatenate([((b * w.Hkv + h) * nbcap + np.arange(nb[b])) for b in range(w.B) for h in range(w.Hkv)])


@pytest.mark.parametrize("w", [
    W("dual_ragged_g4", 3, 2, 8, D, 16, 300, 3000, 40, 80, Lcap=3072),
    W("dual_append_bs32", 2, 2, 4, D, 32, 0, 0, 6, 81, Lcap=640, n_append=70, lens=(600, 97)),
    W("dual_bs128_g7", 2, 1, 7, D, 128, 129, 2000, 4, 82, Lcap=2048),
], ids=lambda w: w.name)
def test_dual_layout_build_and_update(w):
    """The fp32 part equals the fp32 means bit for bit, the bf16 part is its
    round-to-nearest-even bf16 rounding (torch's conversion), and each
    row's radius bounds |m - bf16(m)|_2 + 2^-19 |m|_2 + 2^-60 from above
    and exceeds (1 + 2^-12) |m - bf16(m)|_2 + 2^-18 |m|_2 + 2^-59 by no
    more than fp32 rounding; with an append, through the dual update."""
    a, b, dual = _build_both(w)
    f32, b16, rad = _parts(dual, b.dims)
    rows = torch.from_numpy(_valid_rows(w, b)).cuda()
    ref = a.means.view(-1, D)[rows]
    assert torch.equal(f32[rows], ref)
    assert torch.equal(b16[rows], ref.to(torch.bfloat16))
    m = ref.double()
    dn = torch.linalg.vector_norm(m - ref.to(torch.bfloat16).double(), dim=-1)
    mn = torch.linalg.vector_norm(m, dim=-1)
    r = rad[rows].double()
    assert bool((r >= dn + 2.0 ** -19 * mn + 2.0 ** -60).all())
    assert bool((r <= ((1 + 2.0 ** -12) * dn + 2.0 ** -18 * mn + 2.0 ** -59) * (1 + 2.0 ** -18)).all())
    assert bool((dn > 0).any())  # the rounding moved some rows


SHAPES = [
    W("dual_small_g4", 2, 2, 8, D, 16, 700, 1000, 16, 83, Lcap=1024),
    W("dual_g1_bs32", 3, 1, 1, D, 32, 33, 333, 5, 84, Lcap=400),
    W("dual_nb_edges", 6, 1, 4, D, 16, 0, 0, 8, 85, Lcap=160, lens=(112, 113, 128, 129, 144, 1)),
    W("dual_k2", 3, 2, 6, D, 16, 40, 700, 2, 86, Lcap=704),
    W("dual_cap2048", 1, 2, 8, D, 16, 0, 0, 256, 87, Lcap=2048 * 16, lens=(2048 * 16,)),
    W("dual_cap4097", 1, 2, 4, D, 16, 0, 0, 300, 88, Lcap=4097 * 16, lens=(4097 * 16,)),
    W("dual_cap8193", 1, 1, 4, D, 16, 0, 0, 500, 89, Lcap=8193 * 16, lens=(8193 * 16,)),
    W("dual_every_path", 7, 1, 2, D, 16, 0, 0, 64, 90, Lcap=8193 * 16,
      lens=(1, 64 * 16, 100 * 16 + 3, 4096 * 16, 4097 * 16, 8192 * 16, 8193 * 16)),
    W("dual_halve", 38, 8, 8, D, 16, 16400, 32768, 128, 91, Lcap=32768),
    W("dual_append_1", 2, 2, 8, D, 32, 0, 0, 40, 92, Lcap=4096, n_append=1, lens=(4096, 2049)),
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_dual_select_equals_fp32_select(w):
    a, b, dual = _build_both(w)
    assert np.array_equal(_select(a, a.means, w.k)[0], _select(b, dual, w.k)[0])
    assert np.array_equal(_select(a, a.means, w.k)[1], _select(b, dual, w.k)[1])


@pytest.mark.parametrize("w", random_shapes(16, seed=171, prefix="dual_rand"), ids=lambda w: w.name)
def test_dual_select_equals_fp32_select_random_shapes(w):
    """Seeded random shapes (block sizes 16-128, g 1-8, appends, k from 2 to past the block
    capacity): the dual select's indices and counts equal the fp32 select's."""
    a, b, dual = _build_both(w)
    sa, ca = _select(a, a.means, w.k)
    sb, cb = _select(b, dual, w.k)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)


@pytest.mark.parametrize("name,ks", [("qwen3_8b_32k", None), ("qwen3_14b_ragged", None),
                                     ("qwen3_32b_128k_append", None), ("qwen3_0p6b_sweep", (32, 128, 512))])
def test_dual_select_equals_fp32_select_full_size(name, ks):
    w = ki.WORKLOADS[name]
    a, b, dual = _build_both(w)
    for k in ks or (w.k,):
        sa, ca = _select(a, a.means, k)
        sb, cb = _select(b, dual, k)
        assert np.array_equal(ca, cb) and np.array_equal(sa, sb), (name, k)


@pytest.mark.parametrize("nblocks", [300, 8193])
def test_dual_select_with_all_equal_scores(nblocks):
    """q = 0: every score and every bound is 0, so no candidate can be
    excluded and all are rescored (beyond the 4096-entry list at 8193
    blocks); the tie rule keeps 0..k-2 and the last block."""
    w = W("dual_zeros", 2, 1, 4, D, 16, 0, 0, 50, 93, Lcap=nblocks * 16, lens=(nblocks * 16, nblocks * 16 - 5))
    a, b, dual = _build_both(w)
    for dc in (a, b):
        dc.q.zero_()
    sb, cb = _select(b, dual, w.k)
    sa, ca = _select(a, a.means, w.k)
    assert np.array_equal(sa, sb) and np.array_equal(ca, cb)
    for r in range(w.B):
        nb = -(-int(b.lens_final[r]) // 16)
        assert list(sb[r, 0]) == list(range(w.k - 1)) + [nb - 1]


@pytest.mark.parametrize("nblocks,boosted", [(1024, False), (1024, True), (5000, False)])
def test_dual_select_with_scores_tied_below_bf16_resolution(nblocks, boosted):
    """Every block holds the same key rows except one token, moved by a few
    bf16 ulps in one dim: the fp32 means differ by about 2^-12 relative, far
    below the bf16 copy's resolution, so the bf16 scores cannot order the
    blocks and the band is every candidate (listed at 1024 blocks; beyond
    the list at 5000, so every candidate is rescored).  With `boosted`, a
    seventh of the blocks are scaled by 1.5: the boundary falls inside that
    group, whose members are near-tied among themselves, and the rest is out.
    The dual select must still return the fp32 select's indices."""
    w = W("dual_subres", 2, 2, 8, D, 16, 0, 0, 40, 94, Lcap=nblocks * 16, lens=(nblocks * 16, nblocks * 16 - 300))
    a, b = make_device_case(w), make_device_case(w)
    g = torch.Generator().manual_seed(nblocks + boosted)
    nb = nblocks
    kc = torch.randn(w.B, w.Hkv, 1, D, generator=g).to(torch.bfloat16).expand(w.B, w.Hkv, w.cap, D).clone()
    if boosted:
        grp = torch.rand(nb, generator=g) < 1 / 7
        fac = torch.where(grp, 1.5, 1.0).repeat_interleave(16)[:w.cap].view(1, 1, -1, 1)
        kc = (kc.float() * fac).to(torch.bfloat16)
    bits = kc.view(torch.int16)
    dim = torch.randint(0, D, (nb,), generator=g)
    step = torch.randint(-3, 4, (w.B, w.Hkv, nb), generator=g, dtype=torch.int16)
    bits[:, :, torch.arange(nb) * 16, dim] += step
    kc = kc.cuda()
    for dc in (a, b):
        dc.k_cache.copy_(kc)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_means_build(a.dims, a.k_cache, a.seq_lens, a.means, st)
    dual = kin.alloc_dual_means(b.dims)
    kin.kin_block_means_build_ex(b.dims, b.k_cache, b.seq_lens, dual, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    sa, ca = _select(a, a.means, w.k)
    sb, cb = _select(b, dual, w.k)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)
    # the fp32 means do differ between blocks, below the bf16 copy's resolution
    f32, b16, _ = _parts(dual, b.dims)
    assert len(torch.unique(f32.view(w.B, w.Hkv, -1, D)[0, 0, :nb], dim=0)) > 300
    assert len(torch.unique(b16.view(w.B, w.Hkv, -1, D)[0, 0, :nb], dim=0)) <= 2


@pytest.mark.parametrize("w", [
    W("dual_paged_g4_bs16", 3, 2, 8, D, 16, 300, 1000, 12, 95, Lcap=1024),
    W("dual_paged_bs128", 2, 2, 4, D, 128, 129, 1000, 3, 96, Lcap=1024),
    W("dual_paged_append_7", 2, 2, 8, D, 16, 0, 0, 6, 97, Lcap=200, n_append=7, lens=(100, 44)),
    W("dual_paged_append_1_new_page", 2, 1, 4, D, 32, 0, 0, 3, 98, Lcap=160, n_append=1, lens=(128, 64)),
], ids=lambda w: w.name)
def test_dual_means_from_a_paged_cache_equal_the_contiguous_ones(w):
    """Dual means built (and appended to) through a block table over a shuffled page
    pool: the fp32 rows, bf16 rows and radii equal those built from the contiguous
    cache, byte for byte, and the dual select keeps the same blocks."""
    a, b = make_device_case(w), make_device_case(w)
    pg = to_pages(b, seed=w.seed)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dual_c, dual_p = kin.alloc_dual_means(a.dims), kin.alloc_dual_means(b.dims)
    kin.kin_block_means_build_ex(a.dims, a.k_cache, a.seq_lens, dual_c, dev_status=st)
    kin.kin_block_means_build_ex(b.dims, pg.k, b.seq_lens, dual_p, block_table=pg.table, dev_status=st)
    if w.n_append:
        kin.kin_block_means_update_ex(a.dims, a.k_cache, a.v_cache, dual_c, a.seq_lens, a.k_new, a.v_new,
                                      w.n_append, dev_status=st)
        kin.kin_block_means_update_ex(b.dims, pg.k, pg.v, dual_p, b.seq_lens, b.k_new, b.v_new, w.n_append,
                                      block_table=pg.table, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(a.seq_lens, b.seq_lens)
    rows = torch.from_numpy(_valid_rows(w, a)).cuda()
    for part_c, part_p in zip(_parts(dual_c, a.dims), _parts(dual_p, b.dims)):
        assert torch.equal(part_c[rows].view(torch.uint8), part_p[rows].view(torch.uint8))
    sa, ca = _select(a, dual_c, w.k)
    sb, cb = _select(b, dual_p, w.k)
    assert np.array_equal(ca, cb) and np.array_equal(sa, sb)


def test_dual_means_size():
    dims = kin.make_dims(2, 2, 8, D, 16, 256)
    assert kin.kin_dual_means_bytes(dims) == 2 * 2 * 16 * (D * 6 + 4)
    assert kin.kin_dual_page_means_bytes(dims, 7) == 7 * 2 * (D * 6 + 4)


@pytest.mark.parametrize("name", ["qwen3_8b_32k", "qwen3_32b_128k_append"])
def test_dual_step_against_the_oracle_every_pair(name):
    """The benchmark's default step, at full size: dual means built (and
    appended to), the dual select, the attention; every pair's means (the
    fp32 part), selection, outputs and lse against the oracle."""
    w = ki.WORKLOADS[name]
    dc = make_device_case(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dual = kin.alloc_dual_means(dc.dims)
    kin.kin_block_means_build_ex(dc.dims, dc.k_cache, dc.seq_lens, dual, dev_status=st)
    if w.n_append:
        kin.kin_block_means_update_ex(dc.dims, dc.k_cache, dc.v_cache, dual, dc.seq_lens, dc.k_new, dc.v_new,
                                      w.n_append, dev_status=st)
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    kin.kin_block_topk_select_ex(dc.dims, dc.q, dual, dc.seq_lens, w.k, sel, cnt, ws, st)
    kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, w.k, 0.0, out, lse, ws, st)
    torch.cuda.synchronize()
    gr = GpuResult(sel.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item()))
    assert gr.status == 0
    means = _parts(dual, dc.dims)[0].view(w.B, w.Hkv, -1, D).cpu().numpy()
    del dc.k_cache, dc.v_cache
    torch.cuda.empty_cache()
    near = check_pairs(dc, [(w.k, gr)], all_pairs(w), gpu_means=means)
    print(f"{name} (dual means): {w.B * w.Hkv} pairs against the oracle, {near} near-tie selections")
