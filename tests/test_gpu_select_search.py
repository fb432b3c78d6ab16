"""The top-k's two threshold searches, and large or mixed batches, on the GPU.

Inside the top-k, a search over equal-width score bins is tried first and a
radix search takes over when the score range is empty or the boundary bin is
crowded: crafted block means drive each branch, with the expected selection
taken from the oracle on the same fp32 means (and the allocation-free entry
point must agree bit for bit).  Then a batch of 1030 sequences, and a batch
mixing a bad length with dense and scanned sequences, whose workspace must
stay usable for the next call.
"""
import numpy as np
import pytest
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_testlib import D, all_pairs, check_pairs, gpu_step, make_device_case

pytestmark = pytest.mark.gpu


def _select(dims, q, means, lens, k, noalloc=False):
    B, Hkv = dims.batch, dims.num_kv_heads
    sel = torch.full((B, Hkv, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if noalloc:
        kin.kin_block_topk_select_noalloc(dims, q, means, lens, k, sel, cnt, st)
    else:
        ws = kin.alloc_workspace(dims, k)
        kin.kin_block_topk_select(dims, q, means, lens, k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    return sel.cpu().numpy(), cnt.cpu().numpy(), int(st.item())


def _crafted_case(B, Hkv, g, bs, lens, first_dim_values):
    """q has 1.0 in dim 0 of every head and 0 elsewhere, so a block's score is
    g * m[0] / sqrt(D) computed without rounding in the sums; means carry
    first_dim_values[b][h] (fp32) in dim 0 and a small pattern elsewhere."""
    Lcap = max(lens)
    nbcap = -(-Lcap // bs)
    dims = kin.make_dims(B, Hkv, Hkv * g, D, bs, Lcap)
    q = torch.zeros((B, Hkv * g, D), dtype=torch.bfloat16, device="cuda")
    q[:, :, 0] = 1.0
    means_h = np.zeros((B, Hkv, nbcap, D), np.float32)
    means_h[..., 1:] = 0.25
    for b in range(B):
        for h in range(Hkv):
            v = np.asarray(first_dim_values[b][h], np.float32)
            means_h[b, h, :len(v), 0] = v
    means = torch.from_numpy(means_h).cuda()
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    q_bits = ki.bf16_from_f32(q.float().cpu().numpy())
    return dims, q, means, lens_t, means_h, q_bits


def _oracle_sel(means_h, q_bits, lens, bs, g, k):
    B, Hkv = means_h.shape[:2]
    out = {}
    for b in range(B):
        nb = -(-lens[b] // bs)
        for h in range(Hkv):
            sc = oracle.block_scores(q_bits[b, h * g:(h + 1) * g], means_h[b, h, :nb].astype(np.float64))
            out[b, h] = oracle.select(sc, k)
    return out


def test_crafted_scores_exercise_both_threshold_searches():
    rng = np.random.default_rng(5)
    bs, g, k = 16, 4, 64
    lens = [700 * bs, 640 * bs - 3]
    nbs = [700, 640]
    vals = []
    for b in range(2):
        nb = nbs[b]
        pairs = [
            # well spread: the equal-width bins settle it
            rng.normal(0.0, 1.0, nb),
            # one far outlier: every other block falls in the lowest bin, which
            # is too crowded to rank pairwise, so the radix search runs
            np.where(np.arange(nb) == 17, 1e6, 1.0 + 1e-6 * (np.arange(nb) // 3)),
            # heavy hitters above a cluster with ties of three (the threshold
            # falls inside the cluster: equal scores go to lower indices)
            np.where(rng.random(nb) < 0.05, 50.0 + rng.random(nb), 2.0 + 1e-2 * (np.arange(nb) // 3)),
            # negative scores only
            -1.0 - rng.random(nb),
            # one outlier widens the bins, so the boundary bin holds nearly
            # every block (too many to rank pairwise: the radix search runs),
            # with ties of two around the threshold
            np.where(np.arange(nb) == 5, 1e3,
                     np.where(np.arange(nb) == 9, 0.0, 1.0 + 1e-3 * (np.arange(nb) // 2))),
        ]
        vals.append(pairs)
    dims, q, means, lens_t, means_h, q_bits = _crafted_case(2, 5, g, bs, lens, vals)
    ref = _oracle_sel(means_h, q_bits, lens, bs, g, k)
    sel_f, cnt_f, st_f = _select(dims, q, means, lens_t, k)
    sel_n, cnt_n, st_n = _select(dims, q, means, lens_t, k, noalloc=True)
    assert st_f == 0 and st_n == 0
    assert np.array_equal(sel_f, sel_n) and np.array_equal(cnt_f, cnt_n)
    for (b, h), (rsel, rcnt) in ref.items():
        assert cnt_f[b, h] == rcnt == k
        assert list(sel_f[b, h]) == list(rsel), (b, h)


def test_long_row_boundary_bin_ranked_through_sub_bins():
    """A pair of 9000 blocks (keys in shared memory): one outlier widens the
    bins, the rest climb steeply (v = 0.1 + 39 (i/9000)^4, in ties of two), so
    the boundary bin holds ~280 keys and the threshold is found through its
    sub-bins, one tie pair per sub-bin, with the budget taking one key of the
    deciding pair (the lower index); a second pair with the same blocks
    reversed puts the ties' lower index on the other side."""
    bs, g, k, nb = 16, 4, 601, 9000
    i = np.arange(nb)
    v = 0.1 + 39.0 * ((i // 2) * 2 / nb) ** 4
    v = np.where(i == 5, 1e3, np.where(i == 9, 0.0, v))
    vals = [[v, v[::-1].copy()]]
    lens = [nb * bs]
    dims, q, means, lens_t, means_h, q_bits = _crafted_case(1, 2, g, bs, lens, vals)
    ref = _oracle_sel(means_h, q_bits, lens, bs, g, k)
    sel_f, cnt_f, st_f = _select(dims, q, means, lens_t, k)
    sel_n, cnt_n, st_n = _select(dims, q, means, lens_t, k, noalloc=True)
    assert st_f == 0 and st_n == 0
    assert np.array_equal(sel_f, sel_n) and np.array_equal(cnt_f, cnt_n)
    for (b, h), (rsel, rcnt) in ref.items():
        assert cnt_f[b, h] == rcnt == k
        assert list(sel_f[b, h]) == list(rsel), (b, h)


def test_large_batch_with_dense_scanned_and_bad_lengths():
    """1030 sequences, dense and scanned mixed; every pair against the
    oracle, then one bad length in the middle, flagged and emptied."""
    w = ki.Workload("b1030", 1030, 1, 2, D, 16, 40, 1000, 8, 61, Lcap=1024)
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    check_pairs(dc, [(w.k, gr)], all_pairs(w))
    # a bad length in the middle of the batch
    lens = dc.seq_lens.clone()
    lens[500] = 0
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_topk_select(dc.dims, dc.q, dc.means, lens, w.k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    assert int(cnt[500, 0].item()) == 0 and bool((sel[500, 0] == -1).all())
    assert np.array_equal(sel.cpu().numpy()[:500], gr.sel[:500])


def test_bad_length_among_dense_and_scanned_pairs_then_reuse():
    """A bad length, dense sequences and scanned ones in one batch: the good
    pairs keep their results and the workspace stays usable for the next
    call."""
    w = ki.Workload("mixed", 6, 2, 8, D, 16, 0, 0, 10, 62, Lcap=2048,
                    lens=(2048, 100, 1500, 160, 161, 777))
    dc = make_device_case(w)
    gr = gpu_step(dc, w.k)
    assert gr.status == 0
    lens = dc.seq_lens.clone()
    lens[2] = 5000  # beyond Lcap
    ws = kin.alloc_workspace(dc.dims, w.k)
    sel = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        kin.kin_block_topk_select(dc.dims, dc.q, dc.means, lens, w.k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
    s, c = sel.cpu().numpy(), cnt.cpu().numpy()
    assert np.all(c[2] == 0) and np.all(s[2] == -1)
    keep = [b for b in range(w.B) if b != 2]
    assert np.array_equal(s[keep], gr.sel[keep]) and np.array_equal(c[keep], gr.cnt[keep])
    # the same workspace, back to good lengths: identical to the first result
    st.zero_()
    kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, w.k, sel, cnt, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(sel.cpu().numpy(), gr.sel) and np.array_equal(cnt.cpu().numpy(), gr.cnt)
