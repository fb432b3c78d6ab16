"""Pins for the fp64 oracle, each against something other than the oracle's
own formula: a library routine (torch SDPA, scipy softmax, logsumexp), brute
force over all block subsets, a different but equivalent computation (mean of
per-token logits vs logit of the mean key), invariants (convex hull, constant
V, split-K merge invariance, incremental == from-scratch means) and a
constructed case (a planted block).

The method (block top-k sparse decode attention) is described on the pages
"Kinetics: Memory-Aware Test-Time Scaling" (Architecture Overview;
Implementation, BlockTopKAttention) and "Kinetics: Rethinking Test-Time
Scaling Law" (author response Q4, KV block size and grouping strategy).
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import kin_inputs as ki
import oracle

D = 128


def rand_bf16(rng, shape, scale=1.0):
    return ki.bf16_from_f32((rng.standard_normal(shape) * scale).astype(np.float32))


def f64(bits):
    return ki.bf16_to_f32(bits).astype(np.float64)


# --------------------------------------------------------------- dense == SDPA
@pytest.mark.parametrize("g,bs,lens", [(4, 16, (83, 130)), (1, 32, (64, 31)), (5, 64, (200, 1)),
                                       (8, 16, (16, 17))])
def test_full_budget_is_dense_attention(g, bs, lens):
    """With k >= nb the method is plain softmax(q K^T / sqrt(d)) V over all
    tokens (budget = block size x blocks covers the whole cache)."""
    rng = np.random.default_rng(1 + g + bs)
    B, Hkv = len(lens), 2
    Hq = Hkv * g
    lens = np.array(lens, np.int32)
    Lcap = int(lens.max()) + 7
    q = rand_bf16(rng, (B, Hq, D))
    Kc = rand_bf16(rng, (B, Hkv, Lcap, D))
    Vc = rand_bf16(rng, (B, Hkv, Lcap, D))
    for b in range(B):  # rows beyond the length are poison and must be ignored
        Kc[b, :, lens[b]:] = ki.BF16_NAN
        Vc[b, :, lens[b]:] = ki.BF16_NAN
    nbcap = -(-Lcap // bs)
    means = np.zeros((B, Hkv, nbcap, D))
    for b in range(B):
        for h in range(Hkv):
            m = oracle.block_means(Kc[b, h], int(lens[b]), bs)
            means[b, h, :m.shape[0]] = m
    k = nbcap + 3
    res = oracle.decode_pairs(Hkv=Hkv, Hq=Hq, bs=bs, seq_lens=lens, q=q, Kc=Kc, Vc=Vc, means=means,
                              k=k, scale=1 / math.sqrt(D), pairs=np.arange(B * Hkv))
    for b in range(B):
        L = int(lens[b])
        qt = torch.from_numpy(f64(q[b])).view(1, Hq, 1, D)
        Kt = torch.from_numpy(f64(Kc[b, :, :L])).repeat_interleave(g, dim=0).view(1, Hq, L, D)
        Vt = torch.from_numpy(f64(Vc[b, :, :L])).repeat_interleave(g, dim=0).view(1, Hq, L, D)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt).view(Hq, D).numpy()
        lse_ref = torch.logsumexp((qt @ Kt.transpose(-1, -2)) / math.sqrt(D), dim=-1).view(Hq).numpy()
        for h in range(Hkv):
            p = b * Hkv + h
            nb = -(-L // bs)
            assert res["cnt"][p] == nb
            assert list(res["sel"][p, :nb]) == list(range(nb))
            assert np.all(res["sel"][p, nb:] == -1)
            np.testing.assert_allclose(res["out"][p], ref[h * g:(h + 1) * g], rtol=0, atol=1e-12)
            np.testing.assert_allclose(res["lse"][p], lse_ref[h * g:(h + 1) * g], rtol=1e-13, atol=1e-12)


# ------------------------------------------------------- selection brute force
def brute_force_select(scores, k):
    nb = len(scores)
    if k >= nb:
        return list(range(nb))
    forced = [0, nb - 1]
    best = None
    for combo in itertools.combinations(range(1, nb - 1), k - 2):
        s = sorted(forced + list(combo))
        tot = sum(scores[i] for i in s)
        key = (-tot, tuple(s))
        if best is None or key < best[0]:
            best = (key, s)
    return best[1]


@pytest.mark.parametrize("trial", range(300))
def test_select_maximises_summed_score(trial):
    rng = np.random.default_rng(1000 + trial)
    nb = int(rng.integers(1, 15))
    k = int(rng.integers(2, 7))
    if trial % 3 == 0:
        scores = rng.integers(-3, 4, nb) / 8.0           # many exact ties
    elif trial % 3 == 1:
        scores = rng.standard_normal(nb)
    else:
        scores = np.full(nb, 0.25)                        # all equal
        scores[rng.integers(0, nb)] = -1.0
    sel, cnt = oracle.select(scores, k)
    expect = brute_force_select(list(scores), k)
    assert cnt == len(expect)
    assert list(sel[:cnt]) == expect
    assert np.all(sel[cnt:] == -1)


def test_select_rejects_budget_below_forced_pair():
    _, c = oracle.select(np.zeros(5), 1)
    assert c == -1
    sel, c = oracle.select(np.zeros(1), 1)   # one block fits a budget of one
    assert c == 1 and sel[0] == 0


def test_select_all_equal_prefers_low_indices():
    sel, c = oracle.select(np.zeros(300), 10)
    assert c == 10
    assert list(sel) == list(range(9)) + [299]


def test_select_large_topk_property():
    rng = np.random.default_rng(5)
    nb, k = 2048, 256
    scores = np.round(rng.standard_normal(nb) * 16) / 16   # ties at the boundary
    sel, c = oracle.select(scores, k)
    assert c == k and sel[0] == 0 and sel[-1] == nb - 1
    assert np.all(np.diff(sel) > 0)
    chosen = set(int(i) for i in sel) - {0, nb - 1}
    tau = min(scores[i] for i in chosen)
    for i in range(1, nb - 1):
        if scores[i] > tau:
            assert i in chosen
    eq = [i for i in range(1, nb - 1) if scores[i] == tau]
    taken = [i for i in eq if i in chosen]
    assert taken == eq[:len(taken)]


# ------------------------------------------------------------------ linearity
@pytest.mark.parametrize("L,bs,g", [(150, 16, 5), (64, 32, 1), (257, 64, 8)])
def test_scores_equal_group_sum_of_mean_token_logits(L, bs, g):
    """score(block) from the mean key == sum over the group of the mean of the
    per-token logits q_j . K_t / sqrt(D) over the block's valid tokens."""
    rng = np.random.default_rng(L)
    q = rand_bf16(rng, (g, D))
    K = rand_bf16(rng, (L + 5, D))
    K[L:] = ki.BF16_NAN
    s = oracle.block_scores(q, oracle.block_means(K, L, bs))
    z = f64(q) @ f64(K[:L]).T / math.sqrt(D)           # [g, L]
    nb = -(-L // bs)
    ref = np.array([z[:, i * bs:min((i + 1) * bs, L)].mean(axis=1).sum() for i in range(nb)])
    np.testing.assert_allclose(s, ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------- softmax weights pins
def test_onehot_values_expose_softmax_weights():
    """V_t = e_t makes o_j[t] the weight of token t: compare with scipy's
    softmax of the logits, dense and sparse."""
    rng = np.random.default_rng(3)
    L, bs, g = 100, 16, 3
    q = rand_bf16(rng, (g, D))
    K = rand_bf16(rng, (L, D), 0.7)
    V = np.zeros((L, D), np.uint16)
    V[np.arange(L), np.arange(L)] = 0x3F80        # bf16 1.0
    z = f64(q) @ f64(K).T / math.sqrt(D)
    nb = -(-L // bs)
    out, lse = oracle.attend(q, K, V, L, bs, np.arange(nb), 1 / math.sqrt(D))
    w = out[:, :L]
    np.testing.assert_allclose(w, scipy.special.softmax(z, axis=1), rtol=1e-13, atol=1e-15)
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-14)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(z, axis=1), rtol=1e-14)
    blocks = np.array([0, 2, 6])
    out, _ = oracle.attend(q, K, V, L, bs, blocks, 1 / math.sqrt(D))
    toks = np.concatenate([np.arange(b * bs, min((b + 1) * bs, L)) for b in blocks])
    ref = np.zeros((g, L))
    ref[:, toks] = scipy.special.softmax(z[:, toks], axis=1)
    np.testing.assert_allclose(out[:, :L], ref, rtol=1e-13, atol=1e-15)


def test_output_in_convex_hull_and_constant_values():
    rng = np.random.default_rng(4)
    L, bs, g = 333, 32, 4
    q = rand_bf16(rng, (g, D), 2.0)
    K = rand_bf16(rng, (L, D))
    V = rand_bf16(rng, (L, D))
    blocks = np.array([0, 3, 4, 9, 10])
    out, _ = oracle.attend(q, K, V, L, bs, blocks, 1 / math.sqrt(D))
    toks = np.concatenate([np.arange(b * bs, min((b + 1) * bs, L)) for b in blocks])
    vs = f64(V[toks])
    assert np.all(out >= vs.min(axis=0) - 1e-12)
    assert np.all(out <= vs.max(axis=0) + 1e-12)
    Vc = np.full((L, D), ki.bf16_from_f32(np.array([1.375], np.float32))[0], np.uint16)
    out, _ = oracle.attend(q, K, Vc, L, bs, blocks, 1 / math.sqrt(D))
    np.testing.assert_allclose(out, 1.375, rtol=0, atol=1e-14)


# ------------------------------------------------------------ split-K merge
@pytest.mark.parametrize("nchunks", [1, 2, 7, 13])
def test_chunked_merge_equals_single_pass(nchunks):
    rng = np.random.default_rng(nchunks)
    L, bs, g = 16 * 40 - 5, 16, 5
    q = rand_bf16(rng, (g, D), 1.5)
    K = rand_bf16(rng, (L, D))
    V = rand_bf16(rng, (L, D))
    blocks = np.array(sorted(rng.choice(np.arange(1, 39), 11, replace=False).tolist()) + [0, 39])
    blocks.sort()
    full, lse_full = oracle.attend(q, K, V, L, bs, blocks, 1 / math.sqrt(D))
    parts = np.array_split(blocks, nchunks)
    os_, ms, ls = zip(*[oracle.attend_partial(q, K, V, L, bs, p, 1 / math.sqrt(D)) for p in parts])
    out, lse = oracle.merge(np.stack(os_), np.stack(ms), np.stack(ls))
    np.testing.assert_allclose(out, full, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse_full, rtol=1e-14)


# --------------------------------------------------------------- means update
@pytest.mark.parametrize("bs", [16, 32])
def test_incremental_update_equals_build_from_scratch(bs):
    rng = np.random.default_rng(bs)
    Lcap = 130
    Kall = rand_bf16(rng, (Lcap, D))
    Vall = rand_bf16(rng, (Lcap, D))
    for steps in ([1] * Lcap, [7, 1, 30, 2, 16, 1, 73]):
        Kc = np.zeros((Lcap, D), np.uint16)
        Vc = np.zeros((Lcap, D), np.uint16)
        means = np.zeros((-(-Lcap // bs), D))
        L = 0
        for n in steps:
            oracle.means_update(Kc, Vc, L, Kall[L:L + n], Vall[L:L + n], bs, means)
            L += n
            ref = oracle.block_means(Kall, L, bs)
            assert np.array_equal(means[:ref.shape[0]], ref)
        assert np.array_equal(Kc, Kall) and np.array_equal(Vc, Vall)


def test_means_are_plain_averages():
    """The mean of a block is the arithmetic mean of its valid rows (numpy)."""
    rng = np.random.default_rng(11)
    L, bs = 75, 16
    K = rand_bf16(rng, (L, D))
    m = oracle.block_means(K, L, bs)
    for i in range(m.shape[0]):
        np.testing.assert_allclose(m[i], f64(K[i * bs:min((i + 1) * bs, L)]).mean(axis=0), rtol=1e-15, atol=1e-16)


# ------------------------------------------------------------- planted block
def test_planted_block_is_selected_and_dominates():
    rng = np.random.default_rng(12)
    L, bs, g, k = 16 * 64, 16, 4, 8
    q = rand_bf16(rng, (g, D))
    K = rand_bf16(rng, (L, D))
    V = rand_bf16(rng, (L, D))
    planted = 37
    q0 = f64(q[0])
    K[planted * bs:(planted + 1) * bs] = ki.bf16_from_f32((8.0 * q0).astype(np.float32))
    means = oracle.block_means(K, L, bs)
    scores = oracle.block_scores(q, means)
    sel, c = oracle.select(scores, k)
    assert c == k and planted in sel
    out, _ = oracle.attend(q[:1], K, V, L, bs, sel, 1 / math.sqrt(D))
    np.testing.assert_allclose(out[0], f64(V[planted * bs:(planted + 1) * bs]).mean(axis=0), atol=1e-12)


def test_gather_paged_follows_the_block_table():
    """Token t of a paged sequence is row t % bs of page table[t // bs]: a
    hand-made pool whose rows carry (page, row) markers, an identity layout,
    and a shuffled pool that must give back the contiguous rows."""
    bs, Hkv, D = 4, 2, 3
    pool = np.zeros((5, Hkv, bs, D), np.int32)
    for pg in range(5):
        for h in range(Hkv):
            for r in range(bs):
                pool[pg, h, r] = (pg, h, r)
    table = np.array([3, 0, 4], np.int32)
    got = oracle.gather_paged(pool, table, 10, bs, 1)
    assert got.shape == (10, D)
    for t in range(10):
        assert tuple(got[t]) == (table[t // bs], 1, t % bs)
    rng = np.random.default_rng(3)
    cont = rng.integers(0, 1 << 16, size=(Hkv, 12, D)).astype(np.uint16)  # 3 blocks of bs 4
    ident = cont.reshape(Hkv, 3, bs, D).transpose(1, 0, 2, 3)
    assert np.array_equal(oracle.gather_paged(ident, np.arange(3), 11, bs, 1), cont[1, :11])
    perm = rng.permutation(6)[:3]
    shuffled = np.zeros((6, Hkv, bs, D), np.uint16)
    shuffled[perm] = ident
    assert np.array_equal(oracle.gather_paged(shuffled, perm, 12, bs, 0), cont[0])


def test_round_bf16_matches_torch_conversion():
    """bf16 rounding against torch's float32 -> bfloat16 conversion (round to
    nearest even) on fp32 values, including exact ties and both signs."""
    import torch
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 2000) * 1e3,
                        [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 0.0, 255.5, 3.0]]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64)), want)
    # ties go to even: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7
    assert oracle.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert oracle.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6


def _bits(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_token_topk_full_budget_is_dense_attention():
    import torch
    rng = np.random.default_rng(21)
    g, L, D = 3, 57, 128
    q = _bits(rng.normal(size=(g, D)))
    K = _bits(rng.normal(size=(L + 5, D)))
    V = _bits(rng.normal(size=(L + 5, D)))
    scale = 1 / np.sqrt(D)
    sel, out, lse, _ = oracle.token_topk_attend(q, K, V, L, L + 3, scale)
    assert np.array_equal(sel, np.tile(np.arange(L), (g, 1)))
    qt = torch.from_numpy(oracle.bf16_bits_to_f64(q))[:, None, None, :]
    kt = torch.from_numpy(oracle.bf16_bits_to_f64(K[:L]))[None, None]
    vt = torch.from_numpy(oracle.bf16_bits_to_f64(V[:L]))[None, None]
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt.expand(g, 1, L, D), vt.expand(g, 1, L, D))
    assert np.allclose(out, want[:, 0, 0].numpy(), atol=1e-12, rtol=0)
    logits = (qt[:, 0, 0] @ kt[0, 0].T) * scale
    assert np.allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("trial", range(20))
def test_token_topk_keeps_the_best_set(trial):
    """Brute force over every token subset of the budget's size: the kept set
    maximises the summed logit and is the lexicographically smallest such set
    (ties to the lower index); dyadic logits make ties exact."""
    rng = np.random.default_rng(100 + trial)
    L, D = int(rng.integers(3, 11)), 128
    n = int(rng.integers(1, L))
    q = np.zeros((1, D), np.float32)
    q[0, 0] = 1.0
    K = np.zeros((L, D), np.float32)
    K[:, 0] = rng.integers(-3, 4, size=L) * 0.5
    sel, _, _, z = oracle.token_topk_attend(_bits(q), _bits(K), _bits(K), L, n, 1.0)
    best = max(itertools.combinations(range(L), n), key=lambda s: (sum(z[0, list(s)]), [-i for i in s]))
    assert list(sel[0]) == list(best)


def test_token_topk_weights_are_softmax_of_kept_logits_only():
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(7)
    L, D, n = 40, 128, 9
    q = _bits(rng.normal(size=(1, D)))
    K = _bits(rng.normal(size=(L, D)))
    V = _bits(np.eye(L, D, dtype=np.float32))      # one-hot rows: out exposes the weights (L <= D)
    sel, out, lse, z = oracle.token_topk_attend(q, K, V, L, n, 0.2)
    w = np.zeros(L)
    w[sel[0]] = softmax(z[0, sel[0]])
    assert np.allclose(out[0, :L], w, atol=1e-14)
    assert np.all(out[0, :L][np.setdiff1d(np.arange(L), sel[0])] == 0)
    assert np.isclose(lse[0], logsumexp(z[0, sel[0]]), atol=1e-12)
