"""The near-tie index rule (kin_tiecheck) on planted selections: a swap
across a wide score gap must be refused, a swap across a true near tie
accepted, and a GPU set that keeps a clearly worse item refused even when
the boundary itself is a near tie."""
import numpy as np
import pytest

from kin_tiecheck import TIE_REL, boundary, check_topk_set


def _oracle_keep(scores, cand, n):
    """Top n of the candidates by (score desc, index asc)."""
    order = sorted(cand, key=lambda i: (-scores[i], i))
    return sorted(order[:n])


def test_identical_sets_pass():
    s = np.array([5.0, 4.0, 3.0, 2.0, 1.0])
    assert check_topk_set(s, np.arange(5), [0, 1], [1, 0], eps=1.0) == 0


def test_boundary_swap_across_a_wide_gap_is_refused():
    # k = 3: the 3rd (1.0) and 4th (0.5) best differ by 0.5 >> delta
    s = np.array([3.0, 2.0, 1.0, 0.5, 0.1])
    ref = _oracle_keep(s, range(5), 3)
    assert ref == [0, 1, 2]
    with pytest.raises(AssertionError, match="boundary gap"):
        check_topk_set(s, np.arange(5), ref, [0, 1, 3], eps=1.0)


def test_boundary_swap_across_a_near_tie_passes():
    tau = 1.0
    d = TIE_REL * tau
    s = np.array([3.0, 2.0, tau, tau - 0.5 * d, 0.1])
    ref = _oracle_keep(s, range(5), 3)
    assert check_topk_set(s, np.arange(5), ref, [0, 1, 3], eps=1.0) == 1


def test_exact_tie_swap_passes():
    s = np.array([3.0, 1.0, 1.0, 0.0])
    ref = _oracle_keep(s, range(4), 2)      # ties to the lower index: [0, 1]
    assert ref == [0, 1]
    assert check_topk_set(s, np.arange(4), ref, [0, 2], eps=1.0) == 1


def test_near_tie_boundary_does_not_excuse_a_deep_swap():
    # the boundary (items 2 and 3) is a near tie, but the GPU dropped item 0
    # (far above the boundary) instead of item 2
    tau = 1.0
    d = TIE_REL * tau
    s = np.array([3.0, 2.0, tau, tau - 0.5 * d, 0.1])
    ref = _oracle_keep(s, range(5), 3)
    with pytest.raises(AssertionError, match="beats a kept one"):
        check_topk_set(s, np.arange(5), ref, [1, 2, 3], eps=1.0)


def test_near_tie_boundary_does_not_excuse_a_low_item():
    # the boundary is a near tie, but the GPU kept item 4, far below it
    tau = 1.0
    d = TIE_REL * tau
    s = np.array([3.0, 2.0, tau, tau - 0.5 * d, 0.1])
    ref = _oracle_keep(s, range(5), 3)
    with pytest.raises(AssertionError, match="beats a kept one"):
        check_topk_set(s, np.arange(5), ref, [0, 1, 4], eps=1.0)


def test_delta_floor_covers_scores_near_zero():
    # tau_k ~ 0: delta comes from eps (the scores' natural magnitude)
    s = np.array([2.0, 1e-9, -1e-9, -1.0])
    ref = _oracle_keep(s, range(4), 2)
    assert check_topk_set(s, np.arange(4), ref, [0, 2], eps=1.0) == 1
    with pytest.raises(AssertionError):
        check_topk_set(s, np.arange(4), ref, [0, 2], eps=1e-6)


def test_gap_just_outside_delta_is_refused():
    tau = 10.0
    d = TIE_REL * tau
    s = np.array([20.0, tau, tau - 1.01 * d, 0.0])
    ref = _oracle_keep(s, range(4), 2)
    with pytest.raises(AssertionError, match="boundary gap"):
        check_topk_set(s, np.arange(4), ref, [0, 2], eps=0.0)


def test_count_and_candidate_checks():
    s = np.array([3.0, 2.0, 1.0, 0.0])
    with pytest.raises(AssertionError, match="kept"):
        check_topk_set(s, np.arange(1, 3), [1], [1, 2], eps=1.0)
    with pytest.raises(AssertionError, match="non-candidate"):
        check_topk_set(s, np.arange(1, 3), [1], [0], eps=1.0)
    with pytest.raises(AssertionError, match="duplicate"):
        check_topk_set(s, np.arange(4), [0, 1], [0, 0], eps=1.0)


def test_every_candidate_kept_must_match():
    s = np.array([1.0, 2.0])
    assert check_topk_set(s, np.arange(2), [0, 1], [1, 0], eps=1.0) == 0
    assert boundary(s, np.arange(2), 2)[1] is None


def test_random_planted_swaps():
    """Random score rows: swapping the k-th and (k+1)-th best passes exactly
    when their gap is within delta."""
    rng = np.random.default_rng(0)
    for trial in range(200):
        n = int(rng.integers(4, 60))
        k = int(rng.integers(1, n))
        s = rng.normal(size=n)
        gap = float(rng.choice([0.0, 0.3, 0.9, 1.1, 5.0]))
        order = np.argsort(-s, kind="stable")
        tau_k = abs(s[order[k - 1]])
        eps = 1.0
        delta = TIE_REL * max(tau_k, eps, abs(s[order[k]]))
        s[order[k]] = s[order[k - 1]] - gap * delta
        if gap * delta > 0 and k + 1 < n:
            # keep the (k+2)-th clearly below
            s[order[k + 1:]] = np.minimum(s[order[k + 1:]], s[order[k]] - 10 * delta)
        ref = _oracle_keep(s, range(n), k)
        a, b = order[k - 1], order[k]
        if a not in ref or b in ref:
            continue
        swapped = sorted((set(ref) - {int(a)}) | {int(b)})
        delta = TIE_REL * max(abs(s[a]), abs(s[b]), eps)
        if s[a] - s[b] <= delta:
            assert check_topk_set(s, np.arange(n), ref, swapped, eps) == 1
        else:
            with pytest.raises(AssertionError):
                check_topk_set(s, np.arange(n), ref, swapped, eps)


def test_block_selection_check_on_an_oracle_pair():
    """check_selection (the block path's use of the rule) on a real oracle
    pair, no GPU: the oracle's own set passes; dropping a forced block, a
    swap across the widest boundary gap, and an unsorted set are refused."""
    from types import SimpleNamespace

    import kin_inputs as ki
    from kin_testlib import PairRef, check_selection, oracle_pair

    w = ki.Workload("tiecheck", 1, 1, 4, 128, 16, 0, 0, 8, 7, Lcap=512, lens=(500,))
    lens, _, hh = ki.case_meta(w)
    dc = SimpleNamespace(w=w, hh=hh, lens_final=lens, q_host=ki.fill_q(w.seed, w.B, w.Hq, w.D))
    ref = oracle_pair(dc, 0, 0, w.k)
    nb = ref.means.shape[0]
    sel = ref.sel.copy()
    assert check_selection(dc, 0, 0, w.k, ref, sel, ref.cnt) is True
    # replace the lowest-scoring kept non-forced block by the best left-out one
    kept = [int(i) for i in sel[:ref.cnt] if i not in (0, nb - 1)]
    left = [i for i in range(1, nb - 1) if i not in kept]
    worst = min(kept, key=lambda i: ref.scores[i])
    best = max(left, key=lambda i: ref.scores[i])
    assert ref.scores[worst] - ref.scores[best] > 1e-3   # a real gap on this seed
    bad = np.array(sorted(set(sel[:ref.cnt].tolist()) - {worst} | {best}), dtype=np.int32)
    with pytest.raises(AssertionError, match="boundary gap"):
        check_selection(dc, 0, 0, w.k, ref, bad, ref.cnt)
    # the same swap passes once the two scores are made a near tie
    s2 = ref.scores.copy()
    s2[best] = s2[worst] - 1e-9
    ref2 = PairRef(ref.means, s2, ref.sel, ref.cnt, ref.K, ref.V, ref.L)
    assert check_selection(dc, 0, 0, w.k, ref2, bad, ref.cnt) is False
    no_last = np.array(sorted(set(sel[:ref.cnt].tolist()) - {nb - 1} | {best}), dtype=np.int32)
    with pytest.raises(AssertionError, match="forced"):
        check_selection(dc, 0, 0, w.k, ref, no_last, ref.cnt)
    with pytest.raises(AssertionError, match="ascending"):
        check_selection(dc, 0, 0, w.k, ref, sel[::-1].copy(), ref.cnt)
