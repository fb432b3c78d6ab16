"""The index rule for comparing a GPU top-k selection with the oracle's.

A top-k set is an integer result: it must equal the oracle's exactly, with
one exception.  Where the oracle's k-th and (k+1)-th best scores lie within
delta of each other (delta = 1e-4 relative, with a floor at the scores'
natural magnitude), fp32 rounding on the GPU may legitimately order the
near-tied items the other way.  So a GPU set that differs is accepted only
when

  1. the oracle's boundary itself is a near tie: tau_k - tau_{k+1} <= delta;
  2. the GPU set is a top set of the oracle scores perturbed by at most
     delta: no candidate the GPU left out beats a candidate it kept by more
     than delta (in particular every dropped oracle item scores within delta
     of every added GPU item).

Both the block select (candidates = every block but the forced first and
last) and the token-level top-k (candidates = every token) use this rule.
Pure numpy, so the rule itself is pinned by CPU tests.

Every accepted difference is recorded, per test, so the session summary can
say how often the near-tie branch was taken.
"""
from __future__ import annotations

import os
import threading
from collections import defaultdict

import numpy as np

TIE_REL = 1e-4

# test id -> [items compared, items whose GPU set differed (accepted near ties)]
TALLY = defaultdict(lambda: [0, 0])
_LOCK = threading.Lock()  # the parity tests check pairs on a thread pool


def tie_delta(tau_k: float, tau_k1: float, eps: float) -> float:
    """delta = 1e-4 max(|tau_k|, |tau_k+1|, eps)."""
    return TIE_REL * max(abs(tau_k), abs(tau_k1), eps)


def boundary(scores: np.ndarray, cand: np.ndarray, n_keep: int):
    """The k-th and (k+1)-th largest candidate scores (tau_k, tau_k+1); the
    (k+1)-th is None when every candidate is kept."""
    s = np.sort(np.asarray(scores, dtype=np.float64)[cand])[::-1]
    tau_k = float(s[n_keep - 1]) if n_keep >= 1 else float("inf")
    tau_k1 = float(s[n_keep]) if n_keep < len(s) else None
    return tau_k, tau_k1


def check_topk_set(scores, cand, ref_keep, gpu_keep, eps: float, what=()) -> int:
    """Compare the candidates a GPU kept with the ones the oracle kept.

    scores: oracle scores (fp64) indexed by item; cand: the candidate items
    (forced items excluded); ref_keep / gpu_keep: the kept candidates of the
    oracle and of the GPU; eps: the scores' natural magnitude (delta's floor).
    Returns 0 when the sets are equal, else the number of swapped items;
    raises AssertionError when the difference is not an allowed near tie.
    """
    scores = np.asarray(scores, dtype=np.float64)
    cand = np.asarray(cand, dtype=np.int64)
    ref = set(int(i) for i in ref_keep)
    gpu = set(int(i) for i in gpu_keep)
    cset = set(cand.tolist())
    assert len(gpu) == len(gpu_keep), (*what, "duplicate items in the GPU set")
    assert gpu <= cset, (*what, "GPU kept a non-candidate", sorted(gpu - cset)[:8])
    assert len(gpu) == len(ref), (*what, "GPU kept", len(gpu), "items, oracle", len(ref))
    _record(True, False)
    if gpu == ref:
        return 0
    tau_k, tau_k1 = boundary(scores, cand, len(ref))
    assert tau_k1 is not None, (*what, "every candidate is kept, yet the sets differ")
    delta = tie_delta(tau_k, tau_k1, eps)
    gap = tau_k - tau_k1
    assert gap <= delta, (*what, "sets differ across a boundary gap wider than the tie tolerance",
                          tau_k, tau_k1, gap, delta)
    kept = np.array(sorted(gpu), dtype=np.int64)
    left = np.array(sorted(cset - gpu), dtype=np.int64)
    worst_kept = scores[kept].min()
    best_left = scores[left].max()
    assert best_left - worst_kept <= delta, (*what, "GPU left out an item that beats a kept one by more than delta",
                                            int(left[scores[left].argmax()]), best_left,
                                            int(kept[scores[kept].argmin()]), worst_kept, delta)
    _record(False, True)
    return len(gpu - ref)


def _record(compared: bool, differed: bool) -> None:
    key = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    with _LOCK:
        t = TALLY[key]
        if compared:
            t[0] += 1
        if differed:
            t[1] += 1
