"""fp64 CPU oracle for block top-k sparse decode attention (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product library never calls it.
It wraps ``kin_oracle.c`` (plain C, fp64, OpenMP over (batch, kv head) pairs),
which shares no code with the CUDA library.

Every function takes bf16 inputs as ``np.uint16`` bit patterns, exactly as the
GPU path receives them, and widens them exactly to double.

Parity pins: see tests/test_oracle_pins.py.  Every function here is pinned by
at least one check that does not restate its own formula (dense attention
from a library routine, brute-force subset search, one-hot V weights against
scipy's softmax, per-token logits averaged per block, chunked LSE merges,
incremental vs from-scratch means).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "libkin_oracle.so")
SRC = os.path.join(_HERE, "kin_oracle.c")


def build(verbose: bool = False, src: str = SRC, out: str = LIB) -> None:
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fvisibility=hidden",
           src, "-o", out, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


_lib = None


def _L():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
            build()
        _lib = load(LIB)
    return _lib


def load(path: str):
    """Load an oracle library build (the default one, or a test's variant) and declare its C signatures."""
    lib = ctypes.CDLL(path)
    vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    lib.kin_oracle_block_means.argtypes = [vp, i32, i32, i32, vp]
    lib.kin_oracle_block_scores.argtypes = [vp, i32, vp, i32, i32, vp]
    lib.kin_oracle_select.argtypes = [vp, i32, i32, vp]
    lib.kin_oracle_select.restype = i32
    lib.kin_oracle_attend_partial.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp, i32, dbl, vp, vp, vp]
    lib.kin_oracle_merge.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
    lib.kin_oracle_attend.argtypes = [vp, i32, vp, vp, i32, i32, i32, vp, i32, dbl, vp, vp]
    lib.kin_oracle_means_update.argtypes = [vp, vp, i32, i32, vp, vp, i32, i32, vp]
    lib.kin_oracle_decode_pairs.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                            vp, i32, dbl, vp, i32, vp, vp, vp, vp, vp, i32]
    lib.kin_oracle_decode_pairs.restype = i32
    return lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def block_means(K: np.ndarray, L: int, bs: int) -> np.ndarray:
    """K [>=L, D] bf16 bits -> means [ceil(L/bs), D] fp64 over valid rows."""
    K = _c(K, np.uint16)
    D = K.shape[-1]
    nb = -(-L // bs)
    out = np.zeros((nb, D), dtype=np.float64)
    _L().kin_oracle_block_means(_p(K), L, D, bs, _p(out))
    return out


def block_scores(q_group: np.ndarray, means: np.ndarray) -> np.ndarray:
    """q_group [g, D] bf16 bits, means [nb, D] fp64 -> scores [nb] (scale 1/sqrt(D))."""
    q = _c(q_group, np.uint16)
    m = _c(means, np.float64)
    g, D = q.shape
    out = np.zeros(m.shape[0], dtype=np.float64)
    _L().kin_oracle_block_scores(_p(q), g, _p(m), m.shape[0], D, _p(out))
    return out


def select(scores: np.ndarray, k: int):
    """-> (sel [k] int32 ascending, -1 padded; count).  count -1: k < 2 < nb."""
    s = _c(scores, np.float64)
    sel = np.full(max(k, 1), -1, dtype=np.int32)
    c = _L().kin_oracle_select(_p(s), s.shape[0], k, _p(sel))
    return sel[:k], c


def attend_partial(q_group, K, V, L, bs, blocks, scale):
    q = _c(q_group, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    blk = _c(blocks, np.int32)
    g, D = q.shape
    o = np.zeros((g, D), dtype=np.float64)
    m = np.zeros(g, dtype=np.float64)
    l = np.zeros(g, dtype=np.float64)
    _L().kin_oracle_attend_partial(_p(q), g, _p(K), _p(V), L, D, bs, _p(blk), blk.shape[0],
                                   float(scale), _p(o), _p(m), _p(l))
    return o, m, l


def merge(o_parts, m_parts, l_parts):
    o = _c(o_parts, np.float64)
    m = _c(m_parts, np.float64)
    l = _c(l_parts, np.float64)
    n, g, D = o.shape
    out = np.zeros((g, D), dtype=np.float64)
    lse = np.zeros(g, dtype=np.float64)
    _L().kin_oracle_merge(n, g, D, _p(o), _p(m), _p(l), _p(out), _p(lse))
    return out, lse


def attend(q_group, K, V, L, bs, blocks, scale):
    q = _c(q_group, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    blk = _c(blocks, np.int32)
    g, D = q.shape
    out = np.zeros((g, D), dtype=np.float64)
    lse = np.zeros(g, dtype=np.float64)
    _L().kin_oracle_attend(_p(q), g, _p(K), _p(V), L, D, bs, _p(blk), blk.shape[0],
                           float(scale), _p(out), _p(lse))
    return out, lse


def means_update(Kc, Vc, L0, knew, vnew, bs, means):
    """In place on Kc, Vc [Lcap, D] (uint16) and means [nbcap, D] (fp64)."""
    assert Kc.flags["C_CONTIGUOUS"] and Vc.flags["C_CONTIGUOUS"] and means.flags["C_CONTIGUOUS"]
    kn = _c(knew, np.uint16)
    vn = _c(vnew, np.uint16)
    n, D = kn.shape
    _L().kin_oracle_means_update(_p(Kc), _p(Vc), L0, n, _p(kn), _p(vn), D, bs, _p(means))


def decode_pairs(*, Hkv, Hq, bs, seq_lens, q, Kc, Vc, means, k, scale, pairs, threads=0,
                 want_scores=False):
    """One decode step (scores, select, attend) for the listed (b*Hkv+h) pairs.

    q [B,Hq,D]; Kc, Vc [B,Hkv,Lcap,D] (or any array whose pair p rows are at
    [p]); means [B,Hkv,nbcap,D] fp64.  Returns dict(sel, cnt, out, lse[, scores]).
    """
    q = _c(q, np.uint16)
    Kc = _c(Kc, np.uint16)
    Vc = _c(Vc, np.uint16)
    means = _c(means, np.float64)
    lens = _c(seq_lens, np.int32)
    pairs = _c(pairs, np.int32)
    B, _, D = q.shape
    Lcap = Kc.shape[-2]
    nbcap = means.shape[-2]
    g = Hq // Hkv
    n = pairs.shape[0]
    sel = np.full((n, k), -1, dtype=np.int32)
    cnt = np.zeros(n, dtype=np.int32)
    out = np.zeros((n, g, D), dtype=np.float64)
    lse = np.zeros((n, g), dtype=np.float64)
    sc = np.zeros((n, nbcap), dtype=np.float64) if want_scores else None
    rc = _L().kin_oracle_decode_pairs(B, Hkv, Hq, D, bs, Lcap, nbcap, _p(lens), _p(q), _p(Kc),
                                      _p(Vc), _p(means), k, float(scale), _p(pairs), n, _p(sel),
                                      _p(cnt), _p(out), _p(lse), _p(sc) if sc is not None else None,
                                      threads)
    if rc != 0:
        raise ValueError("oracle: budget k < 2 with more blocks than k")
    res = dict(sel=sel, cnt=cnt, out=out, lse=lse)
    if sc is not None:
        res["scores"] = sc
    return res


def gather_paged(pages: np.ndarray, table_row: np.ndarray, L: int, bs: int, h: int) -> np.ndarray:
    """Logical rows [L, D] of KV head h of one sequence held in a page pool.

    pages [num_pages, Hkv, bs, D]; table_row [>= ceil(L / bs)]: token t lives
    in page table_row[t // bs] at row t % bs.  A paged KV cache stores a
    ragged batch in fixed-size pages ("Kinetics: Rethinking Test-Time Scaling
    Law", response Q3); here the page is one KV block.  Plain indexing, no
    arithmetic: attention over a paged cache is the oracle's attention over
    the rows this returns.
    """
    nb = -(-L // bs)
    blocks = [pages[int(table_row[i]), h] for i in range(nb)]
    return np.concatenate(blocks, axis=0)[:L] if nb else pages[:0, h].reshape(0, pages.shape[-1])


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Values rounded to bfloat16 precision (8 significant bits, ties to even)
    and returned as float64: x = m 2^e with 0.5 <= |m| < 1, m rounded to a
    multiple of 2^-8.  The bf16-means variant of the select keeps each block
    mean at this precision (block means of "Kinetics: Memory-Aware Test-Time
    Scaling", Implementation, stored in half the bytes).  Inputs are finite
    and within bf16's normal range."""
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def block_means_bf16(K: np.ndarray, L: int, bs: int) -> np.ndarray:
    """block_means rounded to bf16 precision (fp64 array)."""
    return round_bf16(block_means(K, L, bs))


def token_topk_attend(q_group: np.ndarray, K: np.ndarray, V: np.ndarray, L: int, k_tokens: int, scale: float):
    """Token-level TopK attention for each query head of one group, in fp64:
    the logits z_t = scale q_j . K_t of every token t < L, the k_tokens tokens
    with the largest z_t (ties to the lower index; every token when
    k_tokens >= L), then softmax over those tokens and the weighted sum of
    their V rows.  TopK attention keeps the keys and values with the highest
    attention scores ("Kinetics: Rethinking Test-Time Scaling Law", response
    Q2, Fig. 8's variant; MagicPIG's abstract on the same pages).
    q_group [g, D], K, V [>= L, D] as bf16 bits.  Returns (sel [g, min(k, L)]
    ascending, out [g, D], lse [g], z [g, L])."""
    q = bf16_bits_to_f64(q_group)
    Kf = bf16_bits_to_f64(np.asarray(K)[:L])
    Vf = bf16_bits_to_f64(np.asarray(V)[:L])
    z = scale * (q @ Kf.T)                         # [g, L]
    n = min(k_tokens, L)
    sels, outs, lses = [], [], []
    for j in range(z.shape[0]):
        order = np.lexsort((np.arange(L), -z[j]))  # z descending, index ascending
        s = np.sort(order[:n])
        zs = z[j, s]
        m = zs.max()
        w = np.exp(zs - m)
        outs.append((w[:, None] * Vf[s]).sum(axis=0) / w.sum())
        lses.append(m + np.log(w.sum()))
        sels.append(s)
    return np.array(sels), np.array(outs), np.array(lses), z


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) widened exactly to fp64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
