"""Helpers shared by the GPU parity tests: build a seeded case on the device,
run the CUDA path through the C ABI binding, and compare with the fp64 oracle
on the same bf16 bits (regenerated on the host for any (batch, kv head)).

Tolerances (from the arithmetic: bf16 inputs, fp32 accumulation, bf16 out):
  * outputs: max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3;
  * lse: |gpu - oracle| <= 1e-3 + 1e-4 |oracle|;
  * block means: |gpu - oracle| <= 1e-5 (fp32 sums of <= 128 bf16 rows);
  * selected indices: bit-exact, except where the oracle's k-th and (k+1)-th
    best scores are within delta = 1e-4 * max(|tau_k|, |tau_k+1|, eps) of each
    other (eps: the mean over blocks of (1/sqrt(D)) sum_j sum_d |q_jd| |m_d|,
    the scores' natural magnitude); there the GPU set may differ only as a
    top set of scores perturbed by at most delta (kin_tiecheck).  When sets
    differ, the output is compared with the oracle recomputed on the GPU's
    set.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

import block_top_sparse_kin_b200 as kin
import kin_inputs as ki
import oracle
from kin_tiecheck import check_topk_set

D = 128
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
MEANS_ABS = 1e-5


@dataclass
class DeviceCase:
    w: ki.Workload
    dims: kin.kin_dims
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    means: torch.Tensor
    seq_lens: torch.Tensor       # device, pre-append lengths (updated in place by append)
    lens_pre: np.ndarray
    lens_final: np.ndarray
    hh: np.ndarray
    q_host: np.ndarray
    k_new: torch.Tensor | None
    v_new: torch.Tensor | None


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def make_device_case(w: ki.Workload, poison: bool = True) -> DeviceCase:
    lens_final, lens_pre, hh = ki.case_meta(w)
    q_host = ki.fill_q(w.seed, w.B, w.Hq, w.D)
    dims = kin.make_dims(w.B, w.Hkv, w.Hq, w.D, w.bs, w.cap)
    seq = torch.from_numpy(lens_pre.copy()).cuda()
    hh_dev = torch.from_numpy(hh).cuda()
    kc = torch.empty((w.B, w.Hkv, w.cap, w.D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    ki.kv_cache_device(w.seed, True, w.B, w.Hkv, w.cap, w.D, w.bs, seq, hh_dev, poison, kc)
    ki.kv_cache_device(w.seed, False, w.B, w.Hkv, w.cap, w.D, w.bs, seq, hh_dev, poison, vc)
    means = torch.full((w.B, w.Hkv, w.nbcap, w.D), float("nan"), dtype=torch.float32, device="cuda")
    kn = vn = None
    if w.n_append:
        kn_h = np.empty((w.B, w.Hkv, w.n_append, w.D), np.uint16)
        vn_h = np.empty_like(kn_h)
        for b in range(w.B):
            for h in range(w.Hkv):
                t0 = int(lens_pre[b])
                kn_h[b, h] = ki.kv_rows(w.seed, True, b * w.Hkv + h, t0, t0 + w.n_append, w.D, w.bs, hh[b, h])
                vn_h[b, h] = ki.kv_rows(w.seed, False, b * w.Hkv + h, t0, t0 + w.n_append, w.D, w.bs, None)
        kn, vn = to_dev_bf16(kn_h), to_dev_bf16(vn_h)
    return DeviceCase(w, dims, to_dev_bf16(q_host), kc, vc, means, seq, lens_pre, lens_final, hh, q_host, kn, vn)


@dataclass
class GpuResult:
    sel: np.ndarray
    cnt: np.ndarray
    out: np.ndarray     # float32 [B,Hq,D]
    lse: np.ndarray
    status: int


def gpu_step(dc: DeviceCase, k: int, ws: torch.Tensor | None = None, build_means: bool = True,
             scale: float = 0.0) -> GpuResult:
    """Means (build, then append if the workload has one), select, attend
    (softmax scale: 0 = the default 1/sqrt(D))."""
    w = dc.w
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if build_means:
        kin.kin_block_means_build(dc.dims, dc.k_cache, dc.seq_lens, dc.means, st)
        if w.n_append:
            kin.kin_block_means_update(dc.dims, dc.k_cache, dc.v_cache, dc.means, dc.seq_lens,
                                       dc.k_new, dc.v_new, w.n_append, st)
    if ws is None:
        ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    kin.kin_block_topk_select(dc.dims, dc.q, dc.means, dc.seq_lens, k, sel, cnt, ws, st)
    kin.kin_sparse_decode_attn(dc.dims, dc.q, dc.k_cache, dc.v_cache, dc.seq_lens, sel, cnt, k, scale,
                               out, lse, ws, st)
    torch.cuda.synchronize()
    return GpuResult(sel.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy(),
                     lse.cpu().numpy(), int(st.item()))


@dataclass
class PairRef:
    means: np.ndarray
    scores: np.ndarray
    sel: np.ndarray
    cnt: int
    K: np.ndarray
    V: np.ndarray
    L: int


def oracle_pair(dc: DeviceCase, b: int, h: int, k: int, bf16_means: bool = False, rows=None) -> PairRef:
    """The oracle's means, scores, selection and the K/V rows of one (b, h);
    rows: the pair's (K, V) when the caller regenerated them already."""
    w = dc.w
    L = int(dc.lens_final[b])
    K, V = rows if rows is not None else ki.pair_rows(w, dc.hh, b, h, L)
    means = oracle.block_means_bf16(K, L, w.bs) if bf16_means else oracle.block_means(K, L, w.bs)
    qg = dc.q_host[b, h * w.g:(h + 1) * w.g]
    scores = oracle.block_scores(qg, means)
    sel, cnt = oracle.select(scores, k)
    return PairRef(means, scores, sel, cnt, K, V, L)


def score_eps(dc: DeviceCase, b: int, h: int, means: np.ndarray) -> float:
    """The block scores' natural magnitude: the mean over blocks of
    (1/sqrt(D)) sum_j sum_d |q_jd| |m_d| (the floor of the tie tolerance)."""
    w = dc.w
    qg = ki.bf16_to_f32(dc.q_host[b, h * w.g:(h + 1) * w.g]).astype(np.float64)
    return float((np.abs(qg).sum(axis=0) @ np.abs(means).T).mean() / math.sqrt(D))


def check_selection(dc: DeviceCase, b: int, h: int, k: int, ref: PairRef, gsel: np.ndarray, gcnt: int):
    """Returns True if identical, False if an allowed near-tie swap; raises
    otherwise.  The forced first and last blocks must be kept; the other
    kept blocks follow the near-tie rule of kin_tiecheck."""
    nb = ref.means.shape[0]
    assert gcnt == ref.cnt, (b, h, gcnt, ref.cnt)
    assert np.all(gsel[gcnt:] == -1), (b, h)
    g = gsel[:gcnt]
    assert np.all(np.diff(g) > 0), (b, h, "not ascending")
    assert np.all((g >= 0) & (g < nb)), (b, h, "block index out of range")
    forced = {0, nb - 1}
    assert forced <= set(g.tolist()), (b, h, "forced blocks missing")
    cand = np.arange(1, nb - 1)
    r = ref.sel[:ref.cnt]
    n = check_topk_set(ref.scores, cand, [i for i in r if i not in forced], [i for i in g if i not in forced],
                       score_eps(dc, b, h, ref.means), what=(b, h))
    return n == 0


def check_pair(dc: DeviceCase, gr: GpuResult, b: int, h: int, k: int, gpu_means: np.ndarray | None = None,
               bf16_means: bool = False, rows=None, scale: float = 0.0):
    """Full parity of one (b, h): means, selection, outputs, lse (softmax
    scale as passed to the attention: 0 = the default 1/sqrt(D)).  With
    bf16_means the oracle scores blocks from its means rounded to bf16, and
    GPU means may differ from them by one bf16 step (the GPU rounds its fp32
    mean, the oracle its fp64 mean)."""
    w = dc.w
    ref = oracle_pair(dc, b, h, k, bf16_means, rows)
    nb = ref.means.shape[0]
    if gpu_means is not None:
        gm = gpu_means[b, h, :nb].astype(np.float64)
        if bf16_means:
            step = np.ldexp(1.0, np.frexp(np.maximum(np.abs(ref.means), 1e-30))[1] - 8)
            assert np.all(np.abs(gm - ref.means) <= step), (b, h)
            assert np.mean(gm != ref.means) < 1e-3, (b, h)
        else:
            err = np.abs(gm - ref.means).max()
            assert err <= MEANS_ABS, (b, h, err)
    same = check_selection(dc, b, h, k, ref, gr.sel[b, h], int(gr.cnt[b, h]))
    blocks = gr.sel[b, h, :gr.cnt[b, h]] if not same else ref.sel[:ref.cnt]
    qg = dc.q_host[b, h * w.g:(h + 1) * w.g]
    o_ref, lse_ref = oracle.attend(qg, ref.K, ref.V, ref.L, w.bs, blocks, scale if scale > 0 else 1 / math.sqrt(D))
    o_gpu = gr.out[b, h * w.g:(h + 1) * w.g].astype(np.float64)
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (b, h, err.max(), err.mean())
    lse_gpu = gr.lse[b, h * w.g:(h + 1) * w.g].astype(np.float64)
    assert np.all(np.abs(lse_gpu - lse_ref) <= 1e-3 + 1e-4 * np.abs(lse_ref)), (b, h, lse_gpu, lse_ref)
    return same, err.max(), err.mean()


def all_pairs(w: ki.Workload):
    return [(b, h) for b in range(w.B) for h in range(w.Hkv)]


def check_pairs(dc: DeviceCase, results, pairs, gpu_means: np.ndarray | None = None, bf16_means: bool = False) -> int:
    """check_pair on every listed (b, h) for every (k, GpuResult) in results
    (one GPU step per budget on the same case), on a pool of host threads:
    each pair's K/V rows are regenerated once and serve every budget (the
    generator and the oracle are C calls that release the GIL).  gpu_means
    is checked with the first result.  Returns how many (pair, budget)
    selections were accepted near ties; any failure raises."""
    def one(bh):
        b, h = bh
        rows = ki.pair_rows(dc.w, dc.hh, b, h, int(dc.lens_final[b]))
        n = 0
        for i, (k, gr) in enumerate(results):
            same, _, _ = check_pair(dc, gr, b, h, k, gpu_means if i == 0 else None, bf16_means, rows)
            n += not same
        return n
    with ThreadPoolExecutor(max(1, os.cpu_count() or 1)) as ex:
        return sum(ex.map(one, pairs))


# ------------------------------------------------------------- paged KV cache
@dataclass
class Pages:
    k: torch.Tensor          # [num_pages, Hkv, bs, D] bf16
    v: torch.Tensor
    table: torch.Tensor      # [B, nbcap] int32 (device); -1 where unmapped
    table_host: np.ndarray
    num_pages: int


def to_pages(dc: DeviceCase, seed: int = 0, spare: int = 3) -> Pages:
    """The case's (pre-append) contiguous cache copied into a shuffled page
    pool: every block a sequence will hold after its append gets a page, in a
    random order, plus `spare` unused pages; unused rows are NaN."""
    w = dc.w
    B, Hkv, cap, D = dc.k_cache.shape
    bs, nbcap = w.bs, w.nbcap
    nbs = [-(-int(L) // bs) for L in dc.lens_final]
    total = sum(nbs)
    P = total + spare
    order = np.random.default_rng(seed).permutation(P)
    table = np.full((B, nbcap), -1, np.int32)
    j = 0
    for b in range(B):
        for i in range(nbs[b]):
            table[b, i] = order[j]
            j += 1
    ib, ii = np.nonzero(table >= 0)
    dst = torch.from_numpy(table[ib, ii].astype(np.int64)).cuda()
    tb, ti = torch.from_numpy(ib).cuda(), torch.from_numpy(ii).cuda()
    pools = []
    for cache in (dc.k_cache, dc.v_cache):
        padded = torch.nn.functional.pad(cache, (0, 0, 0, nbcap * bs - cap))
        blocks = padded.view(B, Hkv, nbcap, bs, D)
        pool = torch.full((P, Hkv, bs, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        pool[dst] = blocks[tb, :, ti]
        pools.append(pool)
    return Pages(pools[0], pools[1], torch.from_numpy(table).cuda(), table, P)


def gpu_step_paged(dc: DeviceCase, pg: Pages, k: int, seq_lens: torch.Tensor, means: torch.Tensor,
                   ws: torch.Tensor | None = None) -> GpuResult:
    """The paged path: means build (+ append), select, attention over pages."""
    w = dc.w
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kin.kin_block_means_build_paged(dc.dims, pg.k, pg.table, seq_lens, means, st)
    if w.n_append:
        kin.kin_block_means_update_paged(dc.dims, pg.k, pg.v, pg.table, means, seq_lens, dc.k_new, dc.v_new,
                                         w.n_append, st)
    if ws is None:
        ws = kin.alloc_workspace(dc.dims, k)
    sel = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    kin.kin_block_topk_select(dc.dims, dc.q, means, seq_lens, k, sel, cnt, ws, st)
    kin.kin_sparse_decode_attn_paged(dc.dims, dc.q, pg.k, pg.v, pg.table, seq_lens, sel, cnt, k, 0.0, out, lse,
                                     ws, st)
    torch.cuda.synchronize()
    return GpuResult(sel.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(),
                     int(st.item()))


def random_shapes(n, seed, prefix="rand"):
    """n seeded random workloads: block size 16-128, g 1-8, 1-4 KV heads, batch 1-4, capacity up to
    20000 tokens, appends of 0, 1 or 5 tokens, k from 2 to a little beyond the block capacity."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        bs = int(rng.choice([16, 32, 64, 128]))
        g = int(rng.integers(1, 9))
        Hkv = int(rng.integers(1, 5))
        B = int(rng.integers(1, 5))
        n_append = int(rng.choice([0, 0, 1, 5]))
        Lcap = int(rng.integers(bs, 20000))
        lens = tuple(int(x) for x in rng.integers(1, Lcap - n_append + 1, size=B))
        nbcap = -(-Lcap // bs)
        k = int(rng.integers(2, nbcap + 3))
        out.append(ki.Workload(f"{prefix}{i}_bs{bs}_g{g}_k{k}", B, Hkv, Hkv * g, D, bs, 0, 0, k, 200 + i, Lcap=Lcap,
                               lens=tuple(L + n_append for L in lens), n_append=n_append))
    return out
