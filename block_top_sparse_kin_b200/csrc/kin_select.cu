// kin_select.cu -- group-summed block scores (HBM scan of the fp32 block
// means) followed by an exact per-(batch, kv-head) block top-k.
//
// Method: block-level top-k sparsity ("Kinetics: Memory-Aware Test-Time
// Scaling", Architecture Overview; Implementation, BlockTopKAttention: scores
// scaled by 1/sqrt(head_dim), top-k over per-block summaries) under a KV
// budget counted in blocks ("Kinetics: Rethinking Test-Time Scaling Law",
// response Q4).  The group score uses linearity: sum_j q_j . m_i =
// (sum_j q_j) . m_i, so each block costs one 128-wide dot product.
//
// Two kernels, the second launched with programmatic dependent launch:
//  1. select_scan_kernel streams every block mean once: the (pair, block)
//     rows are cut into one contiguous, pair-aligned range per warp; a warp
//     reads one 512-byte mean row per load (lane l owns dims 4l..4l+3) and
//     keeps the next 8 rows in flight while reducing the current 8, with a
//     butterfly that halves the rows per lane at each level (8 rows in 9
//     shuffles).  Scores go to workspace, where they stay in L2.
//  2. select_topk_kernel, one CTA per pair (256, 512 or 1024 threads, so
//     that each thread holds 4 of a 4096-block pair's keys), turns the
//     pair's scores into order-preserving uint32 keys, finds the exact
//     threshold (equal-width score bins, then a pairwise rank of the
//     boundary bin; a radix search over the key bits when the range is
//     crowded or degenerate) and writes the kept indices.  Rows too long
//     for registers keep their keys in shared memory (or a scratch row):
//     there the bin pass is fused with the emit's per-lane bit masks, and a
//     crowded boundary bin is ranked through its 256 sub-bins.
// The top-k: the first block and the block holding the newest token are
// always kept, ties go to the lower index, and the kept indices leave
// ascending.  A budget that covers every block the dims allow (k >= nbcap)
// skips both: select_dense_kernel writes the selections directly.
//
// Variants served by the same code: bf16 block means (the scan templated on
// the means type, 16 rows per warp step); block means stored per page of a
// paged cache (select_scan_paged_kernel: 8-lane groups own one scattered
// row each, with the same summation tree, so the scores are bit-identical);
// and the token-level top-k of every query head's logits
// (token_topk_kernel: the same threshold search over an explicit candidate
// range with nothing forced).
#include <type_traits>

#include "kin_internal.cuh"

namespace kin {

#ifndef KIN_SEL_UNROLL
#define KIN_SEL_UNROLL 8
#endif
#ifndef KIN_SEL_CTAS_PER_SM
#define KIN_SEL_CTAS_PER_SM 2
#endif
#ifndef KIN_DUAL_SCAN_V
#define KIN_DUAL_SCAN_V 8  // 16-byte loads per lane per step of the dual-means scan
#endif
#ifndef KIN_DUAL_SCAN_CTAS
#define KIN_DUAL_SCAN_CTAS 2  // its resident CTAs per SM
#endif

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelU = KIN_SEL_UNROLL;  // mean rows per warp per step

// Sums U per-lane partials (one per mean row) over the warp with
// U + 4 - log2(U) shuffles instead of 5 U: each butterfly level halves the
// rows a lane keeps.  Afterwards lane l holds the total of row l >> (5 - log2 U).
template <int U>
__device__ __forceinline__ float warp_sum_rows(float (&v)[U], int lane) {
  constexpr int kLog = U == 1 ? 0 : U == 2 ? 1 : U == 4 ? 2 : U == 8 ? 3 : 4;
  static_assert((1 << kLog) == U && U <= 16, "U must be a power of two <= 16");
#pragma unroll
  for (int s = 0; s < kLog; ++s) {
    const int half = U >> (s + 1);
    const bool upper = (lane >> (4 - s)) & 1;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float keep = upper ? v[j + half] : v[j];
      const float send = upper ? v[j] : v[j + half];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16 >> s);
    }
  }
  float r = v[0];
#pragma unroll
  for (int off = 16 >> kLog; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}


// ------------------------------------------------------------------ top-k
// One CTA of NT threads (256, 512 or 1024, chosen from the block capacity)
// per pair.  Scores become order-preserving uint32 keys (float_key); the
// threshold is found by a search over 256 equal-width score bins, with a
// radix search over the key bits for crowded or degenerate ranges.
constexpr int kListCap = 4096;   // radix: candidates kept after the first pass
constexpr int kRankCap = 512;    // equal-width bins: most boundary-bin keys listed
constexpr int kDirectRank = 64;  // keys in memory: larger boundary bins are ranked through sub-bins
constexpr int kMaxKPT = 8;       // keys per thread on the register path
#ifndef KIN_RANK_SPLIT
#define KIN_RANK_SPLIT 1  // the refinement ranks a band of <= NT / 4 keys with four threads per key
#endif
#ifndef KIN_RESCORE_ROWS
#define KIN_RESCORE_ROWS 4  // fp32 rows in flight per warp when the register path rescores a band
#endif
// 256-bin histograms padded by one word per 8 bins, so a lane reading 8
// consecutive bins (stride 9 words between lanes) hits 32 distinct banks
constexpr int kHistWords = 256 + 32;
__device__ __forceinline__ int hidx(int bin) { return bin + (bin >> 3); }

// The candidates of a top-k over nb keys: indices lo..hi compete for kr
// slots; every other index below nb is forced (always kept).  Block select:
// lo = 1, hi = nb - 2, kr = k - 2 (the first and the newest block forced).
// Token select: lo = 0, hi = nb - 1, kr = k (nothing forced).
struct Cands {
  int lo, hi, kr;
  __device__ __forceinline__ bool has(int i) const { return i >= lo && i <= hi; }
};

template <int NT>
struct TopkSmem {
  static constexpr int NW = NT / 32;
  int hist[2][kHistWords];   // histograms (equal-width bins, or radix digits double-buffered), hidx-padded
  uint32_t list[kListCap];   // radix: candidate indices; equal-width bins: boundary-bin keys (then the deciding sub-bin's)
  int list_n, list_n2;
  int warp_cnt[2][NW];       // emit: per-warp counts of keys taken outright, and equal to the threshold
  uint32_t wmin[NW], wmax[NW];
  int digit, above, bin;
  uint32_t thresh;
  int thresh_take;
  int band_n, in_n;            // dual-means refinement: band keys listed, candidates decided in
  int slot_cnt[kMaxKPT * NW];  // register path: packed (> T, == T) counts per 32-block slot
};

// Inverse of float_key.
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Order-preserving key of the fp32 value whose bits are u.
__device__ __forceinline__ uint32_t key_of_bits(uint32_t u) {
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int NT>
__device__ __forceinline__ void zero_hist(TopkSmem<NT>& sm, int which) {
  for (int i = threadIdx.x; i < kHistWords; i += NT) sm.hist[which][i] = 0;
}

// Every lane of the calling warp gets the bin (counted from the top of a
// 256-bin histogram) holding the kr-th largest key, the count of keys in
// higher bins, and the bin's own count.  Needs 1 <= kr <= total count.
// half < 0: whole-word counts; 0 / 1: the low / high 16 bits of each word
// (two histograms packed in one).
__device__ __forceinline__ void warp_find_bin(const int* hist, int kr, int& bin, int& above, int& cnt, int half = -1) {
  const int lane = threadIdx.x & 31;
  int c[8], tot = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int v = hist[hidx(255 - (lane * 8 + u))];
    c[u] = half < 0 ? v : (v >> (16 * half)) & 0xFFFF;
    tot += c[u];
  }
  int inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  const int excl = inc - tot;
  const bool mine = excl < kr && kr <= inc;
  int b = 0, ab = 0, cn = 0, run = excl;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if (mine && cn == 0 && run + c[u] >= kr) {
      b = 255 - (lane * 8 + u);
      ab = run;
      cn = c[u];
    }
    run += c[u];
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
  bin = __shfl_sync(0xffffffffu, b, src);
  above = __shfl_sync(0xffffffffu, ab, src);
  cnt = __shfl_sync(0xffffffffu, cn, src);
}

// warp_find_bin over the two histograms packed in one word per bin (low
// and high 16 bits), both searches interleaved over one read of the bins:
// the bins holding the kr-th largest of each.  Needs 1 <= kr <= each total.
__device__ __forceinline__ void warp_find_bins_packed(const int* hist, int kr, int& bin_lo, int& bin_hi) {
  const int lane = threadIdx.x & 31;
  int c[8], tl = 0, th = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    c[u] = hist[hidx(255 - (lane * 8 + u))];
    tl += c[u] & 0xFFFF;
    th += c[u] >> 16;
  }
  int il = tl, ih = th;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, il, o), b = __shfl_up_sync(0xffffffffu, ih, o);
    if (lane >= o) {
      il += a;
      ih += b;
    }
  }
  const bool ml = il - tl < kr && kr <= il, mh = ih - th < kr && kr <= ih;
  int bl = 0, bh = 0, rl = il - tl, rh = ih - th;
  bool fl = false, fh = false;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    rl += c[u] & 0xFFFF;
    rh += c[u] >> 16;
    if (ml && !fl && rl >= kr) {
      bl = 255 - (lane * 8 + u);
      fl = true;
    }
    if (mh && !fh && rh >= kr) {
      bh = 255 - (lane * 8 + u);
      fh = true;
    }
  }
  bin_lo = __shfl_sync(0xffffffffu, bl, __ffs(__ballot_sync(0xffffffffu, ml)) - 1);
  bin_hi = __shfl_sync(0xffffffffu, bh, __ffs(__ballot_sync(0xffffffffu, mh)) - 1);
}

// Radix select over the candidate keys keys[1..nb-2]: on entry kr (> 0) is
// how many of them to keep, sm.hist[0] holds the histogram of their top
// bytes and sm.hist[1] is zero.  Up to 4 passes of 8 bits from the top: each
// pass finds the digit whose bin holds the kr-th largest remaining key.
// After the first pass the indices matching the chosen prefix go to a
// compact list, so the later passes visit only those.  A pass whose bin
// holds exactly the keys still needed ends the search: they are all taken.
// On return every key above `prefix` under `mask` is kept, and the first kr
// keys equal to it under the mask (by index).
template <int NT>
__device__ __forceinline__ void radix_threshold(const uint32_t* keys, int nb, const Cands& cd, TopkSmem<NT>& sm,
                                                uint32_t& prefix, uint32_t& mask, int& kr) {
  const int tid = threadIdx.x, lane = tid & 31;
  prefix = 0u;
  mask = 0u;
  bool use_list = false;
#pragma unroll 1
  for (int pass = 0; pass < 4 && kr > 0; ++pass) {
    const int shift = 24 - 8 * pass;
    int* hist = sm.hist[pass & 1];
    if (pass > 0) {
      if (pass == 1) {  // visit every key once more, keep the matching indices
        if (tid == 0) sm.list_n = 0;
        __syncthreads();
        for (int base = 0; base < nb; base += NT) {  // uniform trip count per warp
          const int i = base + tid;
          const uint32_t key = i < nb ? keys[i] : 0u;
          const bool match = cd.has(i) && (key & mask) == prefix;
          if (match) atomicAdd(&hist[hidx((key >> shift) & 0xFFu)], 1);
          if (use_list) {  // one list reservation per warp, lanes take slots in order
            const unsigned m = __ballot_sync(0xffffffffu, match);
            int slot = 0;
            if (lane == 0 && m) slot = atomicAdd(&sm.list_n, __popc(m));
            slot = __shfl_sync(0xffffffffu, slot, 0);
            if (match) sm.list[slot + __popc(m & ((1u << lane) - 1u))] = i;
          }
        }
      } else if (use_list) {
        for (int j = tid; j < sm.list_n; j += NT) {
          const uint32_t key = keys[sm.list[j]];
          if ((key & mask) == prefix) atomicAdd(&hist[hidx((key >> shift) & 0xFFu)], 1);
        }
      } else {
        for (int i = cd.lo + tid; i <= cd.hi; i += NT) {
          const uint32_t key = keys[i];
          if ((key & mask) == prefix) atomicAdd(&hist[hidx((key >> shift) & 0xFFu)], 1);
        }
      }
      zero_hist(sm, (pass + 1) & 1);  // the other buffer is free: ready it for the next pass
      __syncthreads();
    }
    if (tid < 32) {
      int d, a, c;
      warp_find_bin(hist, kr, d, a, c);
      if (tid == 0) {
        sm.digit = d;
        sm.above = a;
        sm.bin = c;
      }
    }
    if (pass == 0) zero_hist(sm, 1);
    __syncthreads();
    prefix |= (uint32_t)sm.digit << shift;
    mask |= 0xFFu << shift;
    kr -= sm.above;
    if (pass == 0) use_list = sm.bin <= kListCap;
    const bool done = sm.bin == kr;  // every key in the bin is taken
    __syncthreads();                 // all threads have read digit/above/bin
    if (done) break;
  }
}

// One round of the emit, every warp's range holding at most 1024 keys: lane
// l's masks cover the 32 keys from i0 (bit b = key i0 + b): gm those taken
// outright, em those equal to the threshold, of which the first kr (by
// index, over the whole row) are taken.  One barrier publishes the warp
// totals; warp scans give every lane its output position; each lane writes
// its taken indices in bit order.  Checks that exactly k were taken.
template <int NT>
__device__ __forceinline__ void emit_round(unsigned gm, unsigned em, int i0, int k, int kr, int32_t* sel,
                                           TopkSmem<NT>& sm, int32_t* dev_status) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ng = __popc(gm), ne = __popc(em);
  int ig = ng, ie = ne;  // inclusive scans over the warp's lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int tg = __shfl_up_sync(0xffffffffu, ig, o), te = __shfl_up_sync(0xffffffffu, ie, o);
    if (lane >= o) {
      ig += tg;
      ie += te;
    }
  }
  if (lane == 31) {
    sm.warp_cnt[0][warp] = ig;
    sm.warp_cnt[1][warp] = ie;
  }
  __syncthreads();
  int sg = lane < NW ? sm.warp_cnt[0][lane] : 0, se = lane < NW ? sm.warp_cnt[1][lane] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {  // inclusive scans over the warps
    const int tg = __shfl_up_sync(0xffffffffu, sg, o), te = __shfl_up_sync(0xffffffffu, se, o);
    if (lane >= o) {
      sg += tg;
      se += te;
    }
  }
  const int gb = (warp ? __shfl_sync(0xffffffffu, sg, warp - 1) : 0) + ig - ng;  // before this lane's first key
  const int eb = (warp ? __shfl_sync(0xffffffffu, se, warp - 1) : 0) + ie - ne;
  unsigned take = gm;
  for (int keep = min(max(kr - eb, 0), ne); keep > 0; --keep) {  // its first equal keys still wanted
    take |= em & (0u - em);
    em &= em - 1u;
  }
  int pos = gb + min(eb, kr);
  while (take) {
    const int b = __ffs(take) - 1;
    take &= take - 1u;
    if (pos < k) sel[pos] = i0 + b;  // never write past the pair's row
    ++pos;
  }
  const int g_all = __shfl_sync(0xffffffffu, sg, 31), e_all = __shfl_sync(0xffffffffu, se, 31);
  if (threadIdx.x == 0 && g_all + min(e_all, kr) != k) set_status(dev_status, KIN_ERR_DEVICE_DATA);
}

// Writes the kept blocks ascending to sel[0..k): the forced blocks 0 and
// nb-1, every candidate whose key under `mask` is above `prefix`, and the
// first kr candidates (by index) whose key under the mask equals it.  Warp w
// owns a contiguous index range in rounds of 1024 keys; in a round, lane l
// owns the 32 consecutive keys from 32 l and reads them in a rotated order
// (step j: key (j + l) mod 32), so the warp's 32 reads hit 32 distinct
// banks, into two 32-bit masks (taken outright; equal to the threshold).
// One round per warp goes straight to emit_round; longer ranges count every
// round first, publish the warp totals, then rebuild each round's masks and
// write (ties go to lower indices).
template <int NT>
__device__ __forceinline__ void emit_selection(const uint32_t* keys, int nb, const Cands& cd, int k, uint32_t prefix,
                                               uint32_t mask, int kr, int32_t* sel, TopkSmem<NT>& sm,
                                               int32_t* dev_status) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int span = ((nb + NW - 1) / NW + 1023) & ~1023;  // per-warp range, whole rounds
  const int w0 = min(warp * span, nb), w1 = min(w0 + span, nb);
  auto chunk_masks = [&](int c0, unsigned& gm, unsigned& em) {
    gm = 0u;
    em = 0u;
    if (c0 + 32 <= w1 && c0 >= cd.lo && c0 + 31 <= cd.hi) {  // 32 candidates
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const int b = (j + lane) & 31;
        const uint32_t key = keys[c0 + b] & mask;
        gm |= (unsigned)(key > prefix) << b;
        em |= (unsigned)(key == prefix) << b;
      }
    } else if (c0 < w1) {
      for (int j = 0; j < 32; ++j) {
        const int b = (j + lane) & 31;
        const int i = c0 + b;
        if (i < w1) {
          const uint32_t key = keys[i] & mask;
          const bool cand = cd.has(i);
          gm |= (unsigned)(!cand || key > prefix) << b;
          em |= (unsigned)(cand && key == prefix) << b;
        }
      }
    }
  };
  if (span <= 1024) {  // CTA-uniform
    unsigned gm, em;
    chunk_masks(w0 + 32 * lane, gm, em);
    emit_round(gm, em, w0 + 32 * lane, k, kr, sel, sm, dev_status);
    return;
  }
  int n_g = 0, n_e = 0;
  for (int c = w0; c < w1; c += 1024) {
    unsigned gm, em;
    chunk_masks(c + 32 * lane, gm, em);
    n_g += __popc(gm);
    n_e += __popc(em);
  }
  n_g = __reduce_add_sync(0xffffffffu, n_g);
  n_e = __reduce_add_sync(0xffffffffu, n_e);
  if (lane == 0) {
    sm.warp_cnt[0][warp] = n_g;
    sm.warp_cnt[1][warp] = n_e;
  }
  __syncthreads();
  // keys before this warp: lane l holds warps 0..l inclusive
  int sg = lane < NW ? sm.warp_cnt[0][lane] : 0, se = lane < NW ? sm.warp_cnt[1][lane] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int tg = __shfl_up_sync(0xffffffffu, sg, o), te = __shfl_up_sync(0xffffffffu, se, o);
    if (lane >= o) {
      sg += tg;
      se += te;
    }
  }
  int g_run = warp ? __shfl_sync(0xffffffffu, sg, warp - 1) : 0;
  int e_run = warp ? __shfl_sync(0xffffffffu, se, warp - 1) : 0;
  for (int c = w0; c < w1; c += 1024) {
    unsigned gm, em;
    chunk_masks(c + 32 * lane, gm, em);
    const int ng = __popc(gm), ne = __popc(em);
    int ig = ng, ie = ne;  // inclusive scans over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tg = __shfl_up_sync(0xffffffffu, ig, o), te = __shfl_up_sync(0xffffffffu, ie, o);
      if (lane >= o) {
        ig += tg;
        ie += te;
      }
    }
    const int gb = g_run + ig - ng, eb = e_run + ie - ne;  // keys before this lane's first
    unsigned take = gm;
    for (int keep = min(max(kr - eb, 0), ne); keep > 0; --keep) {
      take |= em & (0u - em);
      em &= em - 1u;
    }
    int pos = gb + min(eb, kr);
    const int i0 = c + 32 * lane;
    while (take) {
      const int b = __ffs(take) - 1;
      take &= take - 1u;
      if (pos < k) sel[pos] = i0 + b;
      ++pos;
    }
    g_run += __shfl_sync(0xffffffffu, ig, 31);
    e_run += __shfl_sync(0xffffffffu, ie, 31);
  }
  // self-check: exactly k blocks were emitted
  if (warp == NW - 1 && lane == 0 && g_run + min(e_run, kr) != k) set_status(dev_status, KIN_ERR_DEVICE_DATA);
}

// Ranks the c keys sm.list[off..off+c) pairwise: the need-th largest, with
// multiplicity, is the threshold T, and need - #{keys > T} of the keys equal
// to T are kept.  Every thread that finds it writes the same values.  Ends
// with a barrier.
template <int NT>
__device__ __forceinline__ void rank_keys(int off, int c, int need, TopkSmem<NT>& sm) {
  const uint32_t* list = sm.list + off;
  for (int j = threadIdx.x; j < c; j += NT) {
    const uint32_t kj = list[j];
    int gt = 0, ge = 0;
    for (int i = 0; i < c; ++i) {
      const uint32_t ki = list[i];
      gt += ki > kj;
      ge += ki >= kj;
    }
    if (gt < need && need <= ge) {
      sm.thresh = kj;
      sm.thresh_take = need - gt;
    }
  }
  __syncthreads();
}

// rank_keys over c <= NT / 4 keys (off 0) with four threads per key: thread
// 4 j + part counts the keys part, part + 4, ... against key j, and a
// two-step shuffle sums the four counts (a quarter of the serial loop).
// Ends with a barrier.
template <int NT>
__device__ __forceinline__ void rank_keys_split4(int c, int need, TopkSmem<NT>& sm) {
  const int j = threadIdx.x >> 2, part = threadIdx.x & 3;
  const bool mine = j < c;
  const uint32_t kj = mine ? sm.list[j] : 0u;
  int gt = 0, ge = 0;
  if (mine) {
    for (int i = part; i < c; i += 4) {
      const uint32_t ki = sm.list[i];
      gt += ki > kj;
      ge += ki >= kj;
    }
  }
  gt += __shfl_xor_sync(0xffffffffu, gt, 1);
  ge += __shfl_xor_sync(0xffffffffu, ge, 1);
  gt += __shfl_xor_sync(0xffffffffu, gt, 2);
  ge += __shfl_xor_sync(0xffffffffu, ge, 2);
  if (mine && part == 0 && gt < need && need <= ge) {
    sm.thresh = kj;
    sm.thresh_take = need - gt;
  }
  __syncthreads();
}

// The boundary bin's c keys (sm.list[0..c)) ranked pairwise.
template <int NT>
__device__ __forceinline__ void rank_boundary_bin(int c, int need, TopkSmem<NT>& sm) {
  rank_keys(0, c, need, sm);
}

// Sub-bin (0..255) of a key whose scaled score x = (s - s_min) * (256 /
// (s_max - s_min)) fell in equal-width bin `bin`: the fraction of x above the
// bin's lower edge, cut into 256 equal parts.  Non-decreasing in x (the
// subtraction of a constant and the scaling by 2^8 are correctly rounded),
// with explicitly rounded operations so that no call site fuses them.
__device__ __forceinline__ int sub_bin(float x, int bin) {
  const float f = __fmul_rn(__fsub_rn(x, (float)bin), 256.f);
  return min(max((int)f, 0), 255);
}

// The equal-width-bin search fused with the emit, for rows whose emit ranges
// are one round per warp (nb <= 1024 warps): the bin histogram (any order),
// then one pass in the emit's ownership (lane l of warp w: the 32 keys from
// w0 + 32 l, rotated reads) that sets, per lane, the mask of keys taken
// outright (forced, or in a bin above the boundary bin) and the mask of keys
// in the boundary bin, and lists the latter's keys (one reservation per
// warp).  A boundary bin of more than kDirectRank keys also histograms its
// keys' 256 sub-bins (sm.hist[1]) while listing them, and only the sub-bin
// holding the threshold is copied out and ranked pairwise (keys in higher
// sub-bins are larger); a smaller bin is ranked whole.  Then only the
// boundary-bin bits are revisited to split them into above / equal to the
// threshold, and emit_round writes.  Returns false (CTA-uniform, nothing
// written) when the range is empty or not finite, or the boundary bin holds
// more than kRankCap keys.  Expects sm.hist[0] and sm.hist[1] zero.
template <int NT>
__device__ __forceinline__ bool linear_select(const uint32_t* keys, uint8_t* bins, int nb, const Cands& cd, int k,
                                              uint32_t kmin, uint32_t kmax, int32_t* sel, TopkSmem<NT>& sm,
                                              int32_t* dev_status) {
  constexpr int NW = NT / 32;
  const int kr = cd.kr;
  const float lo = key_float(kmin), hi = key_float(kmax);
  const float range = hi - lo;
  const float inv = 256.f / range;
  if (!(isfinite(lo) && isfinite(hi) && range > 0.f && isfinite(range) && isfinite(inv))) return false;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto scaled = [&](uint32_t key) { return __fmul_rn(__fsub_rn(key_float(key), lo), inv); };
  auto bin_of = [&](uint32_t key) { return min((int)scaled(key), 255); };
  for (int i = cd.lo + tid; i <= cd.hi; i += NT) {
    const int bin = bin_of(keys[i]);
    bins[i] = (uint8_t)bin;
    atomicAdd(&sm.hist[0][hidx(bin)], 1);
  }
  if (tid == 0) sm.list_n = sm.list_n2 = 0;
  __syncthreads();
  int bstar, above, c;
  warp_find_bin(sm.hist[0], kr, bstar, above, c);  // every warp, same result
  if (c > kRankCap) return false;
  const bool two_level = c > kDirectRank;
  auto sub_of = [&](uint32_t key) { return sub_bin(scaled(key), bstar); };
  const int span = ((nb + NW - 1) / NW + 1023) & ~1023;  // 1024: one round
  const int w0 = min(warp * span, nb), w1 = min(w0 + span, nb);
  const int c0 = w0 + 32 * lane;
  unsigned gm = 0u, bm = 0u;
  if (c0 + 32 <= w1 && c0 >= cd.lo && c0 + 31 <= cd.hi) {  // 32 candidates
    // the chunk's 32 bins as 8 words, 4 compared at once; word r holds keys
    // c0 + 4r .. c0 + 4r + 3 (byte e: key c0 + 4r + e).  Lane l takes word
    // (j + l / 4) mod 8 at step j: 32 distinct banks.  A compare gives 0xFF
    // per true byte; (m & 0x01010101) * 0x01020408 gathers the four flags
    // into bits 24..27 (byte e's flag to bit 24 + e, no carries).
    const uint32_t b4 = 0x01010101u * (uint32_t)bstar;
    const uint32_t* binw = reinterpret_cast<const uint32_t*>(bins + c0);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = (j + (lane >> 2)) & 7;
      const uint32_t w = binw[r];
      const uint32_t gt = __vcmpgtu4(w, b4), eq = __vcmpeq4(w, b4);
      gm |= (((gt & 0x01010101u) * 0x01020408u) >> 24) << (4 * r);
      bm |= (((eq & 0x01010101u) * 0x01020408u) >> 24) << (4 * r);
    }
  } else if (c0 < w1) {
    for (int j = 0; j < 32; ++j) {
      const int b = (j + lane) & 31;
      const int i = c0 + b;
      if (i < w1) {
        if (!cd.has(i)) {
          gm |= 1u << b;  // forced
        } else {
          const int bin = bins[i];
          gm |= (unsigned)(bin > bstar) << b;
          bm |= (unsigned)(bin == bstar) << b;
        }
      }
    }
  }
  {  // list the boundary bin's keys: one reservation per warp, lanes in order
    const int nbm = __popc(bm);
    int incl = nbm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int slot = 0;
    if (lane == 31 && incl) slot = atomicAdd(&sm.list_n, incl);
    slot = __shfl_sync(0xffffffffu, slot, 31) + incl - nbm;
    for (unsigned m = bm; m; m &= m - 1u, ++slot) {
      const uint32_t key = keys[c0 + __ffs(m) - 1];
      if (slot < kListCap) sm.list[slot] = key;
      if (two_level) atomicAdd(&sm.hist[1][hidx(sub_of(key))], 1);
    }
  }
  __syncthreads();
  if (two_level) {
    int sb, above2, c2;
    warp_find_bin(sm.hist[1], kr - above, sb, above2, c2);  // every warp, same result
    for (int base = 0; base < c; base += NT) {  // copy the sub-bin's keys to list[c..c+c2)
      const int j = base + tid;
      const uint32_t key = j < c ? sm.list[j] : 0u;
      const bool match = j < c && sub_of(key) == sb;
      const unsigned m = __ballot_sync(0xffffffffu, match);
      if (m) {
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&sm.list_n2, __popc(m));
        slot = c + __shfl_sync(0xffffffffu, slot, 0) + __popc(m & ((1u << lane) - 1u));
        if (match && slot < kListCap) sm.list[slot] = key;
      }
    }
    __syncthreads();
    rank_keys(c, c2, kr - above - above2, sm);
  } else {
    rank_keys(0, c, kr - above, sm);
  }
  const uint32_t T = sm.thresh;
  unsigned em = 0u;
  for (unsigned m = bm; m; m &= m - 1u) {
    const int b = __ffs(m) - 1;
    const uint32_t key = keys[c0 + b];
    gm |= (unsigned)(key > T) << b;
    em |= (unsigned)(key == T) << b;
  }
  emit_round(gm, em, c0, k, sm.thresh_take, sel, sm, dev_status);
  return true;
}

// One-pass threshold search for score distributions without extreme
// outliers, over keys in memory, for rows longer than 1024 keys per warp
// (shorter rows take linear_select, which shares its binning and fuses the
// emit).  The candidates' scores are cut into 256
// equal-width bins between the smallest (kmin) and largest (kmax) candidate
// key; the bin of a score, trunc((s - s_min) * (256 / (s_max - s_min))), is a
// non-decreasing function of s (a correctly rounded subtract and multiply,
// then truncation), so every key in a higher bin is larger than every key in
// a lower one.  One histogram finds the bin holding the kr-th largest key;
// its keys (at most kRankCap) are ranked pairwise to find the exact
// threshold key and how many keys equal to it to keep.  Returns false
// (CTA-uniform) when the range is empty or not finite, or the boundary bin
// is too crowded: the caller then runs the radix search.  Expects
// sm.hist[0] zero.
template <int NT>
__device__ __forceinline__ bool linear_threshold(const uint32_t* keys, const Cands& cd, int kr, uint32_t kmin,
                                                 uint32_t kmax, TopkSmem<NT>& sm, uint32_t& thresh,
                                                 int& take) {
  const float lo = key_float(kmin), hi = key_float(kmax);
  const float range = hi - lo;
  const float inv = 256.f / range;
  if (!(isfinite(lo) && isfinite(hi) && range > 0.f && isfinite(range) && isfinite(inv))) return false;
  const int tid = threadIdx.x, lane = tid & 31;
  auto bin_of = [&](uint32_t key) { return min((int)((key_float(key) - lo) * inv), 255); };
  for (int i = cd.lo + tid; i <= cd.hi; i += NT) atomicAdd(&sm.hist[0][hidx(bin_of(keys[i]))], 1);
  if (tid == 0) sm.list_n = 0;
  __syncthreads();
  int bstar, above, c;
  warp_find_bin(sm.hist[0], kr, bstar, above, c);  // every warp, same result
  if (c > kRankCap) return false;
  for (int base = cd.lo; base <= cd.hi; base += NT) {  // uniform trip count per warp
    const int i = base + tid;
    const bool in = i <= cd.hi;
    const uint32_t key = in ? keys[i] : 0u;
    const bool match = in && bin_of(key) == bstar;
    const unsigned m = __ballot_sync(0xffffffffu, match);
    if (m) {  // warp-uniform: one list reservation per warp, lanes take slots in order
      int slot = 0;
      if (lane == 0) slot = atomicAdd(&sm.list_n, __popc(m));
      slot = __shfl_sync(0xffffffffu, slot, 0);
      if (match) sm.list[slot + __popc(m & ((1u << lane) - 1u))] = key;
    }
  }
  __syncthreads();
  rank_boundary_bin(c, kr - above, sm);
  thresh = sm.thresh;
  take = sm.thresh_take;
  return true;
}

// Exact top-(k-2) over keys[1..nb-2] plus the forced blocks 0 and nb-1,
// written ascending to sel[0..k).  kmin / kmax: the smallest and largest
// candidate key; bins: nb bytes of shared memory for the keys' bins, or
// null.  Expects sm.hist[0] and sm.hist[1] zero.
template <int NT>
__device__ __forceinline__ void select_from_keys(const uint32_t* keys, uint8_t* bins, int nb, const Cands& cd, int k,
                                                 uint32_t kmin, uint32_t kmax, int32_t* sel, TopkSmem<NT>& sm,
                                                 int32_t* dev_status) {
  constexpr int NW = NT / 32;
  uint32_t prefix = 0xFFFFFFFFu, mask = 0xFFFFFFFFu;  // kr == 0: no candidate passes
  int kr = cd.kr;
  if (kr > 0) {
    if (bins && nb <= 1024 * NW) {
      if (linear_select(keys, bins, nb, cd, k, kmin, kmax, sel, sm, dev_status)) return;
    } else if (linear_threshold(keys, cd, kr, kmin, kmax, sm, prefix, kr)) {
      emit_selection(keys, nb, cd, k, prefix, mask, kr, sel, sm, dev_status);
      return;
    }
    __syncthreads();  // every warp is done with the bin histogram
    zero_hist(sm, 0);
    __syncthreads();
    for (int i = cd.lo + threadIdx.x; i <= cd.hi; i += NT) atomicAdd(&sm.hist[0][hidx(keys[i] >> 24)], 1);
    __syncthreads();
    kr = cd.kr;
    radix_threshold(keys, nb, cd, sm, prefix, mask, kr);
  }
  emit_selection(keys, nb, cd, k, prefix, mask, kr, sel, sm, dev_status);
}

// Loads a pair's nb scores (written by the scan kernel: read from L2) as
// keys into keys[] (shared memory, or the score row itself), returns the
// smallest and largest candidate key, and zeroes both histograms.  With both
// rows 16-byte aligned, whole groups of 4 scores move as 16-byte loads and
// stores, 8 per thread in flight; the rest one score at a time.
template <int NT>
__device__ __forceinline__ void load_keys(const uint32_t* sc, uint32_t* keys, int nb, const Cands& cd, TopkSmem<NT>& sm,
                                          uint32_t& kmin, uint32_t& kmax) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  int done = 0;
  if (((reinterpret_cast<uintptr_t>(sc) | reinterpret_cast<uintptr_t>(keys)) & 15) == 0) {
    constexpr int kVec = 8;
    const int nv = nb >> 2;
    const uint4* sc4 = reinterpret_cast<const uint4*>(sc);
    uint4* keys4 = reinterpret_cast<uint4*>(keys);
    for (int base = 0; base < nv; base += kVec * NT) {
      uint4 v[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int j = base + u * NT + tid;
        v[u] = j < nv ? __ldcg(sc4 + j) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int j = base + u * NT + tid;
        if (j < nv) {
          const uint4 kk = make_uint4(key_of_bits(v[u].x), key_of_bits(v[u].y), key_of_bits(v[u].z), key_of_bits(v[u].w));
          keys4[j] = kk;
          const int i = 4 * j;
          if (i >= cd.lo && i + 3 <= cd.hi) {
            lo = min(lo, min(min(kk.x, kk.y), min(kk.z, kk.w)));
            hi = max(hi, max(max(kk.x, kk.y), max(kk.z, kk.w)));
          } else {
            if (cd.has(i)) { lo = min(lo, kk.x); hi = max(hi, kk.x); }
            if (cd.has(i + 1)) { lo = min(lo, kk.y); hi = max(hi, kk.y); }
            if (cd.has(i + 2)) { lo = min(lo, kk.z); hi = max(hi, kk.z); }
            if (cd.has(i + 3)) { lo = min(lo, kk.w); hi = max(hi, kk.w); }
          }
        }
      }
    }
    done = nv << 2;
  }
  constexpr int kBatch = 8;
  for (int base = done; base < nb; base += kBatch * NT) {
    uint32_t v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * NT + tid;
      v[u] = i < nb ? __ldcg(sc + i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * NT + tid;
      if (i < nb) {
        const uint32_t key = key_of_bits(v[u]);
        keys[i] = key;
        if (cd.has(i)) {
          lo = min(lo, key);
          hi = max(hi, key);
        }
      }
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    sm.wmin[warp] = lo;
    sm.wmax[warp] = hi;
  }
  zero_hist(sm, 0);
  zero_hist(sm, 1);
  __syncthreads();
  kmin = sm.wmin[0];
  kmax = sm.wmax[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    kmin = min(kmin, sm.wmin[w]);
    kmax = max(kmax, sm.wmax[w]);
  }
}

// The top-k of one row of nb scores with any nb, keys in memory: shared
// memory when nb <= key_cap (skey holds key_cap words, then key_cap bytes
// for the keys' bins), else gkeys (nb words of global scratch, which may be
// the score row itself when nothing reads it afterwards).
template <int NT>
__device__ __forceinline__ void topk_memory(const uint32_t* row, int nb, const Cands& cd, int k, int32_t* sel,
                                            uint32_t* skey, int key_cap, uint32_t* gkeys, TopkSmem<NT>& sm,
                                            int32_t* dev_status) {
  const bool in_smem = nb <= key_cap;
  uint32_t* keys = in_smem ? skey : gkeys;
  uint8_t* bins = in_smem ? reinterpret_cast<uint8_t*>(skey + key_cap) : nullptr;
  uint32_t kmin, kmax;
  load_keys(row, keys, nb, cd, sm, kmin, kmax);
  select_from_keys(keys, bins, nb, cd, k, kmin, kmax, sel, sm, dev_status);
}

// The emit of the register path: thread t owns blocks u * NT + t (u < KPT),
// so every ballot walks the blocks in index order.  Keeps the forced
// blocks, every candidate whose key is above T, and the first `take`
// candidates (by index) whose key equals T.  Per 32-block slot (u, warp)
// one ballot pair counts the keys above the threshold (or forced) and the
// keys equal to it, one barrier publishes the packed counts, every warp
// scans them, and every thread writes its taken indices at their final
// positions.
template <int NT, int KPT>
__device__ __forceinline__ void emit_regs(const uint32_t (&key)[KPT], int nb, const Cands& cd, int k, uint32_t T,
                                          int take, int32_t* sel, TopkSmem<NT>& sm, int32_t* dev_status) {
  constexpr int NW = NT / 32;
  constexpr int kPerLane = KPT * NW / 32;  // slots per lane in the emit's scan
  static_assert(KPT <= kMaxKPT && kPerLane >= 1 && NW % kPerLane == 0, "slot layout");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // slot s = u * NW + warp covers blocks 32 s .. 32 s + 31, in index order
  const unsigned lt = (1u << lane) - 1u;
  auto flags = [&](int u, bool& g, bool& e) {
    const int i = u * NT + tid;
    const bool cand = cd.has(i);
    g = (i < nb && !cand) || (cand && key[u] > T);
    e = cand && key[u] == T;
  };
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    bool g, e;
    flags(u, g, e);
    const unsigned gb = __ballot_sync(0xffffffffu, g), eb = __ballot_sync(0xffffffffu, e);
    if (lane == 0) sm.slot_cnt[u * NW + warp] = __popc(gb) | (__popc(eb) << 16);
  }
  __syncthreads();
  // this warp's slots all sit at offset warp % kPerLane within their owner lane
  const int jw = warp % kPerLane;
  int tot = 0, mine = 0;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    const int v = sm.slot_cnt[lane * kPerLane + j];
    if (j < jw) mine += v;
    tot += v;
  }
  int inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  mine += inc - tot;
  const int all = __shfl_sync(0xffffffffu, inc, 31);
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int base = __shfl_sync(0xffffffffu, mine, (u * NW + warp) / kPerLane);
    bool g, e;
    flags(u, g, e);
    const unsigned gb = __ballot_sync(0xffffffffu, g), eb = __ballot_sync(0xffffffffu, e);
    const int gt_before = (base & 0xFFFF) + __popc(gb & lt);
    const int eq_before = (base >> 16) + __popc(eb & lt);
    if (g || (e && eq_before < take)) {
      const int pos = gt_before + min(eq_before, take);
      if (pos < k) sel[pos] = u * NT + tid;  // never write past the pair's row
    }
  }
  // self-check: exactly k blocks were emitted
  if (tid == 0 && (all & 0xFFFF) + min(all >> 16, take) != k) set_status(dev_status, KIN_ERR_DEVICE_DATA);
}

// The threshold search of the register path over keys already in
// registers (thread t: blocks u * NT + t), then the emit.  Same search as
// the memory path (equal-width bins; the radix search on a crowded or
// degenerate range runs from shared memory).  Only the candidates' keys
// are read.
template <int NT, int KPT>
__device__ __forceinline__ void topk_regs_keys(const uint32_t (&key)[KPT], int nb, const Cands& cd, int k, int32_t* sel,
                                               uint32_t* skey, TopkSmem<NT>& sm, int32_t* dev_status) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int i = u * NT + tid;
    if (cd.has(i)) {
      lo = min(lo, key[u]);
      hi = max(hi, key[u]);
    }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    sm.wmin[warp] = lo;
    sm.wmax[warp] = hi;
  }
  zero_hist(sm, 0);
  if (tid == 0) sm.list_n = 0;
  __syncthreads();
  uint32_t kmin = sm.wmin[0], kmax = sm.wmax[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    kmin = min(kmin, sm.wmin[w]);
    kmax = max(kmax, sm.wmax[w]);
  }

  const int kr = cd.kr;
  uint32_t T = 0xFFFFFFFFu;  // kr == 0: no candidate is above T, none equal is taken
  int take = 0;
  if (kr > 0) {
    const float flo = key_float(kmin), fhi = key_float(kmax);
    const float range = fhi - flo;
    const float inv = 256.f / range;
    bool ok = isfinite(flo) && isfinite(fhi) && range > 0.f && isfinite(range) && isfinite(inv);
    auto bin_of = [&](uint32_t kk) { return min((int)((key_float(kk) - flo) * inv), 255); };
    int bstar = 0, above = 0, c = 0;
    if (ok) {
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        const int i = u * NT + tid;
        if (cd.has(i)) atomicAdd(&sm.hist[0][hidx(bin_of(key[u]))], 1);
      }
      __syncthreads();
      warp_find_bin(sm.hist[0], kr, bstar, above, c);  // every warp, same result
      ok = c <= kRankCap;
    }
    if (!ok) {  // crowded or degenerate range: radix search from shared memory
      __syncthreads();  // every warp is done with the bin histogram
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        const int i = u * NT + tid;
        if (i < nb) skey[i] = key[u];
      }
      zero_hist(sm, 0);
      zero_hist(sm, 1);
      __syncthreads();
      for (int i = cd.lo + tid; i <= cd.hi; i += NT) atomicAdd(&sm.hist[0][hidx(skey[i] >> 24)], 1);
      __syncthreads();
      uint32_t prefix, mask;
      int kr2 = kr;
      radix_threshold(skey, nb, cd, sm, prefix, mask, kr2);
      emit_selection(skey, nb, cd, k, prefix, mask, kr2, sel, sm, dev_status);
      return;
    }
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int i = u * NT + tid;
      const bool match = cd.has(i) && bin_of(key[u]) == bstar;
      const unsigned m = __ballot_sync(0xffffffffu, match);
      if (m) {  // warp-uniform
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&sm.list_n, __popc(m));
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if (match) sm.list[slot + __popc(m & ((1u << lane) - 1u))] = key[u];
      }
    }
    __syncthreads();
    rank_boundary_bin(c, kr - above, sm);
    T = sm.thresh;
    take = sm.thresh_take;
  }

  emit_regs<NT, KPT>(key, nb, cd, k, T, take, sel, sm, dev_status);
}

// The top-k of one pair with nb <= KPT * NT blocks, keys held in registers:
// thread t loads blocks u * NT + t (u < KPT) from the score row.
template <int NT, int KPT>
__device__ __forceinline__ void topk_regs(const uint32_t* row, int nb, const Cands& cd, int k, int32_t* sel, uint32_t* skey,
                                          TopkSmem<NT>& sm, int32_t* dev_status) {
  uint32_t key[KPT];
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int i = u * NT + threadIdx.x;
    key[u] = i < nb ? key_of_bits(__ldcg(row + i)) : 0u;
  }
  topk_regs_keys<NT, KPT>(key, nb, cd, k, sel, skey, sm, dev_status);
}

// ---- kernel 1: the scan.  Rows are numbered per pair in steps of U
// (a pair owns nbp = nbcap rounded up to U row slots, so no step straddles
// two pairs; fewer than 2^31 slots, checked on the host).  The slots are cut
// into one contiguous, U-aligned range per warp; each warp streams its range
// U rows per step, double-buffered, with the group's summed query cached for
// the current pair.  Rows at or beyond a pair's block count, and pairs whose
// budget covers every block, are skipped.
__device__ __forceinline__ int pair_nb(const SelectParams& p, int pair) {
  const int L = __ldg(p.seq_lens + pair / p.Hkv);
  const int nb = (L >= 1 && L <= p.Lcap) ? (L + p.bs - 1) / p.bs : 0;
  return nb > p.k ? nb : 0;  // 0: no scores needed for this pair
}

__device__ __forceinline__ void pair_qsum(const SelectParams& p, int pair, int lane, float (&o)[4]) {
  // the g query rows read from L2 (ld.global.cg) four at a time, summed in
  // row order from 0 (the scan's order)
  const int b = pair / p.Hkv, h = pair - b * p.Hkv;
  const uint2* qg = reinterpret_cast<const uint2*>(p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim) + lane;
  o[0] = o[1] = o[2] = o[3] = 0.f;
  for (int j0 = 0; j0 < p.g; j0 += 4) {
    uint2 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) raw[j] = j0 + j < p.g ? __ldcg(qg + (j0 + j) * (kHeadDim / 4)) : make_uint2(0u, 0u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j0 + j < p.g) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw[j].x));
        const float2 bb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw[j].y));
        o[0] += a.x;
        o[1] += a.y;
        o[2] += bb.x;
        o[3] += bb.y;
      }
    }
  }
}

// Mean rows as loaded (fp32: a float4 of 4 dims per lane; bf16: a uint2 of
// 4 bf16 dims) and as used (4 floats).
template <bool kBf16>
struct MeanLane {
  using Raw = typename std::conditional<kBf16, uint2, float4>::type;
  static __device__ __forceinline__ Raw zero() {
    if constexpr (kBf16) return make_uint2(0u, 0u);
    else return make_float4(0.f, 0.f, 0.f, 0.f);
  }
  static __device__ __forceinline__ float4 widen(Raw r) {
    if constexpr (kBf16) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&r.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&r.y));
      return make_float4(a.x, a.y, b.x, b.y);
    } else {
      return r;
    }
  }
};

// U rows per warp step: 8 fp32 rows or 16 bf16 rows, 4 KB in flight either way.
template <bool kBf16, int U>
__global__ void __launch_bounds__(kSelThreads, KIN_SEL_CTAS_PER_SM) select_scan_kernel(SelectParams p) {
  using ML = MeanLane<kBf16>;
  using Raw = typename ML::Raw;
  pdl_wait();  // means, lengths and q come from earlier work on the stream
  pdl_trigger_early();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kSelWarps;
  const int gw = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int nbp = (p.nbcap + U - 1) / U * U;
  const int steps = p.B * p.Hkv * (nbp / U);
  const int per = (steps + nwarps - 1) / nwarps;
  const int s0 = gw * per, s1 = min(s0 + per, steps);
  if (s0 >= s1) {
    pdl_trigger_late();
    return;
  }

  // step s covers slots s*U .. s*U+U-1 of pair (s*U) / nbp
  int pair = (s0 * U) / nbp;
  int blk = s0 * U - pair * nbp;
  int nb = pair_nb(p, pair);
  float qs[4];
  pair_qsum(p, pair, lane, qs);
  const Raw* mrow = reinterpret_cast<const Raw*>(p.means) + lane;
  auto row_ptr = [&](int pr, int bk) { return mrow + ((int64_t)pr * p.nbcap + bk) * (kHeadDim / 4); };

  Raw cur[U];
#pragma unroll
  for (int u = 0; u < U; ++u) cur[u] = blk + u < nb ? __ldcs(row_ptr(pair, blk + u)) : ML::zero();
  for (int s = s0; s < s1; ++s) {
    // the next step's rows fly during this step's math
    int npair = pair, nblk = blk + U, nnb = nb;
    if (nblk >= nbp) {
      npair = pair + 1;
      nblk = 0;
      nnb = s + 1 < s1 ? pair_nb(p, npair) : 0;
    }
    const bool more = s + 1 < s1;
    Raw nxt[U];
#pragma unroll
    for (int u = 0; u < U; ++u) nxt[u] = more && nblk + u < nnb ? __ldcs(row_ptr(npair, nblk + u)) : ML::zero();
    if (blk < nb) {
      float d[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float4 m = ML::widen(cur[u]);
        d[u] = qs[0] * m.x;
        d[u] = fmaf(qs[1], m.y, d[u]);
        d[u] = fmaf(qs[2], m.z, d[u]);
        d[u] = fmaf(qs[3], m.w, d[u]);
      }
      const float tot = warp_sum_rows<U>(d, lane);
      const int row = lane / (32 / U);
      if ((lane & (32 / U - 1)) == 0 && blk + row < nb)
        p.scores[(int64_t)pair * p.nbcap + blk + row] = tot * p.score_scale;
    }
    if (npair != pair && more) pair_qsum(p, npair, lane, qs);
    pair = npair;
    blk = nblk;
    nb = nnb;
#pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = nxt[u];
  }
  pdl_trigger_late();
}

// ---- kernel 1b: the scan of dual block means' bf16 rows (KIN_MEANS_DUAL).
// Its scores only have to lie within the refinement's error bound of the
// fp32 scan's (an fp32 dot product of depth at most 12, from the same fp32
// summed query), so it is laid out for fewer instructions per byte: a
// half-warp per row, lane x of a half holding dims 8x..8x+7, so one 16-byte
// load per lane covers two rows per warp; an 8-term fma chain per row; and
// a transposing reduction over the 16 lanes of a half: each of the first
// log2(V) levels (xor 8, 4, ...) hands half of the rows a lane keeps to its
// partner (V - 1 shuffles for V rows), plain butterfly levels finish (depth
// 8 + 4 = 12).  V loads per lane per step, U = 2 V rows per warp step,
// contiguous U-aligned step ranges per warp as in the scan above.
template <int V>
__device__ __forceinline__ void dual_qsum(const SelectParams& p, int pair, int x, float (&o)[8]) {
  // dims 8x..8x+7 of the group-summed query, summed in row order from 0
  // (the same fp32 values as pair_qsum's)
  const int b = pair / p.Hkv, h = pair - b * p.Hkv;
  const uint4* qg = reinterpret_cast<const uint4*>(p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim) + x;
#pragma unroll
  for (int c = 0; c < 8; ++c) o[c] = 0.f;
  for (int j0 = 0; j0 < p.g; j0 += 4) {
    uint4 raw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) raw[j] = j0 + j < p.g ? __ldcg(qg + (j0 + j) * (kHeadDim / 8)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j0 + j < p.g) {
        const uint32_t w[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          o[2 * c] += __uint_as_float(w[c] << 16);
          o[2 * c + 1] += __uint_as_float(w[c] & 0xFFFF0000u);
        }
      }
    }
  }
}

template <int V, int CTAS>
__global__ void __launch_bounds__(kSelThreads, CTAS) select_scan_dual_kernel(SelectParams p) {
  static_assert(V == 4 || V == 8, "V loads per lane per step");
  constexpr int U = 2 * V;     // rows per warp per step
  constexpr int kGrp = 16 / V;  // lanes of a half that end holding the same row
  pdl_wait();  // means, lengths and q come from earlier work on the stream
  pdl_trigger_early();
  const int lane = threadIdx.x & 31, hh = lane >> 4, x = lane & 15;
  const int nwarps = gridDim.x * kSelWarps;
  const int gw = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int nbp = (p.nbcap + U - 1) / U * U;
  const int steps = p.B * p.Hkv * (nbp / U);
  const int per = (steps + nwarps - 1) / nwarps;
  const int s0 = gw * per, s1 = min(s0 + per, steps);
  if (s0 >= s1) {
    pdl_trigger_late();
    return;
  }
  // step-local row r = 2 j + hh comes from the lane's j-th load
  const uint4* mrow = reinterpret_cast<const uint4*>(p.means) + hh * (kHeadDim / 8) + x;
  auto load = [&](int pr, int bk, int nbr, bool any, uint4 (&v)[V]) {
    const uint4* b0 = mrow + ((int64_t)pr * p.nbcap + bk) * (kHeadDim / 8);
    if (any && bk + U <= nbr) {
#pragma unroll
      for (int j = 0; j < V; ++j) v[j] = __ldcs(b0 + j * 2 * (kHeadDim / 8));
    } else {
#pragma unroll
      for (int j = 0; j < V; ++j)
        v[j] = any && bk + 2 * j + hh < nbr ? __ldcs(b0 + j * 2 * (kHeadDim / 8)) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  int pair = (s0 * U) / nbp;
  int blk = s0 * U - pair * nbp;
  int nb = pair_nb(p, pair);
  float qs[8];
  dual_qsum<V>(p, pair, x, qs);
  uint4 cur[V];
  load(pair, blk, nb, true, cur);
  for (int s = s0; s < s1; ++s) {
    int npair = pair, nblk = blk + U, nnb = nb;
    if (nblk >= nbp) {
      npair = pair + 1;
      nblk = 0;
      nnb = s + 1 < s1 ? pair_nb(p, npair) : 0;
    }
    const bool more = s + 1 < s1;
    uint4 nxt[V];
    load(npair, nblk, nnb, more, nxt);  // the next step's rows fly during this step's math
    if (blk < nb) {
      float d[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const uint32_t w[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
        float t = qs[0] * __uint_as_float(w[0] << 16);
        t = fmaf(qs[1], __uint_as_float(w[0] & 0xFFFF0000u), t);
#pragma unroll
        for (int c = 1; c < 4; ++c) {
          t = fmaf(qs[2 * c], __uint_as_float(w[c] << 16), t);
          t = fmaf(qs[2 * c + 1], __uint_as_float(w[c] & 0xFFFF0000u), t);
        }
        d[j] = t;
      }
      // transposing levels: at offset 8 >> s, the upper lane keeps the upper
      // half of its rows
#pragma unroll
      for (int sl = 0, half = V / 2; half >= 1; ++sl, half >>= 1) {
        const bool upper = (x >> (3 - sl)) & 1;
#pragma unroll
        for (int j = 0; j < half; ++j) {
          const float keep = upper ? d[j + half] : d[j];
          const float send = upper ? d[j] : d[j + half];
          d[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8 >> sl);
        }
      }
      float tot = d[0];
#pragma unroll
      for (int off = kGrp / 2; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
      const int r = 2 * (x / kGrp) + hh;  // the step-local row this lane holds
      if ((x & (kGrp - 1)) == 0 && blk + r < nb) p.scores[(int64_t)pair * p.nbcap + blk + r] = tot * p.score_scale;
    }
    if (npair != pair && more) dual_qsum<V>(p, npair, x, qs);
    pair = npair;
    blk = nblk;
    nb = nnb;
#pragma unroll
    for (int j = 0; j < V; ++j) cur[j] = nxt[j];
  }
  pdl_trigger_late();
}

// The scan over block means stored per page (the shared-prompt layout),
// found through the page table.  Rows are scattered, so a warp splits into
// 4 groups of 8 lanes, each group owning one mean row at a time: lane x of a
// group holds the 4-dim partials of lanes x, x+8, x+16 and x+24 of the
// contiguous kernel's layout (4 coalesced loads), every lane of a group
// fetches its row's page index itself (no address shuffles), and the row
// total is formed by the same pairing tree as warp_sum_rows (xor 16 and 8
// inside the lane, xor 4, 2, 1 across the group), so the scores equal the
// contiguous kernel's bit for bit.  RG row groups per lane per step keep
// 4 KB of means in flight per warp; the page indices of the next step are
// loaded one step ahead of its rows.
template <bool kBf16>
__global__ void __launch_bounds__(kSelThreads, KIN_SEL_CTAS_PER_SM) select_scan_paged_kernel(SelectParams p) {
  using ML = MeanLane<kBf16>;
  using Raw = typename ML::Raw;
  constexpr int RG = kBf16 ? 4 : 2;  // rows per lane per step
  constexpr int U = 4 * RG;          // rows per warp per step
  pdl_wait();
  pdl_trigger_early();
  const int lane = threadIdx.x & 31, grp = lane >> 3, x = lane & 7;
  const int nwarps = gridDim.x * kSelWarps;
  const int gw = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int nbp = (p.nbcap + U - 1) / U * U;
  const int steps = p.B * p.Hkv * (nbp / U);
  const int per = (steps + nwarps - 1) / nwarps;
  const int s0 = gw * per, s1 = min(s0 + per, steps);
  if (s0 >= s1) {
    pdl_trigger_late();
    return;
  }
  // lane row j of a step is block blk + grp + 4 j
  auto load_pages = [&](int pr, int bk, int nbr, int (&pg)[RG]) {
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      const int r = bk + grp + 4 * j;
      pg[j] = -1;
      if (r < nbr) {
        const int v = __ldg(p.mpages.table + (int64_t)(pr / p.Hkv) * p.mpages.max_blocks + r);
        if (v < 0 || v >= p.mpages.num_pages) {
          if (x == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
        } else {
          pg[j] = v;
        }
      }
    }
  };
  const Raw* mbase = reinterpret_cast<const Raw*>(p.means) + x;
  auto load_rows = [&](int pr, const int (&pg)[RG], Raw (&v)[RG][4]) {
    const int h = pr % p.Hkv;
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      const Raw* row = mbase + ((int64_t)(pg[j] < 0 ? 0 : pg[j]) * p.Hkv + h) * (kHeadDim / 4);
#pragma unroll
      for (int c = 0; c < 4; ++c) v[j][c] = pg[j] >= 0 ? __ldcs(row + 8 * c) : ML::zero();
    }
  };
  // the group-summed query of a pair, at the 4 x 4 dims this lane scores
  auto load_q = [&](int pr, float4 (&qs)[4]) {
    const int b = pr / p.Hkv, h = pr - b * p.Hkv;
    const __nv_bfloat16* qg = p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim;
#pragma unroll
    for (int c = 0; c < 4; ++c) qs[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int jh = 0; jh < p.g; ++jh) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint2 raw = __ldg(reinterpret_cast<const uint2*>(qg + jh * kHeadDim) + x + 8 * c);
        const float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.x));
        const float2 bb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.y));
        qs[c].x += a.x;
        qs[c].y += a.y;
        qs[c].z += bb.x;
        qs[c].w += bb.y;
      }
    }
  };
  auto advance = [&](int& pr, int& bk) {
    bk += U;
    if (bk >= nbp) {
      ++pr;
      bk = 0;
    }
  };

  int pair = (s0 * U) / nbp;
  int blk = s0 * U - pair * nbp;
  int nb = pair_nb(p, pair);
  float4 qs[4];
  load_q(pair, qs);
  int pg[RG];
  load_pages(pair, blk, nb, pg);
  Raw cur[RG][4];
  load_rows(pair, pg, cur);
  int npair = pair, nblk = blk;
  advance(npair, nblk);
  int nnb = s0 + 1 < s1 ? (npair == pair ? nb : pair_nb(p, npair)) : 0;
  int npg[RG];
  load_pages(npair, nblk, nnb, npg);
  for (int s = s0; s < s1; ++s) {
    const bool more = s + 1 < s1;
    Raw nxt[RG][4];
    load_rows(npair, npg, nxt);  // rows with no page (beyond nb, or none) load nothing
    int n2pair = npair, n2blk = nblk;
    advance(n2pair, n2blk);
    const int n2nb = s + 2 < s1 ? (n2pair == npair ? nnb : pair_nb(p, n2pair)) : 0;
    int n2pg[RG];
    load_pages(n2pair, n2blk, n2nb, n2pg);
    if (blk < nb) {
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        float d[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 m = ML::widen(cur[j][c]);
          d[c] = qs[c].x * m.x;
          d[c] = fmaf(qs[c].y, m.y, d[c]);
          d[c] = fmaf(qs[c].z, m.z, d[c]);
          d[c] = fmaf(qs[c].w, m.w, d[c]);
        }
        // lanes x (c 0), x+8 (c 1), x+16 (c 2), x+24 (c 3): pair xor 16, then xor 8
        float t = (d[0] + d[2]) + (d[1] + d[3]);
        t += __shfl_xor_sync(0xffffffffu, t, 4);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        const int r = blk + grp + 4 * j;
        if (x == 0 && r < nb) p.scores[(int64_t)pair * p.nbcap + r] = t * p.score_scale;
      }
    }
    if (npair != pair && more) load_q(npair, qs);
    pair = npair;
    blk = nblk;
    nb = nnb;
    npair = n2pair;
    nblk = n2blk;
    nnb = n2nb;
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      npg[j] = n2pg[j];
#pragma unroll
      for (int c = 0; c < 4; ++c) cur[j][c] = nxt[j][c];
    }
  }
  pdl_trigger_late();
}


// ---- dual means: before the exact top-k, make the pair's score row decide
// exactly.  The scan left s~_i, block i's score from its bf16 mean b_i; s_i
// is the score the fp32 scan computes from the fp32 mean m_i.  With q the
// summed query (the same fp32 values on both sides), d_i = m_i - b_i:
//  * the exact dot products differ by |q . d_i| <= |q|_2 |d_i|_2;
//  * each fp32 dot product (an fma chain and a pairing tree, depth 9) is
//    within 9 2^-24 / (1 - 9 2^-24) of sum |q||x|, at most |q|_2 |m_i|_2
//    (1 + 2^-8) for x = m_i or b_i: 2^-19.8 |q|_2 |m_i|_2 for the two;
//  * the product with the scale rounds each side once more (2^-23 of it);
//  * underflow adds at most 2^-141 to a dot product, 2^-149 to a product.
// The row's stored radius rho_i bounds |d_i|_2 + 2^-19 |m_i|_2 + 2^-60, so
//   |s~_i - s_i| <= e_i = scale (|q|_2 (1 + 2^-10) + 2^-59) rho_i,
// computed rounding up (|q|_2's fp32 sum of squares is within 2^-20 of it;
// the two 2^-59 floors make e_i >= scale 2^-118, above the underflow terms
// for the select's scale 1/sqrt(128)).
// With lower and upper bounds l_i = s~_i - e_i, u_i = s~_i + e_i over the
// candidates:
//  * T_L <= the kr-th largest l (the lower edge of the bin below the one
//    that holds it): a candidate with u < T_L has kr candidates strictly
//    above it and is out;
//  * T_U >= the kr-th largest u (the upper edge of the bin above the one
//    that holds it): a candidate with l > T_U has at most kr - 1 candidates
//    (itself included) that could reach it, so it is in;
//  * the rest, a narrow band around the boundary, is rescored from the fp32
//    rows with the fp32 scan's own arithmetic (the same per-lane fma chain;
//    the same pairing tree, xor 16, 8, 4, 2, 1, which a plain butterfly
//    reproduces exactly since addition is commutative).
// The row then holds the band's exact scores, a value above all of them for
// the candidates that are in and below all of them for those that are out,
// and the exact top-k that follows returns the fp32 selection bit for bit.
// Four barriers: bound ranges, histograms, the listing, the rescoring.
// The error scale of a pair, scale (|q|_2 (1 + 2^-10) + 2^-59) rounding
// up, from the summed query the scan used (qs: the lane's 4 dims).
__device__ __forceinline__ float pair_err_scale(const SelectParams& p, const float (&qs)[4]) {
  float qq = qs[0] * qs[0];
  qq = fmaf(qs[1], qs[1], qq);
  qq = fmaf(qs[2], qs[2], qq);
  qq = fmaf(qs[3], qs[3], qq);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) qq += __shfl_xor_sync(0xffffffffu, qq, off);
  return __fmul_ru(__fadd_ru(__fmul_ru(__fsqrt_ru(qq), 0x1.004p0f), 0x1p-59f), p.score_scale);
}

// The warp's minimum / maximum of v into slots[warp] (as float bits), and
// the fold of NW such slots.
__device__ __forceinline__ void warp_min_to(float v, uint32_t* slots) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, off));
  if ((threadIdx.x & 31) == 0) slots[threadIdx.x >> 5] = __float_as_uint(v);
}
__device__ __forceinline__ void warp_max_to(float v, uint32_t* slots) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  if ((threadIdx.x & 31) == 0) slots[threadIdx.x >> 5] = __float_as_uint(v);
}
// (every warp folds: lane l reads slot l, then a butterfly)
template <int NW>
__device__ __forceinline__ float fold_min(const uint32_t* slots) {
  const int lane = threadIdx.x & 31;
  float v = __uint_as_float(slots[lane < NW ? lane : 0]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
template <int NW>
__device__ __forceinline__ float fold_max(const uint32_t* slots) {
  const int lane = threadIdx.x & 31;
  float v = __uint_as_float(slots[lane < NW ? lane : 0]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// The rows of a pair's blocks in the dual means' arrays: logical, or (kPaged)
// per page through the table, then -1 for a page index outside the pool: a
// zero row, as the per-page scan reads it, and no radius.
template <bool kPaged>
struct DualRows {
  const int32_t* trow;  // per page: the sequence's table row
  int64_t base;         // logical: pair * nbcap; per page: the head h
  int Hkv, num_pages;
  __device__ __forceinline__ DualRows(const SelectParams& p, int64_t pair) {
    Hkv = p.Hkv;
    num_pages = p.mpages.num_pages;
    if constexpr (kPaged) {
      const int64_t b = pair / p.Hkv;
      trow = p.mpages.table + b * p.mpages.max_blocks;
      base = pair - b * p.Hkv;
    } else {
      trow = nullptr;
      base = pair * p.nbcap;
    }
  }
  __device__ __forceinline__ int64_t operator()(int i) const {
    if constexpr (!kPaged) {
      return base + i;
    } else {
      const int page = __ldcg(trow + i);
      return (page < 0 || page >= num_pages) ? -1 : (int64_t)page * Hkv + base;
    }
  }
};

// The fp32 scores of n candidates from their fp32 rows, with the fp32
// scan's own arithmetic: the listed indices list[0..n), or (all) every
// index lo..lo+n-1.  R rows in flight per warp; lane 0 hands each
// result to out(position, index, score).
template <int NT, bool kPaged, int R = 4, typename Out>
__device__ __forceinline__ void rescore_rows(const SelectParams& p, int64_t pair, const float (&qs)[4], int n, bool all,
                                             int lo, const uint32_t* list, Out out) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float4* f32 = reinterpret_cast<const float4*>(p.means_f32) + lane;
  const DualRows<kPaged> rows(p, pair);
  for (int e0 = warp * R; e0 < n; e0 += NW * R) {
    int idx[R];
    float4 m[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      idx[r] = e0 + r < n ? (all ? lo + e0 + r : (int)list[e0 + r]) : -1;
      if constexpr (kPaged) {
        const int64_t row = idx[r] >= 0 ? rows(idx[r]) : -1;
        m[r] = row >= 0 ? __ldg(f32 + row * (kHeadDim / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        m[r] = idx[r] >= 0 ? __ldg(f32 + rows(idx[r]) * (kHeadDim / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float d = qs[0] * m[r].x;
      d = fmaf(qs[1], m[r].y, d);
      d = fmaf(qs[2], m[r].z, d);
      d = fmaf(qs[3], m[r].w, d);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      if (idx[r] >= 0 && lane == 0) out(e0 + r, idx[r], d * p.score_scale);
    }
  }
}

// The bracket of a refinement: T_L and T_U from the histograms of the
// lower and upper bounds (sm.hist[0], sm.hist[1], when lbin / ubin), one
// bin wider than the bins found (the bin function is monotone and computed
// to a few ulps, so every bound in bin b lies within [lo + (b - 1) w,
// lo + (b + 2) w), w the bin width); -inf / +inf without a histogram.  The
// bin width range / 256 is range * 2^-8 with the same directed rounding (a
// multiply instead of a slow directed division).
__device__ __forceinline__ void bracket_from_hists(const int* hl, const int* hu, int kr, bool lbin, bool ubin,
                                                   float lmin, float lr, float umin, float ur, float& TL, float& TU) {
  const float kInf = __int_as_float(0x7f800000);
  TL = -kInf;
  TU = kInf;
  int bl, bu, above, c;
  if (lbin) {
    warp_find_bin(hl, kr, bl, above, c);  // every warp, same result
    if (bl >= 1) TL = __fadd_rd(lmin, __fmul_rd((float)(bl - 1), __fmul_rd(lr, 0x1p-8f)));
  }
  if (ubin) {
    warp_find_bin(hu, kr, bu, above, c);
    if (bu <= 253) TU = __fadd_ru(umin, __fmul_ru((float)(bu + 2), __fmul_ru(ur, 0x1p-8f)));
  }
}

template <int NT, bool kPaged>
__device__ __forceinline__ void refine_scores(const SelectParams& p, int64_t pair, float* row, const Cands& cd,
                                              TopkSmem<NT>& sm) {
  constexpr int NW = NT / 32;
  // candidates per thread: at most 8 below 4096 blocks (256 or 512
  // threads), 32 at 1024 threads (32768 blocks); beyond, every candidate is
  // rescored
  constexpr int kMaxIt = 32;
  const float kInf = __int_as_float(0x7f800000);
  const int tid = threadIdx.x, lane = tid & 31;
  float qs[4];
  pair_qsum(p, (int)pair, lane, qs);  // the fp32 scan's summed query, lane's 4 dims
  const float escale = pair_err_scale(p, qs);
  const float kInfE = __int_as_float(0x7f800000);
  const DualRows<kPaged> rows(p, pair);
  auto err = [&](int i) {  // a block with no page has no radius: undecided
    const int64_t r = rows(i);
    return r < 0 ? kInfE : __fmul_ru(escale, __ldg(p.radii + r));
  };
  uint32_t* slot_c = reinterpret_cast<uint32_t*>(sm.warp_cnt[0]);
  uint32_t* slot_d = reinterpret_cast<uint32_t*>(sm.warp_cnt[1]);
  uint32_t* slot_e = reinterpret_cast<uint32_t*>(sm.slot_cnt);

  // 1. ranges of the lower and the upper bounds, and the largest error
  float l0 = kInf, l1 = -kInf, u0 = kInf, u1 = -kInf, emax = 0.f;
  for (int i = cd.lo + tid; i <= cd.hi; i += NT) {
    const float e = err(i), sv = row[i];
    const float l = __fsub_rd(sv, e), u = __fadd_ru(sv, e);
    l0 = fminf(l0, l);
    l1 = fmaxf(l1, l);
    u0 = fminf(u0, u);
    u1 = fmaxf(u1, u);
    emax = fmaxf(emax, e);
  }
  warp_min_to(l0, sm.wmin);
  warp_max_to(l1, sm.wmax);
  warp_min_to(u0, slot_c);
  warp_max_to(u1, slot_d);
  warp_max_to(emax, slot_e);
  zero_hist(sm, 0);
  zero_hist(sm, 1);
  if (tid == 0) sm.list_n = 0;
  __syncthreads();
  const float lmin = fold_min<NW>(sm.wmin), lmax = fold_max<NW>(sm.wmax);
  const float umin = fold_min<NW>(slot_c), umax = fold_max<NW>(slot_d), emx = fold_max<NW>(slot_e);
  const float lr = lmax - lmin, li = 256.f / lr, ur = umax - umin, ui = 256.f / ur;
  const bool lbin = isfinite(lmin) && isfinite(lmax) && lr > 0.f && isfinite(lr) && isfinite(li);
  const bool ubin = isfinite(umin) && isfinite(umax) && ur > 0.f && isfinite(ur) && isfinite(ui);
  auto lbin_of = [&](float l) { return min((int)((l - lmin) * li), 255); };
  auto ubin_of = [&](float u) { return min((int)((u - umin) * ui), 255); };

  // 2. T_L and T_U; every candidate undecided when the bounds do not spread
  float TL = -kInf, TU = kInf;
  if (lbin || ubin) {
    for (int i = cd.lo + tid; i <= cd.hi; i += NT) {
      const float e = err(i), sv = row[i];
      if (lbin) atomicAdd(&sm.hist[0][hidx(lbin_of(__fsub_rd(sv, e)))], 1);
      if (ubin) atomicAdd(&sm.hist[1][hidx(ubin_of(__fadd_ru(sv, e)))], 1);
    }
    __syncthreads();
    bracket_from_hists(sm.hist[0], sm.hist[1], cd.kr, lbin, ubin, lmin, lr, umin, ur, TL, TU);
  }
  // a rescored score lies within [T_L - 2 emax, T_U + 2 emax] (to a few ulps,
  // far below emax): the decided candidates go outside [T_L - 3 emax,
  // T_U + 3 emax]
  const float below_all = nextafterf(__fsub_rd(TL, __fmul_ru(3.f, emx)), -kInf);
  const float above_all = nextafterf(__fadd_ru(TU, __fmul_ru(3.f, emx)), kInf);
  const bool bracketed = isfinite(below_all) && isfinite(above_all);

  // 3. in (l > T_U), out (u < T_L), or undecided: listed, one reservation per
  //    warp; the decided ones written now
  const bool fits = bracketed && cd.hi - cd.lo + 1 <= kMaxIt * NT;
  for (int j = 0, i = cd.lo + tid; fits && j < kMaxIt; ++j, i += NT) {
    bool open = false;
    if (i <= cd.hi) {
      const float e = err(i), sv = row[i];
      if (__fsub_rd(sv, e) > TU)
        row[i] = above_all;
      else if (__fadd_ru(sv, e) < TL)
        row[i] = below_all;
      else
        open = true;
    }
    const unsigned m = __ballot_sync(0xffffffffu, open);
    if (m) {
      int slot = 0;
      if (lane == 0) slot = atomicAdd(&sm.list_n, __popc(m));
      slot = __shfl_sync(0xffffffffu, slot, 0) + __popc(m & ((1u << lane) - 1u));
      if (open && slot < kListCap) sm.list[slot] = (uint32_t)i;
    }
    if (__all_sync(0xffffffffu, i + NT > cd.hi)) break;
  }
  __syncthreads();
  const int nlist = sm.list_n;
  // too many to list, or no finite bracket: rescore every candidate (the
  // decided ones then get their exact scores back, which is as good)
  const bool all = !fits || nlist > kListCap;

  // 4. rescore them from the fp32 rows
  rescore_rows<NT, kPaged>(p, pair, qs, all ? cd.hi - cd.lo + 1 : nlist, all, cd.lo, sm.list,
                   [&](int, int i, float v) { row[i] = v; });
  __syncthreads();  // the row is final before the top-k reads it
}

// ---- dual means, register path (nb <= KPT NT): the refinement above and
// the exact top-k in one pass over registers.  Every candidate's bf16
// score and radius is loaded once (thread t: blocks u NT + t, the top-k's
// own layout); the bounds, the histograms and the in / out / band split
// run from registers; the band is rescored from the fp32 rows, spread over
// all warps through a shared list, and its exact keys come back through
// shared memory.  The n_in candidates that are in take n_in of the kr
// places and lie above every band score, so the threshold is the
// (kr - n_in)-th largest exact key of the band: with at most kRankCap band
// keys it is found by ranking them pairwise, and the emit follows.  A wider
// band (or no finite bracket, or a band beyond the list, when every
// candidate is rescored) goes to the generic search over the refined keys.
template <int NT, int KPT, bool kPaged>
__device__ __forceinline__ void refine_topk_regs(const SelectParams& p, int64_t pair, int nb, const Cands& cd, int k,
                                                 int32_t* sel, uint32_t* skey, TopkSmem<NT>& sm) {
  constexpr int NW = NT / 32;
  const float kInf = __int_as_float(0x7f800000);
  const int tid = threadIdx.x, lane = tid & 31;
  const int kr = cd.kr;
  if (kr == 0) {  // only the forced blocks are kept
    pdl_wait();
    pdl_trigger_early();
    const uint32_t none[KPT] = {};
    emit_regs<NT, KPT>(none, nb, cd, k, 0xFFFFFFFFu, 0, sel, sm, p.dev_status);
    return;
  }
  // the radii and the query, before the wait: see select_topk_kernel (a
  // block with no page has no radius: undecided)
  float ev[KPT];
  const DualRows<kPaged> rows(p, pair);
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int i = u * NT + tid;
    if constexpr (kPaged) {
      const int64_t r = cd.has(i) ? rows(i) : -2;
      ev[u] = r >= 0 ? __ldcg(p.radii + r) : r == -1 ? kInf : 0.f;
    } else {
      ev[u] = cd.has(i) ? __ldcg(p.radii + rows(i)) : 0.f;
    }
  }
  __shared__ float4 qsh[kHeadDim / 4];  // the summed query, for the rescoring
  float escale;
  {
    float qs[4];
    pair_qsum(p, (int)pair, lane, qs);  // the fp32 scan's summed query, lane's 4 dims
    escale = pair_err_scale(p, qs);
    if (tid < 32) qsh[lane] = make_float4(qs[0], qs[1], qs[2], qs[3]);  // read after the next barrier
  }
  pdl_wait();  // the scores come from the scan kernel
  pdl_trigger_early();
  const float* srow = p.scores + pair * p.nbcap;
  float sv[KPT];
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int i = u * NT + tid;
    sv[u] = cd.has(i) ? __ldcg(srow + i) : 0.f;
  }
  uint32_t* slot_e = reinterpret_cast<uint32_t*>(sm.slot_cnt);

  // 1. the range of the bounds (smallest lower, largest upper), and the
  //    largest error
  float l0 = kInf, u1 = -kInf, emax = 0.f;
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    ev[u] = __fmul_ru(escale, ev[u]);
    if (cd.has(u * NT + tid)) {
      l0 = fminf(l0, __fsub_rd(sv[u], ev[u]));
      u1 = fmaxf(u1, __fadd_ru(sv[u], ev[u]));
      emax = fmaxf(emax, ev[u]);
    }
  }
  warp_min_to(l0, sm.wmin);
  warp_max_to(u1, sm.wmax);
  warp_max_to(emax, slot_e);
  zero_hist(sm, 0);
  if (tid == 0) {
    sm.band_n = 0;
    sm.in_n = 0;
  }
  __syncthreads();
  float lo, hi, emx;
  {  // the three folds interleaved (lane l reads slot l, then one butterfly)
    const int sl = lane < NW ? lane : 0;
    lo = __uint_as_float(sm.wmin[sl]);
    hi = __uint_as_float(sm.wmax[sl]);
    emx = __uint_as_float(slot_e[sl]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      emx = fmaxf(emx, __shfl_xor_sync(0xffffffffu, emx, off));
    }
  }
  const float range = hi - lo, inv = 256.f / range;
  const bool binned = isfinite(lo) && isfinite(hi) && range > 0.f && isfinite(range) && isfinite(inv);

  // 2. T_L and T_U from two histograms over one range, packed in one word
  //    per bin (lower bounds in the low 16 bits, upper bounds in the high):
  //    a candidate whose bounds share a bin, the common case, takes one
  //    atomic.  Bin edges one bin wider, as in refine_scores.
  float TL = -kInf, TU = kInf;
  if (binned) {
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      if (cd.has(u * NT + tid)) {
        const int bl = min((int)((__fsub_rd(sv[u], ev[u]) - lo) * inv), 255);
        const int bu = min((int)((__fadd_ru(sv[u], ev[u]) - lo) * inv), 255);
        if (bl == bu) {
          atomicAdd(&sm.hist[0][hidx(bl)], 0x10001);
        } else {
          atomicAdd(&sm.hist[0][hidx(bl)], 1);
          atomicAdd(&sm.hist[0][hidx(bu)], 0x10000);
        }
      }
    }
    __syncthreads();
    int bl, bu;
    warp_find_bins_packed(sm.hist[0], kr, bl, bu);  // every warp, same result
    if (bl >= 1) TL = __fadd_rd(lo, __fmul_rd((float)(bl - 1), __fmul_rd(range, 0x1p-8f)));
    if (bu <= 253) TU = __fadd_ru(lo, __fmul_ru((float)(bu + 2), __fmul_ru(range, 0x1p-8f)));
  }
  const float below_all = nextafterf(__fsub_rd(TL, __fmul_ru(3.f, emx)), -kInf);
  const float above_all = nextafterf(__fadd_ru(TU, __fmul_ru(3.f, emx)), kInf);
  const bool bracketed = isfinite(below_all) && isfinite(above_all);

  // 3. in (l > T_U), out (u < T_L), or in the band: the warp's ballots
  //    first, then one reservation of list slots and one count of the in
  //    ones per warp, then the band indices listed
  unsigned inm = 0u, bandm = 0u;
  if (bracketed) {
    unsigned mo[KPT];
    int nband = 0, nin = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int i = u * NT + tid;
      bool in = false, open = false;
      if (cd.has(i)) {
        if (__fsub_rd(sv[u], ev[u]) > TU)
          in = true;
        else if (!(__fadd_ru(sv[u], ev[u]) < TL))
          open = true;
      }
      mo[u] = __ballot_sync(0xffffffffu, open);
      nband += __popc(mo[u]);
      nin += __popc(__ballot_sync(0xffffffffu, in));
      inm |= (unsigned)in << u;
      bandm |= (unsigned)open << u;
    }
    int slot = 0;
    if (lane == 0) {
      if (nband) slot = atomicAdd(&sm.band_n, nband);
      if (nin) atomicAdd(&sm.in_n, nin);
    }
    slot = __shfl_sync(0xffffffffu, slot, 0);
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int at = slot + __popc(mo[u] & ((1u << lane) - 1u));
      if (((bandm >> u) & 1u) && at < kListCap) sm.list[at] = (uint32_t)(u * NT + tid);
      slot += __popc(mo[u]);
    }
  }
  __syncthreads();
  const int nlist = sm.band_n, n_in = sm.in_n;
  const bool all = !bracketed || nlist > kListCap;  // then every candidate is rescored

  // 4. the band's (or every candidate's) exact keys, from the fp32 rows
  const float4 q4 = qsh[lane];
  const float qs[4] = {q4.x, q4.y, q4.z, q4.w};
  rescore_rows<NT, kPaged, KIN_RESCORE_ROWS>(p, pair, qs, all ? cd.hi - cd.lo + 1 : nlist, all, cd.lo, sm.list,
                                     [&](int j, int i, float v) {
    const uint32_t kx = key_of_bits(__float_as_uint(v));
    skey[i] = kx;
    if (!all) sm.list[j] = kx;  // the slot this warp just read its index from
  });
  __syncthreads();
  const uint32_t k_in = key_of_bits(__float_as_uint(above_all)), k_out = key_of_bits(__float_as_uint(below_all));
  uint32_t key[KPT];
#pragma unroll
  for (int u = 0; u < KPT; ++u) {
    const int i = u * NT + tid;
    key[u] = !cd.has(i) ? 0u : (all || ((bandm >> u) & 1u)) ? skey[i] : ((inm >> u) & 1u) ? k_in : k_out;
  }

  // 5. the threshold among the band, and the emit
  const int need = kr - n_in;
  if (!all && nlist <= kRankCap && need >= 1 && need <= nlist) {
    if (KIN_RANK_SPLIT && nlist <= NT / 4)
      rank_keys_split4<NT>(nlist, need, sm);  // ends with a barrier
    else
      rank_keys(0, nlist, need, sm);  // ends with a barrier
    emit_regs<NT, KPT>(key, nb, cd, k, sm.thresh, sm.thresh_take, sel, sm, p.dev_status);
  } else {
    topk_regs_keys<NT, KPT>(key, nb, cd, k, sel, skey, sm, p.dev_status);
  }
}

// ---- kernel 2: one CTA of NT threads per pair: dense shortcut, bad-length
// flag, or the exact top-k over the scores the scan left in workspace
// (L2-resident), in registers when nb <= 8 NT.
template <int NT, bool kRefine, bool kPaged = false>
__global__ void __launch_bounds__(NT, 1024 / NT) select_topk_kernel(SelectParams p) {
  // 4 keys per thread need 8 warps (the emit's slot layout): a 128-thread CTA
  // (chosen only for rows of at most 8 NT = 1024 blocks) keeps 8 per thread
  constexpr bool kKpt4 = NT >= 256;
  extern __shared__ uint32_t skey[];  // [nbcap] keys (rows beyond 8 NT blocks: then nbcap bytes of bins)
  __shared__ TopkSmem<NT> sm;
  const int tid = threadIdx.x;
  const int64_t pair = blockIdx.x;
  const int b = (int)(pair / p.Hkv);
  const int k = p.k;
  int32_t* sel = p.sel_idx + pair * k;
  if constexpr (kRefine) {
    // The lengths, the radii, the query and the page table are written by
    // work that completed before the scan's own wait returned (the scan
    // writes only scores), and this grid starts after every scan CTA passed
    // that wait: they are read from L2 (ld.global.cg, the point of
    // coherence) before this grid's wait, while the scan drains.  The register paths wait
    // inside, before their first score load.
    const int L = __ldcg(p.seq_lens + b);
    const int nb = (L >= 1 && L <= p.Lcap) ? (L + p.bs - 1) / p.bs : 0;
    if (nb > k && nb <= 8 * NT) {
      const Cands cd{1, nb - 2, k - 2};  // blocks 0 and nb - 1 forced
      bool done = false;
      if constexpr (kKpt4) {
        if (nb <= 4 * NT) {
          refine_topk_regs<NT, 4, kPaged>(p, pair, nb, cd, k, sel, skey, sm);
          done = true;
        }
      }
      if (!done) refine_topk_regs<NT, 8, kPaged>(p, pair, nb, cd, k, sel, skey, sm);
      if (tid == 0) p.sel_cnt[pair] = k;
      return;
    }
    if (nb > k && !kPaged) {  // the memory path: warm L2 with this pair's radii and query rows
      const char* rb = reinterpret_cast<const char*>(p.radii + pair * p.nbcap);
      for (int t = tid; t < (p.nbcap * 4 + 127) / 128; t += NT) prefetch_l2(rb + t * 128);
      const int h = (int)(pair - (int64_t)b * p.Hkv);
      const char* qg = reinterpret_cast<const char*>(p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim);
      if (tid < 2 * p.g) prefetch_l2(qg + tid * 128);  // g rows of 256 bytes
    }
  }
  pdl_wait();  // scores come from the scan kernel
  pdl_trigger_early();
  const int L = __ldg(p.seq_lens + b);
  if (L < 1 || L > p.Lcap) {
    for (int i = tid; i < k; i += NT) sel[i] = -1;
    if (tid == 0) {
      p.sel_cnt[pair] = 0;
      set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    }
    return;
  }
  const int nb = (L + p.bs - 1) / p.bs;
  if (nb <= k) {  // the budget covers every block: dense
    for (int i = tid; i < k; i += NT) sel[i] = i < nb ? i : -1;
    if (tid == 0) p.sel_cnt[pair] = nb;
    return;
  }
  const uint32_t* row = reinterpret_cast<const uint32_t*>(p.scores + pair * p.nbcap);
  const Cands cd{1, nb - 2, k - 2};  // blocks 0 and nb - 1 forced
  if constexpr (kRefine) {
    refine_scores<NT, kPaged>(p, pair, p.scores + pair * p.nbcap, cd, sm);
    topk_memory<NT>(row, nb, cd, k, sel, skey, p.nbcap, const_cast<uint32_t*>(row), sm, p.dev_status);
  } else if (kKpt4 && nb <= 4 * NT) {
    if constexpr (kKpt4) topk_regs<NT, 4>(row, nb, cd, k, sel, skey, sm, p.dev_status);
  } else if (nb <= 8 * NT) {
    topk_regs<NT, 8>(row, nb, cd, k, sel, skey, sm, p.dev_status);
  } else {
    topk_memory<NT>(row, nb, cd, k, sel, skey, p.nbcap, const_cast<uint32_t*>(row), sm, p.dev_status);
  }
  if (tid == 0) p.sel_cnt[pair] = k;
}

// ---- token-level top-k: one 1024-thread CTA per (sequence, query head)
// keeps the k tokens with the largest logits (ties to the lower index,
// nothing forced), ascending, -1 padded; every token when k >= L.
constexpr int kTokTopkThreads = 1024;
constexpr int kTokKeyCap = 32768;  // keys kept in shared memory up to this many tokens

__global__ void __launch_bounds__(kTokTopkThreads, 1) token_topk_kernel(TokenParams p) {
  extern __shared__ uint32_t skey[];  // [min(Lcap, kTokKeyCap)] keys, then as many bytes of bins
  __shared__ TopkSmem<kTokTopkThreads> sm;
  const int tid = threadIdx.x;
  pdl_wait();  // the logits come from the logits kernel (no early trigger: see token_logits_kernel)
  const int64_t row_id = blockIdx.x;  // b * Hq + query head
  const int b = (int)(row_id / p.Hq);
  const int k = p.kt;
  int32_t* sel = p.sel + row_id * k;
  const int L = __ldg(p.seq_lens + b);
  if (L < 1 || L > p.Lcap) {
    for (int i = tid; i < k; i += kTokTopkThreads) sel[i] = -1;
    if (tid == 0) {
      p.cnt[row_id] = 0;
      set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    }
    return;
  }
  if (L <= k) {
    for (int i = tid; i < k; i += kTokTopkThreads) sel[i] = i < L ? i : -1;
    if (tid == 0) p.cnt[row_id] = L;
    return;
  }
  const uint32_t* row = reinterpret_cast<const uint32_t*>(p.logits + row_id * p.Lcap);
  const Cands cd{0, L - 1, k};
  if (L <= 4 * kTokTopkThreads) topk_regs<kTokTopkThreads, 4>(row, L, cd, k, sel, skey, sm, p.dev_status);
  else if (L <= 8 * kTokTopkThreads) topk_regs<kTokTopkThreads, 8>(row, L, cd, k, sel, skey, sm, p.dev_status);
  else
    topk_memory<kTokTopkThreads>(row, L, cd, k, sel, skey, min(p.Lcap, kTokKeyCap), p.key_scratch + row_id * p.Lcap, sm,
                                 p.dev_status);
  if (tid == 0) p.cnt[row_id] = k;
}

cudaError_t launch_token_topk(const TokenParams& p, cudaStream_t s) {
  const size_t cap = (size_t)(p.Lcap < kTokKeyCap ? p.Lcap : kTokKeyCap);
  const size_t smem = cap * sizeof(uint32_t) + ((cap + 3) & ~size_t(3));  // keys, then their bins
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(token_topk_kernel), 5, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(token_topk_kernel, dim3(p.B * p.Hq), dim3(kTokTopkThreads), smem, s, p);
}

// Threads per top-k CTA: enough for 4 keys per thread (up to 4096 blocks),
// halved (8 keys per thread) while the pairs would need more than one wave
// of CTAs (the launch bounds allow 1024 / NT CTAs per SM), down to 128.
int topk_threads(int nbcap, int64_t pairs) {
  int nt = nbcap <= 1024 ? 256 : nbcap <= 2048 ? 512 : 1024;
  while (nt > 128 && nbcap <= 8 * (nt / 2) && pairs > (int64_t)device_sm_count() * (1024 / nt)) nt /= 2;
  return nt;
}

template <int NT>
cudaError_t launch_topk(const SelectParams& p, cudaStream_t s) {
  // keys (when they do not fit in registers: then also their bins)
  const size_t smem = (size_t)p.nbcap * sizeof(uint32_t) + (p.nbcap > 8 * NT ? ((size_t)p.nbcap + 3) & ~size_t(3) : 0);
  if (p.refine && p.mpages.table) {  // dual means per page
    if (smem > 16 * 1024) {
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(select_topk_kernel<NT, true, true>),
                                        NT <= 256 ? 12 : NT == 512 ? 13 : 14, smem);
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(select_topk_kernel<NT, true, true>, dim3(p.B * p.Hkv), dim3(NT), smem, s, p);
  }
  if (p.refine) {
    if (smem > 16 * 1024) {
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(select_topk_kernel<NT, true>),
                                        NT <= 256 ? 8 : NT == 512 ? 9 : 10, smem);
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(select_topk_kernel<NT, true>, dim3(p.B * p.Hkv), dim3(NT), smem, s, p);
  }
  if (smem > 16 * 1024) {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(select_topk_kernel<NT, false>),
                                      NT <= 256 ? 0 : NT == 512 ? 2 : 3, smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(select_topk_kernel<NT, false>, dim3(p.B * p.Hkv), dim3(NT), smem, s, p);
}

// The selection when the budget covers every block of every sequence the
// dims allow (k >= nbcap): nothing to score.  Every block is kept (sel_cnt
// nb), or sel_cnt 0 and a row of -1 for a length outside [1, Lcap]
// (flagged), one thread per output entry.
__global__ void __launch_bounds__(256) select_dense_kernel(SelectParams p) {
  pdl_wait();
  pdl_trigger_early();
  const int64_t total = (int64_t)p.B * p.Hkv * p.k;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t pair = idx / p.k;
    const int j = (int)(idx - pair * p.k);
    const int L = __ldg(p.seq_lens + pair / p.Hkv);
    const bool bad = L < 1 || L > p.Lcap;
    const int nb = bad ? 0 : (L + p.bs - 1) / p.bs;
    p.sel_idx[idx] = j < nb ? j : -1;
    if (j == 0) {
      p.sel_cnt[pair] = nb;
      if (bad) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    }
  }
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t s) {
  const int64_t resident = (int64_t)device_sm_count() * KIN_SEL_CTAS_PER_SM;
  if (p.k >= p.nbcap) {  // every sequence's blocks fit the budget
    const int64_t want = ((int64_t)p.B * p.Hkv * p.k + 255) / 256;
    const int grid = (int)(want < 4 * resident ? want : 4 * resident);
    return launch_pdl(select_dense_kernel, dim3(grid), dim3(256), 0, s, p);
  }
  const int64_t rows = (int64_t)p.B * p.Hkv * p.nbcap;
  if (p.refine) {  // dual means: the bf16 rows' scan, then the refining top-k
    cudaError_t e;
    if (p.mpages.table) {  // per page: the per-page scan of the bf16 rows
      const int64_t want = (rows + kSelWarps * 2 * kSelU * 4 - 1) / (kSelWarps * 2 * kSelU * 4);
      const int grid = (int)(want < resident ? (want > 0 ? want : 1) : resident);
      e = launch_pdl(select_scan_paged_kernel<true>, dim3(grid), dim3(kSelThreads), 0, s, p);
    } else {
      constexpr int V = KIN_DUAL_SCAN_V, C = KIN_DUAL_SCAN_CTAS;
      const int64_t res = (int64_t)device_sm_count() * C;
      const int64_t want = (rows + kSelWarps * 2 * V * 4 - 1) / (kSelWarps * 2 * V * 4);  // >= 4 steps per warp
      const int grid = (int)(want < res ? (want > 0 ? want : 1) : res);
      e = launch_pdl(select_scan_dual_kernel<V, C>, dim3(grid), dim3(kSelThreads), 0, s, p);
    }
    if (e != cudaSuccess) return e;
    switch (topk_threads(p.nbcap, (int64_t)p.B * p.Hkv)) {
      case 128: return launch_topk<128>(p, s);
      case 256: return launch_topk<256>(p, s);
      case 512: return launch_topk<512>(p, s);
      default: return launch_topk<1024>(p, s);
    }
  }
  const int u = p.means_bf16 ? 2 * kSelU : kSelU;
  const int64_t want = (rows + kSelWarps * u * 4 - 1) / (kSelWarps * u * 4);  // >= 4 steps per warp
  const int grid = (int)(want < resident ? (want > 0 ? want : 1) : resident);
  const dim3 gd(grid), bd(kSelThreads);
  cudaError_t e;
  if (p.mpages.table)
    e = p.means_bf16 ? launch_pdl(select_scan_paged_kernel<true>, gd, bd, 0, s, p)
                     : launch_pdl(select_scan_paged_kernel<false>, gd, bd, 0, s, p);
  else
    e = p.means_bf16 ? launch_pdl(select_scan_kernel<true, 2 * kSelU>, gd, bd, 0, s, p)
                     : launch_pdl(select_scan_kernel<false, kSelU>, gd, bd, 0, s, p);
  if (e != cudaSuccess) return e;
  switch (topk_threads(p.nbcap, (int64_t)p.B * p.Hkv)) {
    case 128: return launch_topk<128>(p, s);
    case 256: return launch_topk<256>(p, s);
    case 512: return launch_topk<512>(p, s);
    default: return launch_topk<1024>(p, s);
  }
}

}  // namespace kin
