// kin_select.cu -- group-summed block scores (HBM scan of the fp32 block
// means) fused with an exact per-(batch, kv-head) block top-k.
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
//  2. select_topk_kernel, one CTA per pair, loads the pair's scores as
//     order-preserving uint32 keys into shared memory and runs an exact
//     radix select (see topk_emit): the first block and the block holding
//     the newest token are always kept, ties go to the lower index, and the
//     kept indices leave ascending.
#include "kin_internal.cuh"

namespace kin {

#ifndef KIN_SEL_UNROLL
#define KIN_SEL_UNROLL 8
#endif
#ifndef KIN_SEL_CTAS_PER_SM
#define KIN_SEL_CTAS_PER_SM 2
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

constexpr int kListCap = 4096;  // candidates kept in a compact list after the first pass

struct SelectSmem {
  int hist[2][256];            // double-buffered radix histogram
  int list[kListCap];          // indices whose key matches the first chosen digit
  int list_n;
  int warp_cnt[3][kSelWarps];  // per-warp counts: forced, > T, == T
  int digit, above, bin;
};

// Warp 0: the digit (descending) whose bin holds the kr-th largest key of the
// histogram, the count of keys in higher digits, and the bin's own count.
__device__ __forceinline__ void find_digit(const int* hist, int kr, SelectSmem& sm) {
  const int lane = threadIdx.x & 31;
  int cnt[8], tot = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    cnt[u] = hist[255 - (lane * 8 + u)];
    tot += cnt[u];
  }
  int inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  const int excl = inc - tot;
  if (excl < kr && kr <= inc) {
    int run = excl;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (run + cnt[u] >= kr) {
        sm.digit = 255 - (lane * 8 + u);
        sm.above = run;
        sm.bin = cnt[u];
        break;
      }
      run += cnt[u];
    }
  }
}

// Exact top-(k-2) over keys[1..nb-2] plus the forced blocks 0 and nb-1,
// written ascending to sel[0..k).  keys live in shared memory; hist[0] must
// already hold the histogram of the candidates' top byte and hist[1] zeros.
//  * Radix select, up to 4 passes of 8 bits from the top: each pass finds the
//    digit whose bin holds the kr-th largest remaining key.  After the first
//    pass the indices matching the chosen prefix go to a compact list, so the
//    later passes visit only those.  A pass whose bin holds exactly the keys
//    still needed ends the search: they are all taken.  The result is a
//    prefix T over the top `mask` bits and kr, the number of keys equal to T
//    (under the mask) to take.
//  * Emit with ballots: warp w owns a contiguous index range; one pass counts
//    its forced / greater / equal keys, one barrier publishes the counts, and
//    a second pass writes the taken indices in order (keys equal to T under
//    the mask are taken in index order while their rank is below kr: ties go
//    to lower indices, and indices leave ascending).
__device__ __forceinline__ void topk_emit(const uint32_t* keys, int nb, int k, int32_t* sel,
                                          SelectSmem& sm, int32_t* dev_status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, mask = 0u;
  int kr = k - 2;
  bool use_list = false;
  if (kr == 0) {  // budget of two: only the forced blocks; no candidate key can pass
    prefix = 0xFFFFFFFFu;
    mask = 0xFFFFFFFFu;
  }
#pragma unroll 1
  for (int pass = 0; pass < 4 && kr > 0; ++pass) {
    const int shift = 24 - 8 * pass;
    int* hist = sm.hist[pass & 1];
    if (pass > 0) {
      if (pass == 1) {  // visit every key once more, keep the matching indices
        if (tid == 0) sm.list_n = 0;
        __syncthreads();
        for (int base = 0; base < nb; base += kSelThreads) {  // uniform trip count per warp
          const int i = base + tid;
          const uint32_t key = i < nb ? keys[i] : 0u;
          const bool match = i >= 1 && i <= nb - 2 && (key & mask) == prefix;
          if (match) atomicAdd(&hist[(key >> shift) & 0xFFu], 1);
          if (use_list) {  // one list reservation per warp, lanes take slots in order
            const unsigned m = __ballot_sync(0xffffffffu, match);
            int slot = 0;
            if (lane == 0 && m) slot = atomicAdd(&sm.list_n, __popc(m));
            slot = __shfl_sync(0xffffffffu, slot, 0);
            if (match) sm.list[slot + __popc(m & ((1u << lane) - 1u))] = i;
          }
        }
      } else if (use_list) {
        for (int j = tid; j < sm.list_n; j += kSelThreads) {
          const uint32_t key = keys[sm.list[j]];
          if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1);
        }
      } else {
        for (int i = 1 + tid; i < nb - 1; i += kSelThreads) {
          const uint32_t key = keys[i];
          if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1);
        }
      }
      sm.hist[(pass + 1) & 1][tid] = 0;  // the other buffer is free: ready it for the next pass
      __syncthreads();
    }
    if (warp == 0) find_digit(hist, kr, sm);
    if (pass == 0) sm.hist[1][tid] = 0;
    __syncthreads();
    prefix |= (uint32_t)sm.digit << shift;
    mask |= 0xFFu << shift;
    kr -= sm.above;
    if (pass == 0) use_list = sm.bin <= kListCap;
    const bool done = sm.bin == kr;  // every key in the bin is taken
    __syncthreads();                 // all threads have read digit/above/bin
    if (done) break;
  }

  // ---- emit
  const int span = ((nb + kSelWarps - 1) / kSelWarps + 31) & ~31;  // per-warp range, whole batches
  const int w0 = min(warp * span, nb), w1 = min(w0 + span, nb);
  const unsigned lt = (1u << lane) - 1u;
  int n_forced = 0, n_gt = 0, n_eq = 0;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const bool in = i < w1;
    const uint32_t key = in ? (keys[i] & mask) : 0u;
    const bool cand = in && i >= 1 && i <= nb - 2;
    n_forced += __popc(__ballot_sync(0xffffffffu, in && !cand));
    n_gt += __popc(__ballot_sync(0xffffffffu, cand && key > prefix));
    n_eq += __popc(__ballot_sync(0xffffffffu, cand && key == prefix));
  }
  if (lane == 0) {
    sm.warp_cnt[0][warp] = n_forced;
    sm.warp_cnt[1][warp] = n_gt;
    sm.warp_cnt[2][warp] = n_eq;
  }
  __syncthreads();
  int eq_base = 0, out_base = 0;
  for (int w = 0; w < warp; ++w) {
    const int e = sm.warp_cnt[2][w];
    const int eq_take = min(max(kr - eq_base, 0), e);  // equal keys warp w takes
    out_base += sm.warp_cnt[0][w] + sm.warp_cnt[1][w] + eq_take;
    eq_base += e;
  }
  int pos = out_base, eq_rank = eq_base;
  for (int base = w0; base < w1; base += 32) {
    const int i = base + lane;
    const bool in = i < w1;
    const uint32_t key = in ? (keys[i] & mask) : 0u;
    const bool cand = in && i >= 1 && i <= nb - 2;
    const bool eq = cand && key == prefix;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const bool take = (in && !cand) || (cand && key > prefix) || (eq && eq_rank + __popc(eq_mask & lt) < kr);
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = pos + __popc(take_mask & lt);
      if (o < k) sel[o] = i;  // never write past the pair's row
    }
    pos += __popc(take_mask);
    eq_rank += __popc(eq_mask);
  }
  // self-check: exactly k blocks were emitted (the last warp ends at k)
  if (warp == kSelWarps - 1 && lane == 0 && pos != k) set_status(dev_status, KIN_ERR_DEVICE_DATA);
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
  const int b = pair / p.Hkv, h = pair - b * p.Hkv;
  const __nv_bfloat16* qg = p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim;
  o[0] = o[1] = o[2] = o[3] = 0.f;
  for (int j = 0; j < p.g; ++j) {
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(qg + j * kHeadDim) + lane);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.x));
    float2 bb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.y));
    o[0] += a.x;
    o[1] += a.y;
    o[2] += bb.x;
    o[3] += bb.y;
  }
}

__global__ void __launch_bounds__(kSelThreads, KIN_SEL_CTAS_PER_SM) select_scan_kernel(SelectParams p) {
  pdl_wait();  // means, lengths and q come from earlier work on the stream
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kSelWarps;
  const int gw = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int nbp = (p.nbcap + kSelU - 1) / kSelU * kSelU;
  const int steps = p.B * p.Hkv * (nbp / kSelU);
  const int per = (steps + nwarps - 1) / nwarps;
  const int s0 = gw * per, s1 = min(s0 + per, steps);
  if (s0 >= s1) {
    pdl_trigger();
    return;
  }

  // step s covers slots s*U .. s*U+U-1 of pair (s*U) / nbp
  int pair = (s0 * kSelU) / nbp;
  int blk = s0 * kSelU - pair * nbp;
  int nb = pair_nb(p, pair);
  float qs[4];
  pair_qsum(p, pair, lane, qs);
  const float4* mrow = reinterpret_cast<const float4*>(p.means) + lane;
  auto row_ptr = [&](int pr, int bk) { return mrow + ((int64_t)pr * p.nbcap + bk) * (kHeadDim / 4); };

  float4 cur[kSelU];
#pragma unroll
  for (int u = 0; u < kSelU; ++u)
    cur[u] = blk + u < nb ? __ldcs(row_ptr(pair, blk + u)) : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = s0; s < s1; ++s) {
    // the next step's rows fly during this step's math
    int npair = pair, nblk = blk + kSelU, nnb = nb;
    if (nblk >= nbp) {
      npair = pair + 1;
      nblk = 0;
      nnb = s + 1 < s1 ? pair_nb(p, npair) : 0;
    }
    const bool more = s + 1 < s1;
    float4 nxt[kSelU];
#pragma unroll
    for (int u = 0; u < kSelU; ++u)
      nxt[u] = more && nblk + u < nnb ? __ldcs(row_ptr(npair, nblk + u)) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (blk < nb) {
      float d[kSelU];
#pragma unroll
      for (int u = 0; u < kSelU; ++u) {
        d[u] = qs[0] * cur[u].x;
        d[u] = fmaf(qs[1], cur[u].y, d[u]);
        d[u] = fmaf(qs[2], cur[u].z, d[u]);
        d[u] = fmaf(qs[3], cur[u].w, d[u]);
      }
      const float tot = warp_sum_rows<kSelU>(d, lane);
      const int row = lane / (32 / kSelU);
      if ((lane & (32 / kSelU - 1)) == 0 && blk + row < nb)
        p.scores[(int64_t)pair * p.nbcap + blk + row] = tot * p.score_scale;
    }
    if (npair != pair && more) pair_qsum(p, npair, lane, qs);
    pair = npair;
    blk = nblk;
    nb = nnb;
#pragma unroll
    for (int u = 0; u < kSelU; ++u) cur[u] = nxt[u];
  }
  pdl_trigger();
}

// ---- kernel 2: one CTA per pair: dense shortcut, bad-length flag, or the
// exact top-k over the scores the scan left in workspace (L2-resident).
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(SelectParams p) {
  extern __shared__ uint32_t skey[];  // [nbcap]
  __shared__ SelectSmem sm;
  const int tid = threadIdx.x;
  pdl_wait();  // scores come from the scan kernel
  const int64_t pair = blockIdx.x;
  const int b = (int)(pair / p.Hkv);
  const int k = p.k;
  int32_t* sel = p.sel_idx + pair * k;
  const int L = __ldg(p.seq_lens + b);
  if (L < 1 || L > p.Lcap) {
    for (int i = tid; i < k; i += kSelThreads) sel[i] = -1;
    if (tid == 0) {
      p.sel_cnt[pair] = 0;
      set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    }
    return;
  }
  const int nb = (L + p.bs - 1) / p.bs;
  if (nb <= k) {  // the budget covers every block: dense
    for (int i = tid; i < k; i += kSelThreads) sel[i] = i < nb ? i : -1;
    if (tid == 0) p.sel_cnt[pair] = nb;
    return;
  }
  // load the scores as keys, building the first pass's histogram on the way
  const float* sc = p.scores + pair * p.nbcap;
  sm.hist[0][tid] = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += 4 * kSelThreads) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kSelThreads + tid;
      v[u] = i < nb ? __ldcg(sc + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kSelThreads + tid;
      if (i < nb) {
        const uint32_t key = float_key(v[u]);
        skey[i] = key;
        if (i >= 1 && i <= nb - 2) atomicAdd(&sm.hist[0][key >> 24], 1);
      }
    }
  }
  __syncthreads();
  topk_emit(skey, nb, k, sel, sm, p.dev_status);
  if (tid == 0) p.sel_cnt[pair] = k;
}

cudaError_t launch_select(const SelectParams& p, int /*chunks_per_pair*/, cudaStream_t s) {
  const size_t smem = (size_t)p.nbcap * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(select_topk_kernel), 0, smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)p.B * p.Hkv * p.nbcap;
  const int64_t want = (rows + kSelWarps * kSelU * 4 - 1) / (kSelWarps * kSelU * 4);  // >= 4 steps per warp
  const int64_t resident = (int64_t)device_sm_count() * KIN_SEL_CTAS_PER_SM;
  const int grid = (int)(want < resident ? (want > 0 ? want : 1) : resident);
  cudaError_t e = launch_pdl(select_scan_kernel, dim3(grid), dim3(kSelThreads), 0, s, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_topk_kernel, dim3(p.B * p.Hkv), dim3(kSelThreads), smem, s, p);
}

}  // namespace kin
