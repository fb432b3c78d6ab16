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
// Work split: a work item is a chunk of `chunk_blocks` blocks of one pair;
// a grid of KIN_SEL_CTAS_PER_SM resident CTAs per SM walks the items.  Warp
// w scans rows w, w + 8, ... of the chunk, one 512-byte mean row per warp
// load (lane l reads dims 4l..4l+3 as one float4), double-buffered so the
// next U rows are in flight while the current U are reduced; a butterfly
// that halves the rows per lane at each level sums U rows in U + 4 - log2 U
// shuffles.  Scores go to workspace (they stay in L2).  The pair's last
// chunk to finish (atomic completion counter, no waiting) runs the top-k: a
// 4-pass 8-bit radix select over order-preserving uint32 keys in shared
// memory finds the threshold key T and how many keys equal to T to take; the
// lowest-index equal keys are taken, which is the (score desc, index asc)
// rule.  Output positions come from two block-wide prefix sums, so indices
// leave ascending.
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

// Exclusive prefix sum over the CTA (256 threads); returns this thread's base.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  int base = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) base += (w < warp) ? warp_tot[w] : 0;
  __syncthreads();
  return base + inc - v;
}

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

struct SelectSmem {
  int hist[256];
  int warp_tot[kSelWarps];
  int digit, above, last;
};

// Exact top-(k-2) over keys[1..nb-2] plus the forced blocks 0 and nb-1,
// written ascending to sel[0..k).  keys live in shared memory.
__device__ __forceinline__ void topk_emit(const uint32_t* keys, int nb, int k, int32_t* sel,
                                          SelectSmem& sm, int32_t* dev_status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- radix select: threshold key T and the number kr of keys == T to take
  uint32_t prefix = 0u, mask = 0u;
  int kr = k - 2;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    sm.hist[tid] = 0;
    __syncthreads();
    for (int i = 1 + tid; i < nb - 1; i += kSelThreads) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 0xFFu], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int cnt[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cnt[u] = sm.hist[255 - (lane * 8 + u)];  // descending digits
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
            break;
          }
          run += cnt[u];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)sm.digit << shift;
    mask |= 0xFFu << shift;
    kr -= sm.above;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // ---- emit: forced {0, nb-1}, keys > T, and the kr lowest-index keys == T
  const int per = (nb + kSelThreads - 1) / kSelThreads;
  const int j0 = min(tid * per, nb), j1 = min(j0 + per, nb);
  int eq = 0;
  for (int i = j0; i < j1; ++i)
    if (i >= 1 && i <= nb - 2 && keys[i] == T) ++eq;
  const int eq_base = block_exclusive_scan(eq, sm.warp_tot);
  int r = eq_base, mine = 0;
  for (int i = j0; i < j1; ++i) {
    const bool cand = i >= 1 && i <= nb - 2;
    const uint32_t key = keys[i];
    bool take = !cand || key > T;
    if (cand && key == T) {
      take = r < kr;
      ++r;
    }
    mine += take;
  }
  int pos = block_exclusive_scan(mine, sm.warp_tot);
  r = eq_base;
  for (int i = j0; i < j1; ++i) {
    const bool cand = i >= 1 && i <= nb - 2;
    const uint32_t key = keys[i];
    bool take = !cand || key > T;
    if (cand && key == T) {
      take = r < kr;
      ++r;
    }
    if (take) {
      if (pos < k) sel[pos] = i;  // never write past the pair's row
      ++pos;
    }
  }
  // self-check: exactly k blocks were emitted (the last thread ends at k)
  if (tid == kSelThreads - 1 && pos != k) set_status(dev_status, KIN_ERR_DEVICE_DATA);
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
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kSelWarps;
  const int gw = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  const int nbp = (p.nbcap + kSelU - 1) / kSelU * kSelU;
  const int steps = p.B * p.Hkv * (nbp / kSelU);
  const int per = (steps + nwarps - 1) / nwarps;
  const int s0 = gw * per, s1 = min(s0 + per, steps);
  if (s0 >= s1) return;

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
}

// ---- kernel 2: one CTA per pair: dense shortcut, bad-length flag, or the
// exact top-k over the scores the scan left in workspace (L2-resident).
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(SelectParams p) {
  extern __shared__ uint32_t skey[];  // [nbcap]
  __shared__ SelectSmem sm;
  const int tid = threadIdx.x;
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
  const float* sc = p.scores + pair * p.nbcap;
  for (int i = tid; i < nb; i += kSelThreads) skey[i] = float_key(__ldcg(sc + i));
  __syncthreads();
  topk_emit(skey, nb, k, sel, sm, p.dev_status);
  if (tid == 0) p.sel_cnt[pair] = k;
}

cudaError_t launch_select(const SelectParams& p, int /*chunks_per_pair*/, cudaStream_t s) {
  const size_t smem = (size_t)p.nbcap * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)p.B * p.Hkv * p.nbcap;
  const int64_t want = (rows + kSelWarps * kSelU * 4 - 1) / (kSelWarps * kSelU * 4);  // >= 4 steps per warp
  const int64_t resident = (int64_t)sms * KIN_SEL_CTAS_PER_SM;
  const int grid = (int)(want < resident ? (want > 0 ? want : 1) : resident);
  select_scan_kernel<<<grid, kSelThreads, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_topk_kernel<<<p.B * p.Hkv, kSelThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kin
