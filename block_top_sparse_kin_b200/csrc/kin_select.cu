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
// Work split: CTA (c, h, b) scans `chunk_blocks` blocks of pair (b, h); one
// warp per 512-byte mean row (lane l reads dims 4l..4l+3 as one float4).
// Scores go to workspace (they stay in L2).  The last CTA of a pair to finish
// (atomic completion counter, no waiting) runs the top-k: a 4-pass 8-bit
// radix select over order-preserving uint32 keys in shared memory finds the
// threshold key T and how many keys equal to T to take; the lowest-index
// equal keys are taken, which is the (score desc, index asc) rule.  Output
// positions come from two block-wide prefix sums, so indices leave ascending.
#include "kin_internal.cuh"

namespace kin {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectParams p) {
  extern __shared__ uint32_t skey[];  // [nbcap], used by the finishing CTA only
  __shared__ int hist[256];
  __shared__ int warp_tot[kSelWarps];
  __shared__ int s_digit, s_above, s_last;

  const int b = blockIdx.z, h = blockIdx.y, c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = (int64_t)b * p.Hkv + h;
  const int k = p.k;
  int32_t* sel = p.sel_idx + pair * k;
  const int L = p.seq_lens[b];

  if (L < 1 || L > p.Lcap) {
    if (c == 0) {
      for (int i = tid; i < k; i += kSelThreads) sel[i] = -1;
      if (tid == 0) {
        p.sel_cnt[pair] = 0;
        set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
      }
    }
    return;
  }
  const int nb = (L + p.bs - 1) / p.bs;
  if (nb <= k) {  // the budget covers every block: dense
    if (c == 0) {
      for (int i = tid; i < k; i += kSelThreads) sel[i] = i < nb ? i : -1;
      if (tid == 0) p.sel_cnt[pair] = nb;
    }
    return;
  }
  const int nchunks = (nb + p.chunk_blocks - 1) / p.chunk_blocks;
  if (c >= nchunks) return;

  // ---- scan: s_i = scale * (sum_j q_j) . m_i for the blocks of this chunk
  float qs[4] = {0.f, 0.f, 0.f, 0.f};
  const __nv_bfloat16* qg = p.q + ((int64_t)b * p.Hq + (int64_t)h * p.g) * kHeadDim;
  for (int j = 0; j < p.g; ++j) {
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(qg + j * kHeadDim) + lane);
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.x));
    float2 bb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&raw.y));
    qs[0] += a.x;
    qs[1] += a.y;
    qs[2] += bb.x;
    qs[3] += bb.y;
  }
  const int i0 = c * p.chunk_blocks;
  const int i1 = min(i0 + p.chunk_blocks, nb);
  const float4* mrow = reinterpret_cast<const float4*>(p.means + pair * p.nbcap * kHeadDim) + lane;
  float* sc = p.scores + pair * p.nbcap;
#ifndef KIN_SEL_UNROLL
#define KIN_SEL_UNROLL 4
#endif
  constexpr int U = KIN_SEL_UNROLL;  // mean rows in flight per warp
  for (int i = i0 + warp; i < i1; i += kSelWarps * U) {
    float4 m[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ii = i + u * kSelWarps;
      m[u] = ii < i1 ? __ldcs(mrow + (int64_t)ii * (kHeadDim / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float d = qs[0] * m[u].x;
      d = fmaf(qs[1], m[u].y, d);
      d = fmaf(qs[2], m[u].z, d);
      d = fmaf(qs[3], m[u].w, d);
      d = warp_sum(d);
      const int ii = i + u * kSelWarps;
      if (lane == 0 && ii < i1) sc[ii] = d * p.score_scale;
    }
  }

  // ---- completion: the last CTA of this pair runs the top-k
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[pair], 1u) == (unsigned)(nchunks - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) p.counters[pair] = 0u;  // ready for the next call
  for (int i = tid; i < nb; i += kSelThreads) skey[i] = float_key(__ldcg(sc + i));
  __syncthreads();

  // ---- radix select over candidates 1..nb-2: threshold key T, ties to take kr
  uint32_t prefix = 0u, mask = 0u;
  int kr = k - 2;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[tid] = 0;
    __syncthreads();
    for (int i = 1 + tid; i < nb - 1; i += kSelThreads) {
      const uint32_t key = skey[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1);
    }
    __syncthreads();
    if (warp == 0) {
      int cnt[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cnt[u] = hist[255 - (lane * 8 + u)];  // descending digits
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
            s_digit = 255 - (lane * 8 + u);
            s_above = run;
            break;
          }
          run += cnt[u];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    mask |= 0xFFu << shift;
    kr -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // ---- emit: forced {0, nb-1}, keys > T, and the kr lowest-index keys == T
  const int per = (nb + kSelThreads - 1) / kSelThreads;
  const int j0 = min(tid * per, nb), j1 = min(j0 + per, nb);
  int eq = 0;
  for (int i = j0; i < j1; ++i)
    if (i >= 1 && i <= nb - 2 && skey[i] == T) ++eq;
  const int eq_base = block_exclusive_scan(eq, warp_tot);
  int r = eq_base, mine = 0;
  for (int i = j0; i < j1; ++i) {
    const bool cand = i >= 1 && i <= nb - 2;
    const uint32_t key = skey[i];
    bool take = !cand || key > T;
    if (cand && key == T) {
      take = r < kr;
      ++r;
    }
    mine += take;
  }
  int pos = block_exclusive_scan(mine, warp_tot);
  r = eq_base;
  for (int i = j0; i < j1; ++i) {
    const bool cand = i >= 1 && i <= nb - 2;
    const uint32_t key = skey[i];
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
  if (tid == kSelThreads - 1 && pos != k) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
  if (tid == 0) p.sel_cnt[pair] = k;
}

cudaError_t launch_select(const SelectParams& p, int grid_x, cudaStream_t s) {
  const size_t smem = (size_t)p.nbcap * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(grid_x, p.Hkv, p.B);
  select_kernel<<<grid, kSelThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kin
