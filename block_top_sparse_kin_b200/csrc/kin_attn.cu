// kin_attn.cu -- split-K flash-decode over the selected KV blocks with an
// in-kernel log-sum-exp merge.
//
// Math: softmax(q K^T / sqrt(d)) V restricted to the tokens of the kept
// blocks ("Kinetics: Memory-Aware Test-Time Scaling", Implementation,
// BlockTopKAttention), evaluated in the online (running max / running sum)
// form so that chunks of the kept blocks can be processed independently and
// merged: o = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c, M = max_c m_c
// (base-2 logits: the scale is folded with log2(e)).
//
// Work split (HBM-bound gather, ~8 KB of K+V per 16 tokens):
//   grid (chunk, kv head, batch); 4 warps per CTA.  A chunk is
//   `chunk_blocks` consecutive entries of the pair's ascending kept-block
//   list; its 16-token tiles are dealt round-robin to the 4 warps.
//   Each warp runs its own STAGES-deep pipeline: lane 0 issues four 2-D TMA
//   loads per tile (K and V, two 64-column halves each, 128-byte swizzle) that
//   complete on the slot's mbarrier; all lanes wait on it (bounded).
//   Per tile and warp: S^T[16 tok x 8 heads] = K Q^T with 8 mma.sync m16n8k16
//   (tokens are M, the GQA group is N, so g <= 8 wastes no rows), online
//   softmax across the 16 tokens with quad shuffles, P^T moved into the B
//   operand with movmatrix, then O^T[128 x 8] += V^T P^T with 8 more MMAs.
//   The 4 warps merge in shared memory; a chunk's partial (o, m, l) goes to
//   workspace and the pair's last chunk to finish (atomic counter, no spin)
//   merges all chunks and writes bf16 out and fp32 lse.
#include "kin_internal.cuh"

namespace kin {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kHalfBox = 16 * 64 * 2;        // bytes of one 16-row x 64-col bf16 box
constexpr int kStageBytes = 4 * kHalfBox;    // K0 K1 V0 V1
#define kNegInf (-__int_as_float(0x7f800000))

template <int STAGES>
constexpr size_t attn_smem_bytes() {
  return (size_t)kAttnWarps * STAGES * kStageBytes + 1024;  // + alignment slack
}

struct TileInfo {
  int64_t grow;  // row in the [B*Hkv*Lcap, D] view
  int nvalid;    // valid tokens in the tile, 0 => skip
  bool bad;      // block index out of range
};

__device__ __forceinline__ TileInfo tile_info(const AttnParams& p, int64_t pair, int warp, int n,
                                              int j0, int tpb, int nb, int L) {
  TileInfo t;
  const int T = warp + kAttnWarps * n;
  const int jj = j0 + T / tpb, sub = T % tpb;
  const int blk = __ldg(p.sel_idx + pair * p.k + jj);
  t.bad = blk < 0 || blk >= nb;
  const int row0 = blk * p.bs + sub * kTileTokens;
  t.nvalid = (t.bad || row0 >= L) ? 0 : min(kTileTokens, L - row0);
  t.grow = pair * p.Lcap + (t.nvalid ? row0 : 0);
  return t;
}

// Zero the bf16 halves of a V^T fragment register whose token is invalid.
__device__ __forceinline__ uint32_t tok_mask(int t, int nvalid) {
  return (t < nvalid ? 0x0000FFFFu : 0u) | (t + 1 < nvalid ? 0xFFFF0000u : 0u);
}

template <int STAGES>
__global__ void __launch_bounds__(kAttnThreads)
    attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kAttnWarps][STAGES];
  __shared__ float s_m[kAttnWarps][kMaxGroup], s_l[kAttnWarps][kMaxGroup];
  __shared__ int s_last;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b = blockIdx.z, h = blockIdx.y, c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = (int64_t)b * p.Hkv + h;
  const int g = p.g;
  const int L = p.seq_lens[b];
  int cnt = p.sel_cnt[pair];
  if (L < 1 || L > p.Lcap) cnt = 0;
  if (cnt > p.k) cnt = p.k;
  if (cnt <= 0) {  // nothing selected (flagged upstream): out = 0, lse = -inf
    if (c == 0) {
      for (int j = 0; j < g; ++j)
        p.out[((int64_t)b * p.Hq + (int64_t)h * g + j) * kHeadDim + tid] = __float2bfloat16_rn(0.f);
      if (p.lse && tid < g) p.lse[(int64_t)b * p.Hq + (int64_t)h * g + tid] = kNegInf;
    }
    return;
  }
  const int nchunks = (cnt + p.chunk_blocks - 1) / p.chunk_blocks;
  if (c >= nchunks) return;
  const int nb = (L + p.bs - 1) / p.bs;
  const int tpb = p.bs / kTileTokens;
  const int j0 = c * p.chunk_blocks;
  const int j1 = min(j0 + p.chunk_blocks, cnt);
  const int total_tiles = (j1 - j0) * tpb;
  const int n_w = warp < total_tiles ? (total_tiles - 1 - warp) / kAttnWarps + 1 : 0;

  // Q fragments (B operand, "col" layout): head = lane/4, dims 16kk + 2(lane%4) (+8).
  uint32_t qf[8][2];
  {
    const int n = lane >> 2;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        p.q + ((int64_t)b * p.Hq + (int64_t)h * g + (n < g ? n : 0)) * kHeadDim);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qf[kk][0] = n < g ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
      qf[kk][1] = n < g ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
    }
  }

  const uint32_t stage0 = smem_u32(smem) + (uint32_t)(warp * STAGES * kStageBytes);
  const uint32_t bar0 = smem_u32(&bars[warp][0]);
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncwarp();

  auto issue = [&](int n) {  // lane 0 only
    const int slot = n % STAGES;
    const uint32_t bar = bar0 + 8 * slot;
    const TileInfo t = tile_info(p, pair, warp, n, j0, tpb, nb, L);
    if (t.nvalid == 0) {
      mbar_arrive(bar);
      return;
    }
    const uint32_t dst = stage0 + (uint32_t)(slot * kStageBytes);
    mbar_arrive_expect_tx(bar, kStageBytes);
    const int32_t y = (int32_t)t.grow;
    tma_load_2d(dst, &tmk, 0, y, bar);
    tma_load_2d(dst + kHalfBox, &tmk, 64, y, bar);
    tma_load_2d(dst + 2 * kHalfBox, &tmv, 0, y, bar);
    tma_load_2d(dst + 3 * kHalfBox, &tmv, 64, y, bar);
  };

  if (lane == 0)
    for (int n = 0; n < n_w && n < STAGES; ++n) issue(n);

  float o[8][4];
#pragma unroll
  for (int dm = 0; dm < 8; ++dm) o[dm][0] = o[dm][1] = o[dm][2] = o[dm][3] = 0.f;
  float m0 = kNegInf, m1 = kNegInf, l0 = 0.f, l1 = 0.f;
  const float sl2 = p.scale_log2;
  const int tq = lane >> 2;                        // token row of C fragments
  const int ta = 2 * (lane & 3);                   // token col of A(V^T) fragments
  const int kr = lane & 15, khi = lane >> 4;       // ldmatrix row/col-chunk for K
  const int vt = (lane & 7) + ((lane >> 4) << 3);  // ldmatrix row for V^T
  const int vsel = (lane >> 3) & 1;

  int n_done = 0;
  bool timed_out = false;
  for (int n = 0; n < n_w; ++n) {
    const int slot = n % STAGES;
    const TileInfo t = tile_info(p, pair, warp, n, j0, tpb, nb, L);
    if (t.bad && lane == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    if (!mbar_wait_bounded(bar0 + 8 * slot, (uint32_t)((n / STAGES) & 1), p.dev_status)) {
      timed_out = true;
      break;
    }
    n_done = n + 1;
    if (t.nvalid > 0) {
      const uint32_t base = stage0 + (uint32_t)(slot * kStageBytes);
      // ---- S^T = K Q^T (two accumulator chains to halve the MMA dependency chain)
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t box = base + (kk < 4 ? 0u : (uint32_t)kHalfBox);
        const int ch = (kk & 3) * 2 + khi;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(box + kr * 128 + ((ch ^ (kr & 7)) << 4), a0, a1, a2, a3);
        if (kk & 1)
          mma_bf16_16816(sb, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
        else
          mma_bf16_16816(sa, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      }
      const bool v0 = tq < t.nvalid, v1 = tq + 8 < t.nvalid;
      const float s0 = v0 ? (sa[0] + sb[0]) * sl2 : kNegInf;
      const float s1 = v0 ? (sa[1] + sb[1]) * sl2 : kNegInf;
      const float s2 = v1 ? (sa[2] + sb[2]) * sl2 : kNegInf;
      const float s3 = v1 ? (sa[3] + sb[3]) * sl2 : kNegInf;
      // ---- online softmax over the tile's 16 tokens (per head column)
      float x0 = fmaxf(s0, s2), x1 = fmaxf(s1, s3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
      }
      const float mn0 = fmaxf(m0, x0), mn1 = fmaxf(m1, x1);
      const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
      const float p0 = exp2f(s0 - mn0), p1 = exp2f(s1 - mn1);
      const float p2 = exp2f(s2 - mn0), p3 = exp2f(s3 - mn1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        o[dm][0] *= al0;
        o[dm][1] *= al1;
        o[dm][2] *= al0;
        o[dm][3] *= al1;
      }
      // ---- P^T into the B operand (k = token, n = head) by 8x8 transposes
      const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
      const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
      const uint32_t mlo = tok_mask(ta, t.nvalid), mhi = tok_mask(ta + 8, t.nvalid);
      // ---- O^T += V^T P^T
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        const int d0 = dm * 16 + vsel * 8;
        const uint32_t box = base + 2u * kHalfBox + (d0 < 64 ? 0u : (uint32_t)kHalfBox);
        const int ch = (d0 & 63) >> 3;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(box + vt * 128 + ((ch ^ (vt & 7)) << 4), a0, a1, a2, a3);
        if (t.nvalid < kTileTokens) {  // invalid rows may hold anything: zero them
          a0 &= mlo;
          a1 &= mlo;
          a2 &= mhi;
          a3 &= mhi;
        }
        mma_bf16_16816(o[dm], a0, a1, a2, a3, pb0, pb1);
      }
    }
    fence_proxy_async_smem();  // our generic reads of the slot precede the next async write
    __syncwarp();
    if (lane == 0 && n + STAGES < n_w) issue(n + STAGES);
  }
  if (timed_out) {
    if (lane == 0) set_status(p.dev_status, KIN_ERR_TIMEOUT);
    // drain the copies this warp still has in flight before its smem is reused
    for (int n = n_done; n < n_w && n < n_done + STAGES; ++n)
      mbar_wait_bounded(bar0 + 8 * (n % STAGES), (uint32_t)((n / STAGES) & 1), nullptr);
    m0 = m1 = kNegInf;
    l0 = l1 = 0.f;
  }

  // ---- per-warp totals of l over the 8 token rows
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  __syncthreads();  // every warp is done with its pipeline smem
  float* so = reinterpret_cast<float*>(smem);  // [warp][head 8][128]
#pragma unroll
  for (int dm = 0; dm < 8; ++dm) {
    const int d = dm * 16 + tq;
    float* w0 = so + ((warp * kMaxGroup) + ta) * kHeadDim;
    w0[d] = o[dm][0];
    w0[kHeadDim + d] = o[dm][1];
    w0[d + 8] = o[dm][2];
    w0[kHeadDim + d + 8] = o[dm][3];
  }
  if (lane < 4) {
    s_m[warp][2 * lane] = m0;
    s_m[warp][2 * lane + 1] = m1;
    s_l[warp][2 * lane] = l0;
    s_l[warp][2 * lane + 1] = l1;
  }
  __syncthreads();

  const int d = tid;  // one output dim per thread
  const int64_t qh0 = (int64_t)b * p.Hq + (int64_t)h * g;
  if (nchunks == 1) {
    for (int j = 0; j < g; ++j) {
      float M = kNegInf;
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][j]);
      float num = 0.f, den = 0.f;
      if (M != kNegInf) {
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
          const float e = exp2f(s_m[w][j] - M);
          num += e * so[(w * kMaxGroup + j) * kHeadDim + d];
          den += e * s_l[w][j];
        }
      }
      p.out[(qh0 + j) * kHeadDim + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
      if (p.lse && d == 0) p.lse[qh0 + j] = den > 0.f ? (M + log2f(den)) * 0.6931471805599453f : kNegInf;
    }
    return;
  }

  // ---- write this chunk's partial, then the last chunk merges all of them
  float* part = p.partials + (pair * p.max_chunks + c) * (int64_t)g * (kHeadDim + 2);
  for (int j = 0; j < g; ++j) {
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][j]);
    float num = 0.f, den = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float e = exp2f(s_m[w][j] - M);
        num += e * so[(w * kMaxGroup + j) * kHeadDim + d];
        den += e * s_l[w][j];
      }
    }
    part[j * (kHeadDim + 2) + d] = num;
    if (d == 0) {
      part[j * (kHeadDim + 2) + kHeadDim] = M;
      part[j * (kHeadDim + 2) + kHeadDim + 1] = den;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[pair], 1u) == (unsigned)(nchunks - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) p.counters[pair] = 0u;
  const float* pp = p.partials + pair * p.max_chunks * (int64_t)g * (kHeadDim + 2);
  for (int j = 0; j < g; ++j) {
    float M = kNegInf;
    for (int cc = 0; cc < nchunks; ++cc)
      M = fmaxf(M, __ldcg(pp + ((int64_t)cc * g + j) * (kHeadDim + 2) + kHeadDim));
    float num = 0.f, den = 0.f;
    if (M != kNegInf) {
      for (int cc = 0; cc < nchunks; ++cc) {
        const float* q = pp + ((int64_t)cc * g + j) * (kHeadDim + 2);
        const float mc = __ldcg(q + kHeadDim);
        if (mc == kNegInf) continue;
        const float e = exp2f(mc - M);
        num += e * __ldcg(q + d);
        den += e * __ldcg(q + kHeadDim + 1);
      }
    }
    p.out[(qh0 + j) * kHeadDim + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
    if (p.lse && d == 0) p.lse[qh0 + j] = den > 0.f ? (M + log2f(den)) * 0.6931471805599453f : kNegInf;
  }
}

constexpr int kAttnStages = 4;

cudaError_t launch_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                        int grid_x, cudaStream_t s) {
  const size_t smem = attn_smem_bytes<kAttnStages>();
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<kAttnStages>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(grid_x, p.Hkv, p.B);
  attn_kernel<kAttnStages><<<grid, kAttnThreads, smem, s>>>(tmk, tmv, p);
  return cudaGetLastError();
}

}  // namespace kin
