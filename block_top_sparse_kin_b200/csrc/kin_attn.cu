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
// Design (an HBM-bound gather of scattered 4 KB K and V tiles, ~1 flop/byte
// per query head):
//  * One CTA per work item = (kv pair, chunk of `chunk_blocks` consecutive
//    entries of the pair's ascending kept-block list); several CTAs share an
//    SM so one CTA's merge overlaps the others' streaming.
//  * Each warp streams its own 16-token tiles (tiles w, w + W, ...) through a
//    KIN_ATTN_STAGES-deep ring in shared memory with 16-byte cp.async copies
//    issued by all 32 lanes (16 per lane per tile), written straight into a
//    128-byte XOR-swizzled layout so ldmatrix reads are bank-conflict free.
//    Rows past the sequence end are zero-filled, never read.  (Measured on
//    B200: one thread issuing TMA/bulk copies of such small tiles tops out
//    near 2 copies/us, so spreading the issue over all lanes is what lets the
//    gather approach HBM speed.)
//  * Per tile: S^T[16 tok x 8 heads] = K Q^T with 8 mma.sync m16n8k16 (tokens
//    are M, the GQA group is N), online softmax over the 16 tokens with quad
//    shuffles, P^T moved into the B operand with movmatrix, O^T[128 x 8] +=
//    V^T P^T with 8 more MMAs.
//  * The warps merge in shared memory.  A single-chunk pair writes bf16 out
//    and fp32 lse directly; otherwise the chunk's partial (o, m, l) goes to
//    workspace and the pair's last chunk to finish (atomic counter, no
//    spinning) merges all of them, staged in shared memory with one round
//    of independent 16-byte loads.
#include "kin_internal.cuh"

namespace kin {

#ifndef KIN_ATTN_WARPS
#define KIN_ATTN_WARPS 4
#endif
#ifndef KIN_ATTN_STAGES
#define KIN_ATTN_STAGES 2
#endif
#ifndef KIN_ATTN_CTAS_PER_SM
#define KIN_ATTN_CTAS_PER_SM 3
#endif

constexpr int kAttnWarps = KIN_ATTN_WARPS;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kStages = KIN_ATTN_STAGES;
constexpr int kHalfBox = 16 * 64 * 2;       // bytes of a 16-row x 64-column bf16 half tile
constexpr int kStageBytes = 4 * kHalfBox;   // K0 K1 V0 V1
constexpr int kRowPad = kHeadDim + 4;       // combine rows padded against bank conflicts
constexpr size_t kPipeBytes = (size_t)kAttnWarps * kStages * kStageBytes;
constexpr size_t kCombBytes = (size_t)kAttnWarps * kMaxGroup * kRowPad * sizeof(float);
static_assert(kAttnThreads >= kHeadDim, "one thread per output dim in the merge");
// (chunk, head) records staged per merge batch: kPipeBytes / (4 kPartStride)
constexpr int kMaxMergeWeights = (int)(kPipeBytes / (sizeof(float) * kPartStride));
static_assert(kMaxItemTiles / kAttnWarps <= 32, "a warp's tiles of one item fit one per lane");
#define kNegInf (-__int_as_float(0x7f800000))

size_t attn_smem_bytes() { return (kPipeBytes > kCombBytes ? kPipeBytes : kCombBytes) + 1024; }

struct ItemInfo {
  int64_t pair;
  int b, h, c, L, nb, cnt, nchunks, j0, ntiles;
};

__device__ __forceinline__ ItemInfo item_info(const AttnParams& p, int u) {
  ItemInfo it;
  it.pair = u / p.max_chunks;
  it.c = u - (int)it.pair * p.max_chunks;
  it.b = (int)(it.pair / p.Hkv);
  it.h = (int)(it.pair - (int64_t)it.b * p.Hkv);
  it.L = __ldg(p.seq_lens + it.b);
  int cnt = __ldg(p.sel_cnt + it.pair);
  if (it.L < 1 || it.L > p.Lcap) cnt = 0;
  if (cnt > p.k) cnt = p.k;
  it.cnt = cnt;
  it.nchunks = cnt > 0 ? (cnt + p.chunk_blocks - 1) / p.chunk_blocks : 0;
  it.nb = (it.L + p.bs - 1) / p.bs;
  it.j0 = it.c * p.chunk_blocks;
  const int j1 = min(it.j0 + p.chunk_blocks, cnt);
  it.ntiles = it.c < it.nchunks ? (j1 - it.j0) * (p.bs / kTileTokens) : 0;
  return it;
}

// Zero the bf16 halves of a V^T fragment register whose token is invalid.
__device__ __forceinline__ uint32_t tok_mask(int t, int nvalid) {
  return (t < nvalid ? 0x0000FFFFu : 0u) | (t + 1 < nvalid ? 0xFFFF0000u : 0u);
}


__global__ void __launch_bounds__(kAttnThreads, KIN_ATTN_CTAS_PER_SM) attn_kernel(AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float s_m[kAttnWarps][kMaxGroup], s_l[kAttnWarps][kMaxGroup];
  __shared__ int s_last;
  // merge: per head running max, sum and rescale; per (chunk, head) weight
  __shared__ float s_mr[kMaxGroup], s_den[kMaxGroup], s_a[kMaxGroup], s_w[kMaxMergeWeights];
  // warp combine: per (warp, head) weight, per head maximum and sum
  __shared__ float s_ww[kAttnWarps][kMaxGroup], s_cm[kMaxGroup], s_cden[kMaxGroup];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = p.g;
  pdl_wait();  // the selection comes from the select kernels
  pdl_trigger_early();
  // Lane l's tile of this warp (tile warp + W l of the chunk): its block
  // index is requested before the pair's length and count, whose round trip
  // it would otherwise follow (a chunk holds at most chunk_blocks blocks,
  // all inside the pair's row of k; entries past the count are checked below).
  const int tpb = p.bs / kTileTokens;
  int blk_spec = -1;
  {
    const int64_t pair0 = blockIdx.x / p.max_chunks;
    const int c0 = (int)(blockIdx.x - pair0 * p.max_chunks);
    const int t = warp + kAttnWarps * lane;
    const int j = c0 * p.chunk_blocks + t / tpb;
    if (t < p.chunk_blocks * tpb && j < p.k) blk_spec = __ldg(p.sel_idx + pair0 * p.k + j);
  }
  const ItemInfo it = item_info(p, blockIdx.x);
  const int64_t qh0 = (int64_t)it.b * p.Hq + (int64_t)it.h * g;
  if (it.cnt <= 0) {  // nothing selected (flagged upstream): out = 0, lse = -inf
    if (it.c == 0 && tid < kHeadDim) {
      for (int j = 0; j < g; ++j) p.out[(qh0 + j) * kHeadDim + tid] = __float2bfloat16_rn(0.f);
      if (p.lse && tid < g) p.lse[qh0 + tid] = kNegInf;
    }
    return;
  }
  if (it.ntiles == 0) return;  // a chunk index past this pair's chunks

  // ---- this warp's tiles t = warp + W n; lane n holds tile n's source
  // offset (elements, into the contiguous cache or the page pool) and its
  // valid row count
  const int n_w = warp < it.ntiles ? (it.ntiles - 1 - warp) / kAttnWarps + 1 : 0;
  int64_t my_off = 0;
  int my_nvalid = 0;
  if (lane < n_w) {
    const int t = warp + kAttnWarps * lane;
    const int blk = blk_spec;
    const int sub = (t - (t / tpb) * tpb) * kTileTokens;
    bool bad = blk < 0 || blk >= it.nb;
    const int64_t off = bad ? -1 : kv_row_offset(p.pages, it.b, it.h, p.Hkv, p.Lcap, p.bs, blk, sub);
    bad = off < 0;
    if (bad) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    const int row0 = blk * p.bs + sub;  // logical token index of the tile's first row
    my_nvalid = (bad || row0 >= it.L) ? 0 : min(kTileTokens, it.L - row0);
    my_off = my_nvalid ? off : 0;
  }

  // Q fragments (B operand, "col" layout): head = lane/4, dims 16kk + 2(lane%4) (+8)
  uint32_t qf[8][2];
  {
    const int n = lane >> 2;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.q + (qh0 + (n < g ? n : 0)) * kHeadDim);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qf[kk][0] = n < g ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
      qf[kk][1] = n < g ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
    }
  }

  const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * kStages * kStageBytes);

  // Issue tile n into its ring slot: lane l copies pieces l + 32 i (i < 8) of
  // the K tile and of the V tile; piece = (row r, 16-byte column cc).
  auto issue = [&](int n) {
    const int64_t off0 = (int64_t)(((uint64_t)(uint32_t)__shfl_sync(0xffffffffu, (int)(my_off >> 32), n & 31) << 32) |
                                   (uint32_t)__shfl_sync(0xffffffffu, (int)(uint32_t)my_off, n & 31));
    const int nv = __shfl_sync(0xffffffffu, my_nvalid, n & 31);
    if (n < n_w && nv > 0) {
      const uint32_t base = ring + (uint32_t)((n % kStages) * kStageBytes);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int piece = lane + 32 * i;
        const int r = piece >> 4, cc = piece & 15;
        const uint32_t off = (uint32_t)((cc >> 3) * kHalfBox + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
        const int64_t src = off0 + (int64_t)(r < nv ? r : 0) * kHeadDim + cc * 8;
        const uint32_t bytes = r < nv ? 16u : 0u;
        cp_async16(base + off, p.k_cache + src, bytes);
        cp_async16(base + 2 * kHalfBox + off, p.v_cache + src, bytes);
      }
    }
    cp_async_commit();  // one group per tile, empty or not, keeps the accounting uniform
  };

#pragma unroll
  for (int n = 0; n < kStages; ++n) issue(n);

  float o[8][4];
#pragma unroll
  for (int dm = 0; dm < 8; ++dm) o[dm][0] = o[dm][1] = o[dm][2] = o[dm][3] = 0.f;
  float m0 = kNegInf, m1 = kNegInf, l0 = 0.f, l1 = 0.f;
  const float sl2 = p.scale_log2;
  const int tq = lane >> 2;                        // token row of C fragments
  const int ta = 2 * (lane & 3);                   // token col of A(V^T) / head col of C
  const int kr = lane & 15, khi = lane >> 4;       // ldmatrix row / column chunk for K
  const int vt = (lane & 7) + ((lane >> 4) << 3);  // ldmatrix row for V^T
  const int vsel = (lane >> 3) & 1;

  for (int n = 0; n < n_w; ++n) {
    cp_async_wait<kStages - 1>();  // this lane's copies of tile n have landed
    __syncwarp();                  // ... and every other lane's
    const int nvalid = __shfl_sync(0xffffffffu, my_nvalid, n & 31);
    if (nvalid > 0) {
      const uint32_t base = ring + (uint32_t)((n % kStages) * kStageBytes);
      // ---- S^T = K Q^T (two accumulator chains halve the MMA dependency chain)
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
      const bool v0 = tq < nvalid, v1 = tq + 8 < nvalid;
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
      const uint32_t mlo = tok_mask(ta, nvalid), mhi = tok_mask(ta + 8, nvalid);
      // ---- O^T += V^T P^T
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
        const int d0 = dm * 16 + vsel * 8;
        const uint32_t box = base + 2u * kHalfBox + (d0 < 64 ? 0u : (uint32_t)kHalfBox);
        const int ch = (d0 & 63) >> 3;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(box + vt * 128 + ((ch ^ (vt & 7)) << 4), a0, a1, a2, a3);
        if (nvalid < kTileTokens) {  // zero-filled rows: keep them out exactly
          a0 &= mlo;
          a1 &= mlo;
          a2 &= mhi;
          a3 &= mhi;
        }
        mma_bf16_16816(o[dm], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();  // every lane is done reading slot n % S before it is refilled
    issue(n + kStages);
  }
  cp_async_wait<0>();

  // ---- per-warp totals of l over the 8 token rows, then the cross-warp merge
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  __syncthreads();  // every warp is done with its ring; the combine area reuses it
  float* comb = reinterpret_cast<float*>(smem);  // [warp][head][kRowPad]
#pragma unroll
  for (int dm = 0; dm < 8; ++dm) {
    const int d = dm * 16 + tq;
    float* w0 = comb + ((warp * kMaxGroup) + ta) * kRowPad;
    w0[d] = o[dm][0];
    w0[kRowPad + d] = o[dm][1];
    w0[d + 8] = o[dm][2];
    w0[kRowPad + d + 8] = o[dm][3];
  }
  if (lane < 4) {
    s_m[warp][2 * lane] = m0;
    s_m[warp][2 * lane + 1] = m1;
    s_l[warp][2 * lane] = l0;
    s_l[warp][2 * lane + 1] = l1;
  }
  __syncthreads();

  // per head j (thread j < g): the maximum over the warps, each warp's
  // weight and the weighted sum; then every thread combines its output dim
  if (tid < g) {
    const int j = tid;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][j]);
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float e = M == kNegInf ? 0.f : exp2f(s_m[w][j] - M);
      s_ww[w][j] = e;
      den += e * s_l[w][j];
    }
    s_cm[j] = M;
    s_cden[j] = den;
  }
  __syncthreads();
  const int d = tid;  // one output dim per thread (threads >= kHeadDim idle)
  const int gd = d < kHeadDim ? g : 0;
  auto combined = [&](int j) {
    float num = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) num += s_ww[w][j] * comb[(w * kMaxGroup + j) * kRowPad + d];
    return num;
  };
  if (it.nchunks == 1) {
    for (int j = 0; j < gd; ++j) {
      const float num = combined(j), den = s_cden[j];
      p.out[(qh0 + j) * kHeadDim + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
      if (p.lse && d == 0) p.lse[qh0 + j] = den > 0.f ? (s_cm[j] + log2f(den)) * 0.6931471805599453f : kNegInf;
    }
    return;
  }

  // ---- write this chunk's partial; the pair's last chunk merges all of them
  float* part = p.partials + (it.pair * p.max_chunks + it.c) * (int64_t)g * kPartStride;
  for (int j = 0; j < gd; ++j) {
    part[j * kPartStride + d] = combined(j);
    if (d == 0) {
      part[j * kPartStride + kHeadDim] = s_cm[j];
      part[j * kPartStride + kHeadDim + 1] = s_cden[j];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.counters[it.pair], 1u) == (unsigned)(it.nchunks - 1));
  __syncthreads();
  if (!s_last) return;

  // Merge all chunks of the pair: their partial records are staged in shared
  // memory (the idle ring and combine area: every thread passed the two
  // barriers above after its last read of the combine rows) with one round
  // of 16-byte cp.async copies per batch of chunks that fits.  Threads j < g
  // then fold head j's maxima and sums and leave one weight per (chunk,
  // head) in shared memory, and every thread folds its output dim with
  // independent, unrolled reads, so a merge costs about one L2 round trip.
  __threadfence();
  if (tid == 0) p.counters[it.pair] = 0u;  // ready for the next call
  const int rec = g * kPartStride;                                  // floats per chunk
  const int per_batch = (int)(kPipeBytes / (sizeof(float) * rec));  // chunks staged at once
  const float4* src4 = reinterpret_cast<const float4*>(p.partials + it.pair * p.max_chunks * (int64_t)rec);
  const float* stage = reinterpret_cast<const float*>(smem);
  const uint32_t stage_s = smem_u32(smem);
  float num[kMaxGroup];
#pragma unroll
  for (int j = 0; j < kMaxGroup; ++j) num[j] = 0.f;
  if (tid < g) {
    s_mr[tid] = kNegInf;
    s_den[tid] = 0.f;
  }
  for (int cb = 0; cb < it.nchunks; cb += per_batch) {
    const int nbat = min(per_batch, it.nchunks - cb);
    const int n4 = nbat * rec / 4;
    const float4* s4 = src4 + (int64_t)cb * (rec / 4);
    for (int i = tid; i < n4; i += kAttnThreads) cp_async16(stage_s + 16u * (uint32_t)i, s4 + i, 16u);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    // the staged records are dead in memory: drop their L2 lines without a
    // write-back (only lines wholly inside this batch's records, so no other
    // pair's records are touched; the next call rewrites them before reading)
    {
      const uintptr_t lo = reinterpret_cast<uintptr_t>(s4), hi = lo + (uintptr_t)n4 * 16u;
      const uintptr_t first = (lo + 127u) & ~uintptr_t(127);
      const int nlines = hi > first ? (int)((hi - first) >> 7) : 0;
      for (int i = tid; i < nlines; i += kAttnThreads) discard_l2_line(reinterpret_cast<const void*>(first + 128u * i));
    }
    if (tid < g) {  // head j: batch maximum, rescale of the running sums, chunk weights
      const int j = tid;
      float Mb = kNegInf;
      for (int c = 0; c < nbat; ++c) Mb = fmaxf(Mb, stage[(c * g + j) * kPartStride + kHeadDim]);
      const float Mr = s_mr[j];
      const float Mn = fmaxf(Mr, Mb);
      const float a = Mn == kNegInf ? 0.f : exp2f(Mr - Mn);
      float dd = s_den[j] * a;
      for (int c = 0; c < nbat; ++c) {
        const float* r = stage + (c * g + j) * kPartStride;
        const float e = (Mn == kNegInf || r[kHeadDim] == kNegInf) ? 0.f : exp2f(r[kHeadDim] - Mn);
        s_w[c * g + j] = e;
        dd += e * r[kHeadDim + 1];
      }
      s_a[j] = a;
      s_mr[j] = Mn;
      s_den[j] = dd;
    }
    __syncthreads();
    if (d < kHeadDim) {  // chunk-outer, head-inner: g independent accumulation chains
#pragma unroll
      for (int j = 0; j < kMaxGroup; ++j)
        if (j < g) num[j] *= s_a[j];
      for (int c = 0; c < nbat; ++c) {
        const float* rc = stage + c * g * kPartStride + d;
#pragma unroll
        for (int j = 0; j < kMaxGroup; ++j)
          if (j < g) num[j] += s_w[c * g + j] * rc[j * kPartStride];
      }
    }
    __syncthreads();  // the next batch overwrites the staging area and the weights
  }
  if (d < kHeadDim) {
#pragma unroll
    for (int j = 0; j < kMaxGroup; ++j) {
      if (j < g) {
        const float den = s_den[j];
        p.out[(qh0 + j) * kHeadDim + d] = __float2bfloat16_rn(den > 0.f ? num[j] / den : 0.f);
        if (p.lse && d == 0)
          p.lse[qh0 + j] = den > 0.f ? (s_mr[j] + log2f(den)) * 0.6931471805599453f : kNegInf;
      }
    }
  }
}

cudaError_t launch_attn(const AttnParams& p, int num_items, cudaStream_t s) {
  const size_t smem = attn_smem_bytes();
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(attn_kernel), 1, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_kernel, dim3(num_items), dim3(kAttnThreads), smem, s, p);
}

}  // namespace kin
