// kin_token.cu -- token-level top-k attention: the variant the Kinetics
// authors compare Block-TopK attention with ("Kinetics: Rethinking Test-Time
// Scaling Law", response Q2: Fig. 8 uses TopK attention, Figs. 10/21/22
// Block-TopK).  Each query head keeps the k tokens with the largest
// attention logits (MagicPIG's abstract on the same page list: TopK
// attention selects the keys and values with the highest attention scores)
// and attends over those only.
//
// Three kernels, chained with programmatic dependent launch:
//  1. token_logits_kernel: every logit z_t = scale * q_j . K_t of every query
//     head, a dense pass over K (the cost the block method avoids): per warp
//     a 2-stage ring of 16-token K tiles filled by all-lane 16-byte cp.async
//     into a 128-byte XOR-swizzled layout, S^T = K Q^T with 8 mma.sync
//     m16n8k16 per tile (tokens = M, the GQA group = N), fp32 logits to
//     workspace.
//  2. token_topk_kernel (kin_select.cu): the exact top-k per query head.
//  3. token_attn_kernel: one 4-warp CTA per query head stages the kept
//     indices and logits in shared memory (segments of 2048, running
//     maximum), gathers the kept V rows (one coalesced 256-byte warp load
//     per row, 16 rows in flight per lane) and sums them weighted by
//     exp(z_t - max z) in fp32.
#include "kin_internal.cuh"

namespace kin {

namespace {

constexpr int kTokWarps = 4;
constexpr int kTokThreads = kTokWarps * 32;
constexpr int kTokStages = 2;
constexpr int kTokChunkTiles = 32;                // 16-token tiles per logits CTA (512 tokens)
constexpr int kTokHalfBox = 16 * 64 * 2;          // 16 rows x 64 columns of bf16
constexpr int kTokStageBytes = 2 * kTokHalfBox;   // one K tile
constexpr int kTokSmem = kTokWarps * kTokStages * kTokStageBytes + 1024;
#define kTokNegInf (-__int_as_float(0x7f800000))

// grid: B * Hkv * ceil(Lcap / 512) items, item = (pair, 512-token chunk)
__global__ void __launch_bounds__(kTokThreads) token_logits_kernel(TokenParams p) {
  extern __shared__ uint8_t tok_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tok_smem_raw) + 1023) & ~uintptr_t(1023));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  // No early launch_dependents in the token kernels: the next grid launches
  // as this one's CTAs exit.  With all three triggering early a 32K decode
  // batch took 668.8 us per call against 593.4 us without (each alone cost
  // 0 to 8 us; the three together the rest).
  const int chunks = (p.Lcap + kTokChunkTiles * kTileTokens - 1) / (kTokChunkTiles * kTileTokens);
  const int64_t pair = blockIdx.x / chunks;
  const int c = (int)(blockIdx.x - pair * chunks);
  const int b = (int)(pair / p.Hkv), h = (int)(pair - (int64_t)b * p.Hkv);
  const int L = __ldg(p.seq_lens + b);
  if (L < 1 || L > p.Lcap) return;  // flagged by the top-k kernel
  const int t0 = c * kTokChunkTiles * kTileTokens;
  if (t0 >= L) return;
  const int ntiles = min(kTokChunkTiles, (L - t0 + kTileTokens - 1) / kTileTokens);
  const int n_w = warp < ntiles ? (ntiles - 1 - warp) / kTokWarps + 1 : 0;
  const int g = p.g;

  // Q fragments (B operand, "col" layout): head = lane/4, dims 16kk + 2(lane%4) (+8)
  uint32_t qf[8][2];
  {
    const int n = lane >> 2;
    const uint32_t* qrow =
        reinterpret_cast<const uint32_t*>(p.q + ((int64_t)b * p.Hq + (int64_t)h * g + (n < g ? n : 0)) * kHeadDim);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qf[kk][0] = n < g ? __ldg(qrow + kk * 8 + (lane & 3)) : 0u;
      qf[kk][1] = n < g ? __ldg(qrow + kk * 8 + 4 + (lane & 3)) : 0u;
    }
  }
  const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * kTokStages * kTokStageBytes);
  const __nv_bfloat16* kbase = p.k_cache + pair * (int64_t)p.Lcap * kHeadDim;

  // tile n of this warp covers tokens t0 + 16 (warp + 4 n) ..; lane l copies
  // pieces l + 32 i (i < 8), piece = (row r, 16-byte column cc)
  auto issue = [&](int n) {
    if (n < n_w) {
      const int row0 = t0 + (warp + kTokWarps * n) * kTileTokens;
      const int nv = min(kTileTokens, L - row0);
      const uint32_t base = ring + (uint32_t)((n % kTokStages) * kTokStageBytes);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int piece = lane + 32 * i;
        const int r = piece >> 4, cc = piece & 15;
        const uint32_t off = (uint32_t)((cc >> 3) * kTokHalfBox + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
        cp_async16(base + off, kbase + (int64_t)(row0 + (r < nv ? r : 0)) * kHeadDim + cc * 8, r < nv ? 16u : 0u);
      }
    }
    cp_async_commit();  // one group per tile, empty or not
  };
#pragma unroll
  for (int n = 0; n < kTokStages; ++n) issue(n);

  const int tq = lane >> 2, ta = 2 * (lane & 3);
  const int kr = lane & 15, khi = lane >> 4;
  float* zrow = p.logits + ((int64_t)b * p.Hq + (int64_t)h * g) * p.Lcap;
  for (int n = 0; n < n_w; ++n) {
    cp_async_wait<kTokStages - 1>();
    __syncwarp();
    const uint32_t base = ring + (uint32_t)((n % kTokStages) * kTokStageBytes);
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t box = base + (kk < 4 ? 0u : (uint32_t)kTokHalfBox);
      const int ch = (kk & 3) * 2 + khi;
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(box + kr * 128 + ((ch ^ (kr & 7)) << 4), a0, a1, a2, a3);
      if (kk & 1)
        mma_bf16_16816(sb, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      else
        mma_bf16_16816(sa, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
    }
    const int row0 = t0 + (warp + kTokWarps * n) * kTileTokens;
    const int tok0 = row0 + tq, tok1 = row0 + tq + 8;
    if (ta < g) {
      if (tok0 < L) zrow[(int64_t)ta * p.Lcap + tok0] = (sa[0] + sb[0]) * p.scale;
      if (tok1 < L) zrow[(int64_t)ta * p.Lcap + tok1] = (sa[2] + sb[2]) * p.scale;
    }
    if (ta + 1 < g) {
      if (tok0 < L) zrow[(int64_t)(ta + 1) * p.Lcap + tok0] = (sa[1] + sb[1]) * p.scale;
      if (tok1 < L) zrow[(int64_t)(ta + 1) * p.Lcap + tok1] = (sa[3] + sb[3]) * p.scale;
    }
    __syncwarp();  // every lane is done reading slot n % S before it is refilled
    issue(n + kTokStages);
  }
  cp_async_wait<0>();
}

constexpr int kTokAttnWarps = 4;
constexpr int kTokAttnThreads = kTokAttnWarps * 32;
constexpr int kTokSeg = 2048;                               // kept tokens staged per segment
constexpr int kTokSegPerThread = kTokSeg / kTokAttnThreads;  // 16
constexpr int kTokVRows = 16;                               // V rows in flight per lane

// one CTA per (sequence, query head): out = sum_t e^(z_t - M) V_t / sum_t e^(z_t - M)
// over the kept tokens, lse = M + ln sum_t e^(z_t - M).  The kept tokens are
// taken in segments of kTokSeg: each thread fetches its 16 indices, then
// their 16 logits, all in flight together, into shared memory; the running
// maximum M is raised to the segment's and the partial sums rescaled; then
// warp w streams its quarter of the segment's V rows, 16 rows in flight per
// lane (lane l owns dims 4l .. 4l + 3).
__global__ void __launch_bounds__(kTokAttnThreads, 7) token_attn_kernel(TokenParams p) {
  __shared__ int s_t[kTokSeg];
  __shared__ float s_z[kTokSeg];
  __shared__ __align__(16) float s_acc[kTokAttnWarps][kHeadDim];
  __shared__ float s_red[kTokAttnWarps];
  __shared__ float s_l[kTokAttnWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();  // the kept tokens come from the top-k kernel (no early trigger: see the logits kernel)
  const int64_t row_id = blockIdx.x;
  const int b = (int)(row_id / p.Hq), j = (int)(row_id - (int64_t)b * p.Hq), h = j / p.g;
  const int cnt = min(__ldg(p.cnt + row_id), p.kt);
  __nv_bfloat16* out = p.out + row_id * kHeadDim;
  if (cnt <= 0) {
    if (tid < kHeadDim) out[tid] = __float2bfloat16_rn(0.f);
    if (tid == 0 && p.lse) p.lse[row_id] = kTokNegInf;
    return;
  }
  const int32_t* sel = p.sel + row_id * p.kt;
  const float* z = p.logits + row_id * p.Lcap;
  const uint2* vbase = reinterpret_cast<const uint2*>(p.v_cache + ((int64_t)b * p.Hkv + h) * p.Lcap * kHeadDim) + lane;
  constexpr float kLog2e = 1.4426950408889634f;
  float M = kTokNegInf;  // running maximum over the segments so far (CTA-uniform)
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, lsum = 0.f;
  for (int s0 = 0; s0 < cnt; s0 += kTokSeg) {
    const int ns = min(kTokSeg, cnt - s0);
    // stage the segment's indices and logits; its maximum
    int tv[kTokSegPerThread];
#pragma unroll
    for (int r = 0; r < kTokSegPerThread; ++r) {
      const int i = r * kTokAttnThreads + tid;
      tv[r] = i < ns ? __ldg(sel + s0 + i) : 0;
    }
    float mx = kTokNegInf;
#pragma unroll
    for (int r = 0; r < kTokSegPerThread; ++r) {
      const int i = r * kTokAttnThreads + tid;
      if (i < ns) {
        const float zi = z[tv[r]];
        s_t[i] = tv[r];
        s_z[i] = zi;
        mx = fmaxf(mx, zi);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    float Mn = M;
#pragma unroll
    for (int w = 0; w < kTokAttnWarps; ++w) Mn = fmaxf(Mn, s_red[w]);
    if (Mn > M) {  // rescale what the earlier segments summed
      const float sc = M == kTokNegInf ? 0.f : exp2f((M - Mn) * kLog2e);
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] *= sc;
      lsum *= sc;
      M = Mn;
    }
    const float ml2 = M * kLog2e;
    // warp w: segment rows [r0, r1), in batches of 32 (lane l: row r0 + 32 q + l's index and weight)
    const int per = (ns + kTokAttnWarps - 1) / kTokAttnWarps;
    const int r0 = min(warp * per, ns), r1 = min(r0 + per, ns);
    for (int base = r0; base < r1; base += 32) {
      const int i = base + lane;
      const int t = i < r1 ? s_t[i] : 0;
      const float e = i < r1 ? exp2f(s_z[i] * kLog2e - ml2) : 0.f;
      lsum += e;
      const int nb = min(32, r1 - base);
      for (int u0 = 0; u0 < nb; u0 += kTokVRows) {
        uint2 v[kTokVRows];
#pragma unroll
        for (int u = 0; u < kTokVRows; ++u) {
          const int tt = __shfl_sync(0xffffffffu, t, (u0 + u) & 31);
          v[u] = u0 + u < nb ? __ldg(vbase + (int64_t)tt * (kHeadDim / 4)) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kTokVRows; ++u) {
          const float wu = __shfl_sync(0xffffffffu, e, (u0 + u) & 31);  // 0 past the batch's end
          const float2 lo = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v[u].x));
          const float2 hi = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v[u].y));
          acc[0] = fmaf(wu, lo.x, acc[0]);
          acc[1] = fmaf(wu, lo.y, acc[1]);
          acc[2] = fmaf(wu, hi.x, acc[2]);
          acc[3] = fmaf(wu, hi.y, acc[3]);
        }
      }
    }
    __syncthreads();  // the next segment overwrites s_t, s_z and s_red
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  reinterpret_cast<float4*>(s_acc[warp])[lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  if (lane == 0) s_l[warp] = lsum;
  __syncthreads();
  if (tid < kHeadDim) {
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kTokAttnWarps; ++w) {
      num += s_acc[w][tid];
      den += s_l[w];
    }
    out[tid] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
    if (tid == 0 && p.lse) p.lse[row_id] = den > 0.f ? M + logf(den) : kTokNegInf;
  }
}

}  // namespace

cudaError_t launch_token_logits(const TokenParams& p, cudaStream_t s) {
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(token_logits_kernel), 6, kTokSmem);
  if (e != cudaSuccess) return e;
  const int chunks = (p.Lcap + kTokChunkTiles * kTileTokens - 1) / (kTokChunkTiles * kTileTokens);
  return launch_pdl(token_logits_kernel, dim3(p.B * p.Hkv * chunks), dim3(kTokThreads), (size_t)kTokSmem, s, p);
}

cudaError_t launch_token_attn(const TokenParams& p, cudaStream_t s) {
  return launch_pdl(token_attn_kernel, dim3(p.B * p.Hq), dim3(kTokAttnThreads), 0, s, p);
}

}  // namespace kin
