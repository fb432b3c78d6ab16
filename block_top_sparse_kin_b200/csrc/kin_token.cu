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
//  3. token_attn_kernel: one CTA per query head gathers the kept V rows
//     (one coalesced 256-byte warp load per row, 8 rows in flight per lane)
//     and sums them weighted by exp(z_t - max z) in fp32.
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
  pdl_trigger_early();
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

constexpr int kTokAttnWarps = 8;
constexpr int kTokAttnThreads = kTokAttnWarps * 32;

// one CTA per (sequence, query head): out = sum_t e^(z_t - M) V_t / sum_t e^(z_t - M)
// over the kept tokens, lse = M + ln sum_t e^(z_t - M)
__global__ void __launch_bounds__(kTokAttnThreads) token_attn_kernel(TokenParams p) {
  __shared__ __align__(16) float s_acc[kTokAttnWarps][kHeadDim];
  __shared__ float s_red[kTokAttnWarps];
  __shared__ float s_l[kTokAttnWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();  // the kept tokens come from the top-k kernel
  pdl_trigger_early();
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
  // pass 1: the largest kept logit
  float mx = kTokNegInf;
  for (int i = tid; i < cnt; i += kTokAttnThreads) mx = fmaxf(mx, z[__ldg(sel + i)]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  float M = s_red[0];
#pragma unroll
  for (int w = 1; w < kTokAttnWarps; ++w) M = fmaxf(M, s_red[w]);
  const float ml2 = M * 1.4426950408889634f;

  // pass 2: warp w takes kept tokens [w per, (w + 1) per) in batches of 32:
  // lane l fetches token l's index and weight, then the warp streams the
  // batch's V rows 8 at a time (lane l owns dims 4l .. 4l + 3)
  const uint2* vbase = reinterpret_cast<const uint2*>(p.v_cache + ((int64_t)b * p.Hkv + h) * p.Lcap * kHeadDim) + lane;
  const int per = (cnt + kTokAttnWarps - 1) / kTokAttnWarps;
  const int i0 = warp * per, i1 = min(i0 + per, cnt);
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, lsum = 0.f;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    const int t = i < i1 ? __ldg(sel + i) : 0;
    const float e = i < i1 ? exp2f(z[t] * 1.4426950408889634f - ml2) : 0.f;
    lsum += e;
    const int nb = min(32, i1 - base);
    for (int u0 = 0; u0 < nb; u0 += 8) {
      uint2 v[8];
      float w8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int src = (u0 + u) & 31;
        const int tt = __shfl_sync(0xffffffffu, t, src);
        w8[u] = __shfl_sync(0xffffffffu, e, src);
        v[u] = u0 + u < nb ? __ldg(vbase + (int64_t)tt * (kHeadDim / 4)) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u0 + u < nb) {
          const float2 lo = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v[u].x));
          const float2 hi = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v[u].y));
          acc[0] = fmaf(w8[u], lo.x, acc[0]);
          acc[1] = fmaf(w8[u], lo.y, acc[1]);
          acc[2] = fmaf(w8[u], hi.x, acc[2]);
          acc[3] = fmaf(w8[u], hi.y, acc[3]);
        }
      }
    }
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
