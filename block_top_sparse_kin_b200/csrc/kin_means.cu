// kin_means.cu -- block mean keys: build for a prefilled cache, and the
// append-and-refresh update of a decode step.
//
// The block summary is the mean key over the block's valid tokens (the block
// mean of "Kinetics: Memory-Aware Test-Time Scaling", Implementation,
// BlockTopKAttention, read along the key axis).  Means are summed in fp32 in
// token order and divided by the valid-row count, so a refreshed block is
// bit-identical to one built from scratch.
//
// Layout: one warp per block; lane l owns dims 4l..4l+3, so every cache row is
// one coalesced 256-byte warp load and every mean one 512-byte warp store.
// K/V rows are addressed through kv_row_offset, so the same kernels serve
// the contiguous cache and the paged pool (a block's rows are contiguous in
// both).
#include "kin_internal.cuh"

namespace kin {

__device__ __forceinline__ void add_row4(float (&acc)[4], uint2 raw) {
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  acc[0] += a.x;
  acc[1] += a.y;
  acc[2] += b.x;
  acc[3] += b.y;
}

// grid (ceil(nbcap / 8), Hkv, B), 256 threads: warp w of CTA x owns block 8x + w.
__global__ void __launch_bounds__(256) means_build_kernel(MeansBuildParams p) {
  pdl_wait();
  pdl_trigger_early();
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.seq_lens[b];
  if (L < 0 || L > p.Lcap) {
    if (blockIdx.x == 0 && h == 0 && threadIdx.x == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    return;
  }
  const int i = blockIdx.x * 8 + warp;
  const int nb = (L + p.bs - 1) / p.bs;
  if (i >= nb) return;
  const int t0 = i * p.bs;
  const int t1 = min(t0 + p.bs, L);
  const int64_t base = kv_row_offset(p.pages, b, h, p.Hkv, p.Lcap, p.bs, i, 0);  // the block's rows are contiguous
  if (base < 0) {  // page index outside the pool: block skipped
    if (lane == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    return;
  }
  const uint2* src = reinterpret_cast<const uint2*>(p.k_cache + base) + lane;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int t = t0;
  for (; t + 8 <= t1; t += 8) {  // 8 rows in flight per lane
    uint2 r[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) r[u] = __ldg(src + (int64_t)(t - t0 + u) * (kHeadDim / 4));
#pragma unroll
    for (int u = 0; u < 8; ++u) add_row4(acc, r[u]);
  }
  for (; t < t1; ++t) add_row4(acc, __ldg(src + (int64_t)(t - t0) * (kHeadDim / 4)));
  const float n = (float)(t1 - t0);
  float4 m = make_float4(__fdiv_rn(acc[0], n), __fdiv_rn(acc[1], n), __fdiv_rn(acc[2], n),
                         __fdiv_rn(acc[3], n));
  const int64_t mrow = means_row_index(p.pages, p.means_per_page, b, h, p.Hkv, p.nbcap, i);
  if (mrow >= 0) store_mean(p.means, p.means_bf16, p.mean_rows, mrow, lane, m);
}

// grid (B), 256 threads.  One CTA owns a whole sequence so that the length
// it reads and the length it writes back cannot race with another CTA.
constexpr int kUpdRows = 32;                // rows staged per warp and batch
constexpr int kRowBytes = kHeadDim * 2;     // one bf16 K row
constexpr int kUpdThreads = 256;
constexpr size_t kUpdSmem = (size_t)(kUpdThreads / 32) * kUpdRows * kRowBytes;  // 64 KB

__global__ void __launch_bounds__(kUpdThreads) means_update_kernel(MeansUpdateParams p) {
  extern __shared__ __align__(16) uint8_t upd_rows[];  // [warp][kUpdRows][kRowBytes]
  pdl_wait();
  pdl_trigger_early();
  const int b = blockIdx.x;
  const int L0 = p.seq_lens[b];
  const int n = p.n_new;
  if (L0 < 0 || (int64_t)L0 + n > p.Lcap) {
    if (threadIdx.x == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
    return;
  }
  const int L1 = L0 + n;
  // 1. copy the new rows into the caches (16-byte chunks, 16 per row); a row
  //    whose page index lies outside the pool is skipped and flagged
  const int64_t chunks = (int64_t)p.Hkv * n * (kHeadDim / 8);
  for (int64_t c = threadIdx.x; c < chunks; c += blockDim.x) {
    const int h = (int)(c / ((int64_t)n * 16));
    const int64_t rem = c - (int64_t)h * n * 16;
    const int r = (int)(rem / 16), q16 = (int)(rem % 16);
    const int t = L0 + r;
    const int64_t row = kv_row_offset(p.pages, b, h, p.Hkv, p.Lcap, p.bs, t / p.bs, t % p.bs);
    if (row < 0) {
      set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
      continue;
    }
    const int64_t src = (((int64_t)b * p.Hkv + h) * n + r) * 16 + q16;
    const int64_t dst = row / 8 + q16;
    reinterpret_cast<uint4*>(p.k_cache)[dst] = reinterpret_cast<const uint4*>(p.k_new)[src];
    reinterpret_cast<uint4*>(p.v_cache)[dst] = reinterpret_cast<const uint4*>(p.v_new)[src];
  }
  // 2. recompute the mean of every touched block from its valid rows; rows
  //    below L0 come from the cache, newer rows straight from k_new.  A warp
  //    copies up to 32 rows of its block into shared memory with 16-byte
  //    cp.async (one memory round trip), then sums them in token order.
  const int first = L0 / p.bs, last = (L1 - 1) / p.bs;
  const int nblk = last - first + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const uint32_t rows_s = smem_u32(upd_rows) + (uint32_t)(warp * kUpdRows * kRowBytes);
  const uint2* rows_r = reinterpret_cast<const uint2*>(upd_rows + warp * kUpdRows * kRowBytes) + lane;
  for (int task = warp; task < p.Hkv * nblk; task += nwarps) {
    const int h = task / nblk, i = first + task % nblk;
    const int64_t pair = (int64_t)b * p.Hkv + h;
    const int t0 = i * p.bs, t1 = min(t0 + p.bs, L1);
    const int64_t base = kv_row_offset(p.pages, b, h, p.Hkv, p.Lcap, p.bs, i, 0);  // rows contiguous
    if (base < 0) {  // page index outside the pool: this block's mean is left as it was
      if (lane == 0) set_status(p.dev_status, KIN_ERR_DEVICE_DATA);
      continue;
    }
    const uint8_t* cache = reinterpret_cast<const uint8_t*>(p.k_cache + base);  // row t0 of block i
    const uint8_t* fresh = reinterpret_cast<const uint8_t*>(p.k_new + pair * n * kHeadDim);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t = t0; t < t1; t += kUpdRows) {
      const int nrows = min(kUpdRows, t1 - t);
      for (int c = lane; c < nrows * 16; c += 32) {  // 16 pieces of 16 bytes per row
        const int r = t + (c >> 4), piece = c & 15;
        const uint8_t* src = r < L0 ? cache + (int64_t)(r - t0) * kRowBytes : fresh + (int64_t)(r - L0) * kRowBytes;
        cp_async16(rows_s + (uint32_t)(c * 16), src + piece * 16, 16u);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncwarp();
      for (int r = 0; r < nrows; ++r) add_row4(acc, rows_r[r * (kRowBytes / 8)]);
      __syncwarp();  // every lane is done reading before the next batch lands
    }
    const float cnt = (float)(t1 - t0);
    float4 m = make_float4(__fdiv_rn(acc[0], cnt), __fdiv_rn(acc[1], cnt), __fdiv_rn(acc[2], cnt),
                           __fdiv_rn(acc[3], cnt));
    const int64_t mrow = means_row_index(p.pages, p.means_per_page, b, h, p.Hkv, p.nbcap, i);
    if (mrow >= 0) store_mean(p.means, p.means_bf16, p.mean_rows, mrow, lane, m);
  }
  __syncthreads();
  if (threadIdx.x == 0) p.seq_lens[b] = L1;
  pdl_trigger_late();
}

cudaError_t launch_means_build(const MeansBuildParams& p, cudaStream_t s) {
  return launch_pdl(means_build_kernel, dim3((p.nbcap + 7) / 8, p.Hkv, p.B), dim3(256), 0, s, p);
}

cudaError_t launch_means_update(const MeansUpdateParams& p, cudaStream_t s) {
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(means_update_kernel), 4, kUpdSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(means_update_kernel, dim3(p.B), dim3(kUpdThreads), kUpdSmem, s, p);
}

}  // namespace kin
