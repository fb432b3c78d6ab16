// kin_internal.cuh -- shared device helpers and launch-parameter structs of
// libkin.so (sm_100a).  Not part of the public ABI (see include/kin.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kin.h"

namespace kin {

constexpr int kHeadDim = 128;
constexpr int kMaxGroup = 8;
constexpr int kMaxBlocksPerSeq = 32768;
constexpr int kTileTokens = 16;  // tokens per attention tile (one m16 MMA row block)

// Bounded waits give up after this many SM clock cycles (about 0.5 s at 2 GHz).
constexpr long long kWaitLimitCycles = 1000000000LL;

// ----------------------------------------------------------------- status
__device__ __forceinline__ void set_status(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// ---------------------------------------------------- order-preserving keys
// Maps fp32 bits to uint32 so that unsigned order == float order.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------- PTX: mbarriers, TMA
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of the barrier.  Gives up (returns false) after
// kWaitLimitCycles, or early once another warp has recorded KIN_ERR_TIMEOUT
// in *abort_flag (nullable), so one stuck copy cannot stall a whole grid.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  const int32_t* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (clock64() - t0 > kWaitLimitCycles) return false;
      if (abort_flag && *reinterpret_cast<const volatile int32_t*>(abort_flag) == KIN_ERR_TIMEOUT)
        return false;
    }
  }
}

// 2-D tiled TMA load global -> shared, completion counted on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// -------------------------------------------------- PTX: warp-level MMA path
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C (fp32)
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------- launch params
struct MeansBuildParams {
  const __nv_bfloat16* k_cache;
  const int32_t* seq_lens;
  float* means;
  int32_t* dev_status;
  int B, Hkv, Lcap, bs, nbcap;
};

struct MeansUpdateParams {
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float* means;
  int32_t* seq_lens;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  int32_t* dev_status;
  int B, Hkv, Lcap, bs, nbcap, n_new;
};

struct SelectParams {
  const __nv_bfloat16* q;
  const float* means;
  const int32_t* seq_lens;
  int32_t* sel_idx;
  int32_t* sel_cnt;
  float* scores;        // workspace [B*Hkv][nbcap]
  uint32_t* counters;   // workspace [B*Hkv], zero between calls
  int32_t* dev_status;
  int B, Hkv, Hq, g, bs, Lcap, nbcap, k, chunk_blocks;
  float score_scale;
};

struct AttnParams {
  const __nv_bfloat16* q;
  const int32_t* seq_lens;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  __nv_bfloat16* out;
  float* lse;
  float* partials;      // workspace [B*Hkv][max_chunks][g][D + 2]
  uint32_t* counters;   // workspace [B*Hkv], zero between calls
  int32_t* dev_status;
  int B, Hkv, Hq, g, bs, Lcap, k, chunk_blocks, max_chunks;
  float scale_log2;     // softmax_scale * log2(e)
};

// Launchers (one per kernel family); return the launch error.
cudaError_t launch_means_build(const MeansBuildParams& p, cudaStream_t s);
cudaError_t launch_means_update(const MeansUpdateParams& p, cudaStream_t s);
cudaError_t launch_select(const SelectParams& p, int grid_x, cudaStream_t s);
cudaError_t launch_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                        int grid_x, cudaStream_t s);

}  // namespace kin
