/*
 * kg_cuda.cu -- device side of the seeded synthetic input generator: fills a
 * K or V cache [B][Hkv][Lcap][D] (bf16 bits) on the GPU so that caches of
 * many GB need no host staging.  Bit-identical to kg_host.c (same kg_core.h,
 * compiled with --fmad=false so no add/mul pair is fused).
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "kg_core.h"

__global__ void kg_fill_kv_kernel(uint32_t seed, int is_k, int B, int Hkv, int Lcap, int D, int bs,
                                  const int32_t* __restrict__ seq_lens, const uint8_t* __restrict__ hh,
                                  int nbcap, int poison, uint16_t* __restrict__ out) {
  const int nd4 = D / 4;
  const int64_t groups_per_pair = (int64_t)Lcap * nd4;
  const int64_t total = (int64_t)B * Hkv * groups_per_pair;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (int64_t)gridDim.x * blockDim.x) {
    int64_t p = g / groups_per_pair;
    int64_t r = g - p * groups_per_pair;
    int t = (int)(r / nd4);
    int d4 = (int)(r - (int64_t)t * nd4);
    int b = (int)(p / Hkv);
    int L = seq_lens[b] < Lcap ? seq_lens[b] : Lcap;
    uint16_t v[4];
    if (t < L) {
      double z[4];
      kg_normal4(seed, is_k ? KG_TID_K : KG_TID_V, (uint32_t)(t * nd4 + d4), (uint32_t)p, z);
      int heavy = is_k && hh && hh[p * nbcap + t / bs];
      if (heavy) {
        double bz[4];
        kg_normal4(seed, KG_TID_BETA, (uint32_t)d4, (uint32_t)p, bz);
        for (int e = 0; e < 4; ++e) z[e] = z[e] + 2.0 * bz[e];
      }
      for (int e = 0; e < 4; ++e) v[e] = kg_d2bf16(z[e]);
    } else {
      uint16_t fill = poison ? (uint16_t)0x7FC0u : (uint16_t)0u;
      for (int e = 0; e < 4; ++e) v[e] = fill;
    }
    uint2 w;
    w.x = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
    w.y = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
    *reinterpret_cast<uint2*>(out + g * 4) = w;
  }
}

extern "C" __attribute__((visibility("default")))
int kg_cuda_fill_kv_cache(uint32_t seed, int is_k, int B, int Hkv, int Lcap, int D, int bs,
                          const int32_t* seq_lens_dev, const uint8_t* hh_dev, int nbcap, int poison,
                          uint16_t* out_dev, void* stream) {
  if (D % 4 != 0 || B <= 0 || Hkv <= 0 || Lcap <= 0 || bs <= 0) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t total = (int64_t)B * Hkv * Lcap * (D / 4);
  int64_t blocks = (total + 255) / 256;
  int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  kg_fill_kv_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      seed, is_k, B, Hkv, Lcap, D, bs, seq_lens_dev, hh_dev, nbcap, poison, out_dev);
  return (int)cudaGetLastError();
}
