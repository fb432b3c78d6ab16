/*
 * kg_host.c -- host (CPU) side of the seeded synthetic input generator.
 * Builds q, the K/V fields, ragged sequence lengths and the heavy-hitter
 * block choice for a decode batch.  Bit-identical to kg_cuda.cu because both
 * evaluate kg_core.h with IEEE double arithmetic and no FMA contraction.
 */
#include <stdint.h>
#include <string.h>
#include "kg_core.h"

#define KG_EXPORT __attribute__((visibility("default")))

KG_EXPORT void kg_philox(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  kg_philox4x32_10(ctr, key, out);
}
KG_EXPORT double kg_log_d(double u) { return kg_log(u); }
KG_EXPORT void kg_sincos_turns_d(double t, double* s, double* c) { kg_sincos_turns(t, s, c); }
KG_EXPORT void kg_normal4_d(uint32_t seed, uint32_t tid, uint32_t c0, uint32_t c1, double z[4]) {
  kg_normal4(seed, tid, c0, c1, z);
}
KG_EXPORT void kg_bf16_from_f32(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = kg_bf16_rne(x[i]);
}

/* q[b][j][d] ~ N(0,1), bf16 bits.  Counter (d/4, b*Hq + j). */
KG_EXPORT void kg_fill_q(uint32_t seed, int B, int Hq, int D, uint16_t* out) {
  for (int r = 0; r < B * Hq; ++r)
    for (int d4 = 0; d4 < D / 4; ++d4) {
      double z[4];
      kg_normal4(seed, KG_TID_Q, (uint32_t)d4, (uint32_t)r, z);
      for (int e = 0; e < 4; ++e) out[(int64_t)r * D + d4 * 4 + e] = kg_d2bf16(z[e]);
    }
}

/* Sequence lengths: Lmin + floor(x * (Lmax - Lmin + 1) / 2^32), x = Philox word 0. */
KG_EXPORT void kg_seq_lens(uint32_t seed, int B, int Lmin, int Lmax, int32_t* out) {
  uint64_t span = (uint64_t)(Lmax - Lmin + 1);
  for (int b = 0; b < B; ++b) {
    uint32_t ctr[4] = {(uint32_t)b, 0u, 0u, 0u}, key[2] = {seed, (uint32_t)KG_TID_LEN}, x[4];
    kg_philox4x32_10(ctr, key, x);
    out[b] = Lmin + (int32_t)(((uint64_t)x[0] * span) >> 32);
  }
}

/* Heavy-hitter blocks of every (b, kv head): m = round(nb * num / den) blocks,
 * half rounded up, chosen uniformly without replacement by selection sampling
 * (Knuth, TAOCP vol. 2, 3.4.2, Algorithm S) with integer acceptance tests.
 * nb = ceil(seq_lens[b] / bs).  out is [B][Hkv][nbcap], 1 = heavy. */
KG_EXPORT void kg_heavy_flags(uint32_t seed, int B, int Hkv, int nbcap, int bs,
                              const int32_t* seq_lens, int num, int den, uint8_t* out) {
  memset(out, 0, (size_t)B * Hkv * nbcap);
  for (int b = 0; b < B; ++b) {
    int nb = (seq_lens[b] + bs - 1) / bs;
    if (nb > nbcap) nb = nbcap;
    int64_t m = ((int64_t)nb * num * 2 + den) / (2 * (int64_t)den);
    for (int h = 0; h < Hkv; ++h) {
      uint32_t pair = (uint32_t)(b * Hkv + h);
      int64_t need = m;
      uint8_t* f = out + ((int64_t)b * Hkv + h) * nbcap;
      for (int i = 0; i < nb && need > 0; ++i) {
        uint32_t ctr[4] = {(uint32_t)i, pair, 0u, 0u}, key[2] = {seed, (uint32_t)KG_TID_HH}, x[4];
        kg_philox4x32_10(ctr, key, x);
        uint64_t remaining = (uint64_t)(nb - i);
        if ((uint64_t)x[0] * remaining < ((uint64_t)need << 32)) { f[i] = 1; --need; }
      }
    }
  }
}

/* Rows [t0, t1) of the K (is_k=1) or V field of one pair, bf16 bits [t1-t0][D].
 * hh_pair: that pair's heavy flags (only read for K). */
KG_EXPORT void kg_fill_kv_rows(uint32_t seed, int is_k, uint32_t pair, int t0, int t1,
                               int D, int bs, const uint8_t* hh_pair, uint16_t* out) {
  double beta[4 * 64];
  int nd4 = D / 4;
  if (is_k)
    for (int d4 = 0; d4 < nd4 && d4 < 64; ++d4) kg_normal4(seed, KG_TID_BETA, (uint32_t)d4, pair, beta + 4 * d4);
  for (int t = t0; t < t1; ++t) {
    int hh = is_k && hh_pair && hh_pair[t / bs];
    for (int d4 = 0; d4 < nd4; ++d4) {
      double z[4];
      kg_normal4(seed, is_k ? KG_TID_K : KG_TID_V, (uint32_t)(t * nd4 + d4), pair, z);
      for (int e = 0; e < 4; ++e) {
        double v = z[e];
        if (hh) v = v + 2.0 * beta[4 * d4 + e];
        out[(int64_t)(t - t0) * D + 4 * d4 + e] = kg_d2bf16(v);
      }
    }
  }
}

/* Whole cache [B][Hkv][Lcap][D] on the host: rows < seq_lens[b] from the field,
 * rows >= seq_lens[b] set to bf16 NaN when poison != 0, else to zero. */
KG_EXPORT void kg_fill_kv_cache(uint32_t seed, int is_k, int B, int Hkv, int Lcap, int D, int bs,
                                const int32_t* seq_lens, const uint8_t* hh, int nbcap, int poison,
                                uint16_t* out) {
  #pragma omp parallel for schedule(dynamic, 1)
  for (int p = 0; p < B * Hkv; ++p) {
    int b = p / Hkv;
    int L = seq_lens[b] < Lcap ? seq_lens[b] : Lcap;
    uint16_t* dst = out + (int64_t)p * Lcap * D;
    kg_fill_kv_rows(seed, is_k, (uint32_t)p, 0, L, D, bs, hh ? hh + (int64_t)p * nbcap : 0, dst);
    uint16_t fill = poison ? (uint16_t)0x7FC0u : (uint16_t)0u;
    for (int64_t i = (int64_t)L * D; i < (int64_t)Lcap * D; ++i) dst[i] = fill;
  }
}
