/*
 * kin_oracle.c -- plain, slow, fp64 CPU oracle for block top-k sparse decode
 * attention.  TEST INFRASTRUCTURE ONLY: tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may call it; the product path never does.
 * It shares no code with the CUDA library (no common headers, helpers or
 * tables); its inputs are bf16 bit patterns, widened exactly to double.
 *
 * Sources (web pages on Kinetics, cited by title and section):
 *  [P1] "Kinetics: Memory-Aware Test-Time Scaling" (skillmd.com), sections
 *       "Architecture Overview" (block-level top-k sparsity) and
 *       "Implementation", class BlockTopKAttention (scores scaled by
 *       1/sqrt(head_dim), block representation as a mean over the block,
 *       top-k over blocks, softmax then weighted sum of V).
 *  [P2] "Kinetics: Rethinking Test-Time Scaling Law" (paperhub.cn), author
 *       response Q4 "KV block size and grouping strategy" (KV budget =
 *       block size x number of top-k blocks; pairs (16,64), (32,32), (64,16))
 *       and response Q3 "Diverse prompt lengths" (ragged KV lengths).
 * Where the pages are silent the plainest reading is taken (mean key per
 * block over its valid tokens; GQA scores summed over the query heads of the
 * group; the first block and the block holding the newest token always kept
 * and counted in the budget; ties to the lower block index).
 *
 * Every function works on one (batch, kv head) pair except the batch driver
 * kin_oracle_decode_pairs, which loops over pairs with OpenMP.
 */
#define _GNU_SOURCE
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

/* exact widening of a bf16 bit pattern */
ORC_EXPORT double kin_oracle_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static int nblocks_of(int L, int bs) { return (L + bs - 1) / bs; }

/* Block means [P1 Implementation, mean over a block; read along the key axis]:
 * m_i[d] = (1/n_i) sum_{t in block i, t < L} K[t][d], n_i = valid tokens. */
ORC_EXPORT void kin_oracle_block_means(const uint16_t* K, int L, int D, int bs, double* means) {
  int nb = nblocks_of(L, bs);
  for (int i = 0; i < nb; ++i) {
    int t0 = i * bs, t1 = (i + 1) * bs < L ? (i + 1) * bs : L;
    for (int d = 0; d < D; ++d) {
      double s = 0.0;
      for (int t = t0; t < t1; ++t) s += kin_oracle_bf16_to_f64(K[(int64_t)t * D + d]);
      means[(int64_t)i * D + d] = s / (double)(t1 - t0);
    }
  }
}

/* Block scores [P1 Implementation, scores scaled by 1/sqrt(head_dim)]:
 * s_i = (1/sqrt(D)) sum_{j in group} q_j . m_i   (g query heads of one KV head). */
ORC_EXPORT void kin_oracle_block_scores(const uint16_t* q, int g, const double* means, int nb,
                                        int D, double* scores) {
  double scale = 1.0 / sqrt((double)D);
  for (int i = 0; i < nb; ++i) {
    double s = 0.0;
    for (int j = 0; j < g; ++j) {
      double dot = 0.0;
      for (int d = 0; d < D; ++d)
        dot += kin_oracle_bf16_to_f64(q[(int64_t)j * D + d]) * means[(int64_t)i * D + d];
      s += dot;
    }
    scores[i] = scale * s;
  }
}

static int cmp_desc_then_index(const void* a, const void* b, void* ctx) {
  const double* sc = (const double*)ctx;
  int ia = *(const int*)a, ib = *(const int*)b;
  if (sc[ia] > sc[ib]) return -1;
  if (sc[ia] < sc[ib]) return 1;
  return (ia > ib) - (ia < ib);
}
static int cmp_int_asc(const void* a, const void* b) {
  int ia = *(const int32_t*)a, ib = *(const int32_t*)b;
  return (ia > ib) - (ia < ib);
}

/* Block top-k [P1 Architecture Overview + Implementation (top-k over block
 * scores); P2 Q4 (budget counted in blocks)].  k is the total block budget.
 * If k >= nb every block is kept.  Otherwise the forced set F = {0, nb-1}
 * is kept and the remaining k-2 blocks are the best of 1..nb-2 ordered by
 * (score descending, index ascending).  Writes k entries: the chosen block
 * indices ascending, then -1 padding.  Returns the count, or -1 if k < 2 and
 * nb > k (the forced pair does not fit).  The ordering step is a library
 * sort (qsort_r) with that comparison. */
ORC_EXPORT int kin_oracle_select(const double* scores, int nb, int k, int32_t* sel) {
  if (k >= nb) {
    for (int i = 0; i < k; ++i) sel[i] = i < nb ? i : -1;
    return nb;
  }
  if (k < 2) return -1;
  int nc = nb - 2;
  int* cand = (int*)malloc(sizeof(int) * (nc > 0 ? nc : 1));
  for (int i = 0; i < nc; ++i) cand[i] = i + 1;
  qsort_r(cand, (size_t)nc, sizeof(int), cmp_desc_then_index, (void*)scores);
  sel[0] = 0;
  sel[1] = nb - 1;
  for (int i = 0; i < k - 2; ++i) sel[2 + i] = cand[i];
  free(cand);
  qsort(sel, (size_t)k, sizeof(int32_t), cmp_int_asc);
  return k;
}

/* Softmax attention over the tokens of a list of blocks [P1 Implementation:
 * softmax(q K^T / sqrt(d)) then weighted sum of V], unnormalised form:
 * z_t = scale q_j . K_t ; m_j = max_t z_t ; l_j = sum_t e^{z_t - m_j} ;
 * o_j = sum_t e^{z_t - m_j} V_t.  Tokens t >= L are not part of any block. */
ORC_EXPORT void kin_oracle_attend_partial(const uint16_t* q, int g, const uint16_t* K,
                                          const uint16_t* V, int L, int D, int bs,
                                          const int32_t* blocks, int nblocks, double scale,
                                          double* o, double* m, double* l) {
  int ntok = 0;
  for (int b = 0; b < nblocks; ++b) {
    int t0 = blocks[b] * bs, t1 = t0 + bs < L ? t0 + bs : L;
    if (t1 > t0) ntok += t1 - t0;
  }
  double* z = (double*)malloc(sizeof(double) * (ntok > 0 ? ntok : 1));
  for (int j = 0; j < g; ++j) {
    int c = 0;
    double mx = -INFINITY;
    for (int b = 0; b < nblocks; ++b) {
      int t0 = blocks[b] * bs, t1 = t0 + bs < L ? t0 + bs : L;
      for (int t = t0; t < t1; ++t) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
          dot += kin_oracle_bf16_to_f64(q[(int64_t)j * D + d]) *
                 kin_oracle_bf16_to_f64(K[(int64_t)t * D + d]);
        z[c] = scale * dot;
        if (z[c] > mx) mx = z[c];
        ++c;
      }
    }
    double lsum = 0.0;
    double* oj = o + (int64_t)j * D;
    for (int d = 0; d < D; ++d) oj[d] = 0.0;
    c = 0;
    for (int b = 0; b < nblocks; ++b) {
      int t0 = blocks[b] * bs, t1 = t0 + bs < L ? t0 + bs : L;
      for (int t = t0; t < t1; ++t) {
        double w = exp(z[c++] - mx);
        lsum += w;
        for (int d = 0; d < D; ++d) oj[d] += w * kin_oracle_bf16_to_f64(V[(int64_t)t * D + d]);
      }
    }
    m[j] = mx;
    l[j] = lsum;
  }
  free(z);
}

/* Log-sum-exp merge of partial softmax results (split-K decode):
 * M = max_s m_s ; o = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s ;
 * lse = M + ln sum_s e^{m_s - M} l_s.  Parts are [nparts][g][D] / [nparts][g]. */
ORC_EXPORT void kin_oracle_merge(int nparts, int g, int D, const double* o_parts,
                                 const double* m_parts, const double* l_parts, double* out,
                                 double* lse) {
  for (int j = 0; j < g; ++j) {
    double M = -INFINITY;
    for (int s = 0; s < nparts; ++s)
      if (m_parts[s * g + j] > M) M = m_parts[s * g + j];
    double den = 0.0;
    for (int d = 0; d < D; ++d) out[(int64_t)j * D + d] = 0.0;
    for (int s = 0; s < nparts; ++s) {
      double w = exp(m_parts[s * g + j] - M);
      den += w * l_parts[s * g + j];
      for (int d = 0; d < D; ++d)
        out[(int64_t)j * D + d] += w * o_parts[((int64_t)s * g + j) * D + d];
    }
    for (int d = 0; d < D; ++d) out[(int64_t)j * D + d] /= den;
    if (lse) lse[j] = M + log(den);
  }
}

/* Normalised attention over the selected blocks of one pair. */
ORC_EXPORT void kin_oracle_attend(const uint16_t* q, int g, const uint16_t* K, const uint16_t* V,
                                  int L, int D, int bs, const int32_t* blocks, int nblocks,
                                  double scale, double* out, double* lse) {
  double* o = (double*)malloc(sizeof(double) * (size_t)g * D);
  double* m = (double*)malloc(sizeof(double) * (size_t)g);
  double* l = (double*)malloc(sizeof(double) * (size_t)g);
  kin_oracle_attend_partial(q, g, K, V, L, D, bs, blocks, nblocks, scale, o, m, l);
  kin_oracle_merge(1, g, D, o, m, l, out, lse);
  free(o);
  free(m);
  free(l);
}

/* Append n rows at position L0 of one pair's cache and recompute the means
 * of every block the new rows touch (blocks L0/bs .. (L0+n-1)/bs), each from
 * its valid rows by the block-mean definition above. */
ORC_EXPORT void kin_oracle_means_update(uint16_t* Kc, uint16_t* Vc, int L0, int n,
                                        const uint16_t* knew, const uint16_t* vnew, int D, int bs,
                                        double* means) {
  if (n <= 0) return;
  memcpy(Kc + (int64_t)L0 * D, knew, sizeof(uint16_t) * (size_t)n * D);
  memcpy(Vc + (int64_t)L0 * D, vnew, sizeof(uint16_t) * (size_t)n * D);
  int L = L0 + n;
  for (int i = L0 / bs; i <= (L - 1) / bs; ++i) {
    int t0 = i * bs, t1 = (i + 1) * bs < L ? (i + 1) * bs : L;
    for (int d = 0; d < D; ++d) {
      double s = 0.0;
      for (int t = t0; t < t1; ++t) s += kin_oracle_bf16_to_f64(Kc[(int64_t)t * D + d]);
      means[(int64_t)i * D + d] = s / (double)(t1 - t0);
    }
  }
}

/* One decode step (scores, select, attend) for a list of (b, kv head) pairs
 * of a batch whose caches are [B][Hkv][Lcap][D] and whose means are
 * [B][Hkv][nbcap][D] (fp64, from kin_oracle_block_means).  Query head j uses
 * kv head j / g.  Outputs per listed pair p (index into `pairs`):
 * sel [np][k], cnt [np], out [np][g][D], lse [np][g], scores [np][nbcap]
 * (scores may be NULL).  Parallel over pairs with OpenMP (threads <= 0: all). */
ORC_EXPORT int kin_oracle_decode_pairs(int B, int Hkv, int Hq, int D, int bs, int Lcap, int nbcap,
                                       const int32_t* seq_lens, const uint16_t* q,
                                       const uint16_t* Kc, const uint16_t* Vc,
                                       const double* means, int k, double scale,
                                       const int32_t* pairs, int npairs, int32_t* sel,
                                       int32_t* cnt, double* out, double* lse, double* scores,
                                       int threads) {
  int g = Hq / Hkv;
  int bad = 0;
  int nt = threads > 0 ? threads : omp_get_max_threads();
  (void)B;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(|: bad)
  for (int pi = 0; pi < npairs; ++pi) {
    int p = pairs[pi];
    int b = p / Hkv, h = p % Hkv;
    int L = seq_lens[b];
    int nb = nblocks_of(L, bs);
    double* sc = (double*)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    const uint16_t* qg = q + ((int64_t)b * Hq + (int64_t)h * g) * D;
    kin_oracle_block_scores(qg, g, means + (int64_t)p * nbcap * D, nb, D, sc);
    if (scores) {
      for (int i = 0; i < nbcap; ++i) scores[(int64_t)pi * nbcap + i] = i < nb ? sc[i] : 0.0;
    }
    int32_t* s = sel + (int64_t)pi * k;
    int c = kin_oracle_select(sc, nb, k, s);
    cnt[pi] = c;
    if (c < 0) {
      bad |= 1;
    } else {
      kin_oracle_attend(qg, g, Kc + (int64_t)p * Lcap * D, Vc + (int64_t)p * Lcap * D, L, D, bs, s,
                        c, scale, out + (int64_t)pi * g * D, lse + (int64_t)pi * g);
    }
    free(sc);
  }
  return bad ? -1 : 0;
}
