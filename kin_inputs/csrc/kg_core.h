/*
 * kg_core.h -- seeded synthetic input generator shared by the host library
 * (gcc) and the device library (nvcc).  It holds none of the attention
 * method's arithmetic: only a counter-based random number generator, a
 * normal transform and the float -> bf16 rounding used to build inputs.
 *
 * Every value is a pure function of (seed, stream id, counter), so any slice
 * of a tensor can be regenerated on the host without materialising the rest.
 * Host and device builds must produce identical bits, so every step is
 * integer arithmetic or IEEE-754 double add/mul/div/sqrt with FMA contraction
 * disabled at compile time (gcc -ffp-contract=off, nvcc --fmad=false).
 *
 * Published definitions followed:
 *  - Philox4x32-10: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
 *    "Parallel random numbers: as easy as 1, 2, 3", SC'11, section 4.
 *  - Box-Muller transform: G. E. P. Box, M. E. Muller, "A note on the
 *    generation of random normal deviates", Ann. Math. Stat. 29 (1958).
 *  - ln(m) by the series ln(m) = 2 atanh((m-1)/(m+1)) on m in [1/sqrt2, sqrt2];
 *    sin/cos by their Taylor series on [-pi/4, pi/4] after an exact
 *    quarter-turn reduction.  Both are written out here from the mathematics.
 */
#ifndef KG_CORE_H
#define KG_CORE_H

#include <stdint.h>
#if !defined(__CUDACC__)
#include <math.h>
#endif

#if defined(__CUDACC__)
#define KG_FN static __host__ __device__ __forceinline__
#else
#define KG_FN static inline
#endif

/* stream ids: one independent Philox key per tensor of a synthetic case */
enum {
  KG_TID_Q = 1,     /* q [B,Hq,D] */
  KG_TID_K = 2,     /* K field [B,Hkv,t,D] */
  KG_TID_V = 3,     /* V field [B,Hkv,t,D] */
  KG_TID_BETA = 4,  /* heavy-hitter key bias [B,Hkv,D] */
  KG_TID_HH = 5,    /* heavy-hitter block choice */
  KG_TID_LEN = 6    /* ragged sequence lengths [B] */
};

#define KG_PHILOX_M0 0xD2511F53u
#define KG_PHILOX_M1 0xCD9E8D57u
#define KG_PHILOX_W0 0x9E3779B9u
#define KG_PHILOX_W1 0xBB67AE85u

/* Philox4x32 with 10 rounds: counter c[4], key k[2] -> out[4]. */
KG_FN void kg_philox4x32_10(const uint32_t c_in[4], const uint32_t k_in[2], uint32_t out[4]) {
  uint32_t c0 = c_in[0], c1 = c_in[1], c2 = c_in[2], c3 = c_in[3];
  uint32_t k0 = k_in[0], k1 = k_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += KG_PHILOX_W0; k1 += KG_PHILOX_W1; }
    uint64_t p0 = (uint64_t)KG_PHILOX_M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)KG_PHILOX_M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* uniform in the open interval (0, 1): (x + 1/2) / 2^32, exact in double */
KG_FN double kg_u01(uint32_t x) { return ((double)x + 0.5) * (1.0 / 4294967296.0); }

KG_FN uint64_t kg_dbits(double x) {
  union { double d; uint64_t u; } c; c.d = x; return c.u;
}
KG_FN double kg_bitsd(uint64_t u) {
  union { double d; uint64_t u; } c; c.u = u; return c.d;
}

/* natural log of a normal positive double u (u in (0,1) here) */
KG_FN double kg_log(double u) {
  uint64_t b = kg_dbits(u);
  int e = (int)((b >> 52) & 0x7FF) - 1023;
  double m = kg_bitsd((b & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull); /* [1,2) */
  if (m > 1.4142135623730951) { m = m * 0.5; e += 1; }
  double s = (m - 1.0) / (m + 1.0);
  double s2 = s * s;
  /* 2 s sum_{n=0..12} s2^n / (2n+1), |s| <= 0.1716 -> truncation < 1e-19 */
  double p = 1.0 / 25.0;
  p = p * s2 + 1.0 / 23.0;
  p = p * s2 + 1.0 / 21.0;
  p = p * s2 + 1.0 / 19.0;
  p = p * s2 + 1.0 / 17.0;
  p = p * s2 + 1.0 / 15.0;
  p = p * s2 + 1.0 / 13.0;
  p = p * s2 + 1.0 / 11.0;
  p = p * s2 + 1.0 / 9.0;
  p = p * s2 + 1.0 / 7.0;
  p = p * s2 + 1.0 / 5.0;
  p = p * s2 + 1.0 / 3.0;
  p = p * s2 + 1.0;
  double lnm = 2.0 * s * p;
  return (double)e * 0.6931471805599453 + lnm;
}

/* sin and cos of 2*pi*t for t in [0,1) */
KG_FN void kg_sincos_turns(double t, double* s_out, double* c_out) {
  double t4 = t * 4.0;                 /* exact */
  int q = (int)t4;                     /* floor, t4 >= 0 */
  double f = t4 - (double)q;           /* exact, [0,1) */
  if (f >= 0.5) { f = f - 1.0; q += 1; }
  double x = f * 1.5707963267948966;   /* [-pi/4, pi/4] */
  double x2 = x * x;
  /* sin x = x sum_{n=0..8} (-1)^n x^{2n} / (2n+1)! */
  double sp = 1.0 / 355687428096000.0;          /* 1/17! */
  sp = sp * x2 - 1.0 / 1307674368000.0;         /* 1/15! */
  sp = sp * x2 + 1.0 / 6227020800.0;            /* 1/13! */
  sp = sp * x2 - 1.0 / 39916800.0;              /* 1/11! */
  sp = sp * x2 + 1.0 / 362880.0;                /* 1/9!  */
  sp = sp * x2 - 1.0 / 5040.0;                  /* 1/7!  */
  sp = sp * x2 + 1.0 / 120.0;                   /* 1/5!  */
  sp = sp * x2 - 1.0 / 6.0;                     /* 1/3!  */
  sp = sp * x2 + 1.0;
  double sn = x * sp;
  /* cos x = sum_{n=0..9} (-1)^n x^{2n} / (2n)! */
  double cp = -1.0 / 6402373705728000.0;        /* 1/18! */
  cp = cp * x2 + 1.0 / 20922789888000.0;        /* 1/16! */
  cp = cp * x2 - 1.0 / 87178291200.0;           /* 1/14! */
  cp = cp * x2 + 1.0 / 479001600.0;             /* 1/12! */
  cp = cp * x2 - 1.0 / 3628800.0;               /* 1/10! */
  cp = cp * x2 + 1.0 / 40320.0;                 /* 1/8!  */
  cp = cp * x2 - 1.0 / 720.0;                   /* 1/6!  */
  cp = cp * x2 + 1.0 / 24.0;                    /* 1/4!  */
  cp = cp * x2 - 1.0 / 2.0;                     /* 1/2!  */
  cp = cp * x2 + 1.0;
  double cs = cp;
  switch (q & 3) {
    case 0: *s_out = sn; *c_out = cs; break;
    case 1: *s_out = cs; *c_out = -sn; break;
    case 2: *s_out = -sn; *c_out = -cs; break;
    default: *s_out = -cs; *c_out = sn; break;
  }
}

/* Four N(0,1) deviates (double) from one Philox block: Box-Muller on the
 * pairs (out0, out1) and (out2, out3); element j of the group of four is
 * r*cos for even j and r*sin for odd j. */
KG_FN void kg_normal4(uint32_t seed, uint32_t tid, uint32_t c0, uint32_t c1, double z[4]) {
  uint32_t ctr[4] = {c0, c1, 0u, 0u};
  uint32_t key[2] = {seed, tid};
  uint32_t x[4];
  kg_philox4x32_10(ctr, key, x);
  for (int p = 0; p < 2; ++p) {
    double u1 = kg_u01(x[2 * p]);
    double u2 = kg_u01(x[2 * p + 1]);
    double r = sqrt(-2.0 * kg_log(u1));
    double sn, cs;
    kg_sincos_turns(u2, &sn, &cs);
    z[2 * p] = r * cs;
    z[2 * p + 1] = r * sn;
  }
}

KG_FN uint32_t kg_fbits(float x) {
  union { float f; uint32_t u; } c; c.f = x; return c.u;
}

/* IEEE float -> bf16 bits, round to nearest even; NaN -> canonical quiet NaN */
KG_FN uint16_t kg_bf16_rne(float x) {
  uint32_t u = kg_fbits(x);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)0x7FC0u;
  uint32_t bias = 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)((u + bias) >> 16);
}

KG_FN uint16_t kg_d2bf16(double v) { return kg_bf16_rne((float)v); }

/* One element of a K or V field of pair p = b*Hkv + h, token row t, dim d.
 * K gets 2*beta[p][d] added when its block is a heavy hitter (hh != 0). */
KG_FN double kg_kv_value(uint32_t seed, int is_k, uint32_t pair, uint32_t t,
                         uint32_t d, int D, int hh) {
  double z[4];
  uint32_t grp = t * (uint32_t)(D / 4) + d / 4u;
  kg_normal4(seed, is_k ? (uint32_t)KG_TID_K : (uint32_t)KG_TID_V, grp, pair, z);
  double v = z[d & 3u];
  if (is_k && hh) {
    double bz[4];
    kg_normal4(seed, (uint32_t)KG_TID_BETA, d / 4u, pair, bz);
    v = v + 2.0 * bz[d & 3u];
  }
  return v;
}

#endif /* KG_CORE_H */
