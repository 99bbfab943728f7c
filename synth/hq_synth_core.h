/*
 * hq_synth_core.h -- counter-based generator of synthetic tensor-parallel partial sums.
 *
 * This header holds none of the compression method's arithmetic.  It only turns
 * (seed, purpose, batch, rank, element) into a bf16 input value, and it is compiled
 * twice: by gcc into the host generator (hq_synth.c) and by nvcc into the device
 * generator (hq_synth_gpu.cu).  Both builds disable floating-point contraction, and
 * every step below is an IEEE-754 basic operation (+, -, *, /, sqrt, conversions),
 * so the two builds produce bit-identical values.  Transcendentals are therefore
 * written out here from their series rather than taken from libm / CUDA's math
 * library:
 *   - natural log: x = m * 2^e with m in [sqrt(1/2), sqrt(2)),
 *     ln m = 2 * atanh((m-1)/(m+1)) by its odd power series;
 *   - cos(2*pi*u): quadrant reduction, then the Taylor series of sin and cos
 *     on [0, pi/2).
 * These only have to be deterministic and accurate to ~1e-15, not correctly rounded.
 *
 * Random bits: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014).  Draw i of the stream keyed by `key` is the SplitMix64
 * output function applied to key + (i + 1) * gamma, so any element can be generated
 * on its own (counter-based).
 */
#ifndef HQ_SYNTH_CORE_H
#define HQ_SYNTH_CORE_H

#include <stdint.h>

#ifdef __CUDACC__
#define SYN_FN static __host__ __device__ __forceinline__
#else
#define SYN_FN static inline
#endif

#define SYN_GAMMA 0x9E3779B97F4A7C15ULL

/* Stream purposes. */
enum { SYN_COLSTD = 1, SYN_PERM = 2, SYN_CALIB = 3, SYN_EVAL = 4 };
/* Value distributions. */
enum { SYN_DIST_NORMAL = 0, SYN_DIST_STUDENT_T3 = 1, SYN_DIST_UNIFORM = 2 };
/* Draws reserved per element; draw 15 decides a spike. */
#define SYN_DRAWS_PER_ELEM 16ULL

SYN_FN uint64_t syn_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

SYN_FN uint64_t syn_draw(uint64_t key, uint64_t i) {
  return syn_mix(key + (i + 1ULL) * SYN_GAMMA);
}

SYN_FN uint64_t syn_key(uint64_t seed, uint64_t purpose, uint64_t batch, uint64_t rank) {
  uint64_t k = syn_draw(seed, purpose);
  k = syn_draw(k, batch);
  return syn_draw(k, rank);
}

/* Uniform double in [0, 1) from the top 53 bits: both steps are exact. */
SYN_FN double syn_u01(uint64_t u) { return (double)(u >> 11) * 0x1.0p-53; }

SYN_FN uint64_t syn_dbits(double x) {
#ifdef __CUDA_ARCH__
  return (uint64_t)__double_as_longlong(x);
#else
  union { double d; uint64_t u; } v;
  v.d = x;
  return v.u;
#endif
}

SYN_FN double syn_dfrom(uint64_t b) {
#ifdef __CUDA_ARCH__
  return __longlong_as_double((long long)b);
#else
  union { double d; uint64_t u; } v;
  v.u = b;
  return v.d;
#endif
}

/* ln x for a normal, finite x > 0. */
SYN_FN double syn_log(double x) {
  uint64_t b = syn_dbits(x);
  int e = (int)((b >> 52) & 0x7FF) - 1023;
  double m = syn_dfrom((b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL); /* [1, 2) */
  if (m > 1.4142135623730951) {
    m = m * 0.5;
    e = e + 1;
  }
  double s = (m - 1.0) / (m + 1.0);
  double s2 = s * s;
  /* sum_{j=0}^{13} s2^j / (2j+1), Horner form */
  double p = 1.0 / 27.0;
  p = p * s2 + 1.0 / 25.0;
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
  return (double)e * 0.69314718055994531 + 2.0 * s * p;
}

/* cos(2*pi*u) for u in [0, 1). */
SYN_FN double syn_cos2pi(double u) {
  double v = u * 4.0;            /* exact */
  int q = (int)v;                /* quadrant 0..3 */
  double f = v - (double)q;      /* exact, in [0, 1) */
  double a = f * 1.5707963267948966;
  double a2 = a * a;
  /* cos a = sum (-1)^n a^(2n)/(2n)!,  sin a = a * sum (-1)^n a^(2n)/(2n+1)!  (n <= 11) */
  double c = -1.0 / 1.1240007277776077e21;  /* -1/22! */
  c = c * a2 + 1.0 / 2.43290200817664e18;   /* 1/20! */
  c = c * a2 - 1.0 / 6.402373705728e15;     /* 1/18! */
  c = c * a2 + 1.0 / 20922789888000.0;      /* 1/16! */
  c = c * a2 - 1.0 / 87178291200.0;         /* 1/14! */
  c = c * a2 + 1.0 / 479001600.0;           /* 1/12! */
  c = c * a2 - 1.0 / 3628800.0;             /* 1/10! */
  c = c * a2 + 1.0 / 40320.0;               /* 1/8!  */
  c = c * a2 - 1.0 / 720.0;                 /* 1/6!  */
  c = c * a2 + 1.0 / 24.0;                  /* 1/4!  */
  c = c * a2 - 1.0 / 2.0;                   /* 1/2!  */
  c = c * a2 + 1.0;
  double s = -1.0 / 2.585201673888498e22;   /* -1/23! */
  s = s * a2 + 1.0 / 5.109094217170944e19;  /* 1/21! */
  s = s * a2 - 1.0 / 1.21645100408832e17;   /* 1/19! */
  s = s * a2 + 1.0 / 355687428096000.0;     /* 1/17! */
  s = s * a2 - 1.0 / 1307674368000.0;       /* 1/15! */
  s = s * a2 + 1.0 / 6227020800.0;          /* 1/13! */
  s = s * a2 - 1.0 / 39916800.0;            /* 1/11! */
  s = s * a2 + 1.0 / 362880.0;              /* 1/9!  */
  s = s * a2 - 1.0 / 5040.0;                /* 1/7!  */
  s = s * a2 + 1.0 / 120.0;                 /* 1/5!  */
  s = s * a2 - 1.0 / 6.0;                   /* 1/3!  */
  s = s * a2 + 1.0;
  s = s * a;
  switch (q) {
    case 0: return c;
    case 1: return -s;
    case 2: return -c;
    default: return s;
  }
}

/* Box-Muller (cosine branch) from draws d and d+1 of the element's stream. */
SYN_FN double syn_normal(uint64_t key, uint64_t d) {
  double u1 = 1.0 - syn_u01(syn_draw(key, d));  /* (0, 1] */
  double u2 = syn_u01(syn_draw(key, d + 1));
  double r = sqrt(-2.0 * syn_log(u1));
  return r * syn_cos2pi(u2);
}

/* Round a float to bf16, nearest-even; NaN becomes the quiet NaN 0x7FC0. */
SYN_FN uint16_t syn_f32_to_bf16(float f) {
#ifdef __CUDA_ARCH__
  uint32_t u = (uint32_t)__float_as_uint(f);
#else
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
#endif
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * One element x[rank][t][h] of a batch: the element's stream key is the rank's key,
 * its draws start at (t*H + h) * SYN_DRAWS_PER_ELEM.
 *   normal:     colscale[h] * N(0,1)
 *   student_t3: colscale[h] * N0 / sqrt((N1^2 + N2^2 + N3^2) / 3)
 *   uniform:    2u - 1 (colscale ignored)
 * With probability spike_p the value is multiplied by spike_mult.
 */
SYN_FN uint16_t syn_element(uint64_t rank_key, uint64_t elem, int dist, double colscale,
                            double spike_p, double spike_mult) {
  uint64_t d0 = elem * SYN_DRAWS_PER_ELEM;
  double v;
  if (dist == SYN_DIST_UNIFORM) {
    v = 2.0 * syn_u01(syn_draw(rank_key, d0)) - 1.0;
  } else if (dist == SYN_DIST_STUDENT_T3) {
    double n0 = syn_normal(rank_key, d0);
    double n1 = syn_normal(rank_key, d0 + 2);
    double n2 = syn_normal(rank_key, d0 + 4);
    double n3 = syn_normal(rank_key, d0 + 6);
    double chi = (n1 * n1 + n2 * n2) + n3 * n3;
    v = colscale * (n0 / sqrt(chi / 3.0));
  } else {
    v = colscale * syn_normal(rank_key, d0);
  }
  if (spike_p > 0.0 && syn_u01(syn_draw(rank_key, d0 + 15)) < spike_p) v = v * spike_mult;
  return syn_f32_to_bf16((float)v);
}

#endif /* HQ_SYNTH_CORE_H */
