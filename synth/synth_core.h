/*
 * synth_core.h -- the seeded synthetic-input generator shared by the fp64
 * oracle (host) and the GPU pool fill (device).
 *
 * This module draws random inputs only: packed q words, bf16 scales/biases,
 * fp32 activations and router weights.  It holds none of the expert step's
 * arithmetic (no dequant, no matvec, no routing).
 *
 * Generator: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used counter-style: draw i of stream `key`
 * is mix(key + (i+1)*GOLDEN), so any element can be regenerated on its own.
 *
 * Every floating-point step uses only IEEE-754 correctly rounded +, -, *, /
 * and sqrt on doubles, in a fixed order, so the host (gcc, -ffp-contract=off)
 * and the device (nvcc, --fmad=false) produce bit-identical values.  For that
 * reason the natural log and the cosine of Box-Muller are evaluated here from
 * their series (atanh series for ln, Taylor series for cos) instead of calling
 * libm or CUDA's math library, whose last-bit results differ.
 */
#ifndef QE_SYNTH_CORE_H
#define QE_SYNTH_CORE_H

#include <stdint.h>

#ifdef __CUDACC__
#define SY_FN static __host__ __device__ __forceinline__
#else
#define SY_FN static inline
#include <math.h>
#include <string.h>
#endif

#define SY_GOLDEN 0x9E3779B97F4A7C15ULL

/* Tensor ids: one independent stream per (seed, a, b, tensor). */
enum {
  SY_T_GATE_WQ = 1, SY_T_GATE_S = 2, SY_T_GATE_B = 3,
  SY_T_UP_WQ = 4,   SY_T_UP_S = 5,   SY_T_UP_B = 6,
  SY_T_DOWN_WQ = 7, SY_T_DOWN_S = 8, SY_T_DOWN_B = 9,
  SY_T_ROUTER = 10, SY_T_X = 11,     SY_T_PERM = 12,
  /* GatedDeltaNet decode step: state, query, key, value, decay, write strength */
  SY_T_GDN_S = 13, SY_T_GDN_Q = 14, SY_T_GDN_K = 15, SY_T_GDN_V = 16,
  SY_T_GDN_ALPHA = 17, SY_T_GDN_BETA = 18
};

/* Value kinds a fill can produce. */
enum {
  SY_K_U32 = 0,          /* raw 32 random bits per element (packed q words) */
  SY_K_BF16_UNIFORM = 1, /* bf16(float(lo + (hi-lo)*u)), u ~ U(0,1)          */
  SY_K_BF16_NORMAL = 2,  /* bf16(float(p0 * z)), z ~ N(0,1)                  */
  SY_K_F32_NORMAL = 3    /* float(p0 * z)                                    */
};

SY_FN uint64_t sy_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Draw i of the stream keyed by `key` (splitmix64 output i from state key). */
SY_FN uint64_t sy_draw(uint64_t key, uint64_t i) {
  return sy_mix(key + (i + 1ULL) * SY_GOLDEN);
}

/* Stream key of (seed, a, b, tensor); a is a layer, b an expert or token id. */
SY_FN uint64_t sy_key(uint64_t seed, uint32_t a, uint32_t b, uint32_t tensor) {
  uint64_t s = sy_mix(seed + SY_GOLDEN);
  uint64_t id = ((uint64_t)a << 40) ^ ((uint64_t)b << 8) ^ (uint64_t)tensor;
  return sy_mix(s ^ sy_mix(id + 0x632BE59BD9B4E019ULL));
}

SY_FN uint64_t sy_d2u(double d) {
#ifdef __CUDA_ARCH__
  return (uint64_t)__double_as_longlong(d);
#else
  uint64_t u; memcpy(&u, &d, 8); return u;
#endif
}
SY_FN double sy_u2d(uint64_t u) {
#ifdef __CUDA_ARCH__
  return __longlong_as_double((long long)u);
#else
  double d; memcpy(&d, &u, 8); return d;
#endif
}
SY_FN uint32_t sy_f2u(float f) {
#ifdef __CUDA_ARCH__
  return (uint32_t)__float_as_uint(f);
#else
  uint32_t u; memcpy(&u, &f, 4); return u;
#endif
}
SY_FN double sy_sqrt(double x) {
#ifdef __CUDA_ARCH__
  return __dsqrt_rn(x);
#else
  return sqrt(x);
#endif
}

/* Uniform on the open interval (0,1) from the top 53 bits. Exact. */
SY_FN double sy_uniform(uint64_t r) {
  return ((double)(r >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* ln(u) for a positive normal double: u = m * 2^e with m in [sqrt(1/2), sqrt(2)),
 * ln(m) = 2 atanh(t), t = (m-1)/(m+1), |t| <= 0.1716, atanh by its odd series
 * (14 terms, truncation below 1e-24 relative). */
SY_FN double sy_ln(double u) {
  const double LN2 = 0.6931471805599453094;
  const double SQRT2 = 1.4142135623730950488;
  uint64_t b = sy_d2u(u);
  int e = (int)((b >> 52) & 0x7FF) - 1023;
  double m = sy_u2d((b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL);
  if (m > SQRT2) { m = m * 0.5; e = e + 1; }
  double t = (m - 1.0) / (m + 1.0);
  double t2 = t * t;
  double s = 0.0;
  for (int k = 13; k >= 0; --k) s = s * t2 + 1.0 / (double)(2 * k + 1);
  return (double)e * LN2 + 2.0 * (t * s);
}

/* cos(2*pi*v) for v in (0,1): fold to theta in [0, pi/2] by the symmetries
 * cos(2pi v) = cos(2pi(1-v)) and cos(2pi a) = -cos(2pi(1/2-a)), then the
 * Taylor series of cos in nested form (15 terms, truncation below 1e-26). */
SY_FN double sy_cos2pi(double v) {
  const double TWO_PI = 6.283185307179586477;
  double a = v;
  if (a > 0.5) a = 1.0 - a;
  double sign = 1.0;
  if (a > 0.25) { a = 0.5 - a; sign = -1.0; }
  double th = a * TWO_PI;
  double th2 = th * th;
  double r = 1.0;
  for (int k = 15; k >= 1; --k) r = 1.0 - (th2 / (double)((2 * k - 1) * (2 * k))) * r;
  return sign * r;
}

/* Standard normal number i of stream `key` (Box-Muller, cosine branch). */
SY_FN double sy_normal(uint64_t key, uint64_t i) {
  double u1 = sy_uniform(sy_draw(key, 2 * i));
  double u2 = sy_uniform(sy_draw(key, 2 * i + 1));
  return sy_sqrt(-2.0 * sy_ln(u1)) * sy_cos2pi(u2);
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
SY_FN uint16_t sy_bf16_rne(float f) {
  uint32_t u = sy_f2u(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Element i of a fill of the given kind, as raw bits in the low 16/32 bits. */
SY_FN uint32_t sy_element(int kind, uint64_t key, uint64_t i, double p0, double p1) {
  switch (kind) {
    case SY_K_U32:
      return (uint32_t)(sy_draw(key, i) >> 32);
    case SY_K_BF16_UNIFORM: {
      double u = sy_uniform(sy_draw(key, i));
      return sy_bf16_rne((float)(p0 + (p1 - p0) * u));
    }
    case SY_K_BF16_NORMAL:
      return sy_bf16_rne((float)(p0 * sy_normal(key, i)));
    default: /* SY_K_F32_NORMAL */
      return sy_f2u((float)(p0 * sy_normal(key, i)));
  }
}

SY_FN int sy_kind_bytes(int kind) {
  return (kind == SY_K_BF16_UNIFORM || kind == SY_K_BF16_NORMAL) ? 2 : 4;
}

#endif /* QE_SYNTH_CORE_H */
