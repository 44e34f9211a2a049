/*
 * synth_core.h -- counter-based seeded generator for the synthetic inputs
 * (embeddings X, projection Y, MLP weights W_j, compression weights W_L and
 * LayerNorm affine parameters).
 *
 * This header is the ONLY source shared by the fp64 oracle side and the CUDA
 * side. It holds no arithmetic of the Wukong layer: it only turns
 * (seed, tensor id, element index) into a number and rounds that number to the
 * storage type. Both sides compile this same source (gcc with
 * -ffp-contract=off for the host, nvcc with -fmad=false for the device), and
 * every step below is an integer operation or one of +, -, *, /, sqrt, which
 * IEEE 754 rounds the same way on both, so both sides see identical bits.
 *
 * Definition (every value is a pure function of its coordinates):
 *   mix(z)        SplitMix64 finaliser: z += 0x9E3779B97F4A7C15, then the two
 *                 xor-shift-multiply rounds and a final xor-shift (Steele,
 *                 Lea & Flood, "Fast splittable pseudorandom number
 *                 generators", OOPSLA 2014).
 *   key(s, t)     = mix(mix(s) ^ (t * 0xD1B54A32D192ED03))
 *   bits(key, c)  = mix(key + c * 0x9E3779B97F4A7C15)
 *   u_open(b)     = ((b >> 11) + 1) * 2^-53      in (0, 1]
 *   u_half(b)     = (b >> 11) * 2^-53            in [0, 1)
 *   normal(key,i) : Box-Muller (Box & Muller 1958) on the pair p = i >> 1,
 *                   u1 = u_open(bits(key, 2p)), u2 = u_half(bits(key, 2p+1)),
 *                   r = sqrt(-2 ln u1), even i -> r cos(2 pi u2),
 *                   odd i -> r sin(2 pi u2).
 *   ln, cos, sin and exp are evaluated by the short series below (written
 *   here from their Taylor / atanh expansions), not by a math library, so
 *   that the host and the device agree to the bit.
 *   Storage rounding: double -> bf16 by round-to-nearest-even directly on the
 *   double's bits; double -> fp32 by the IEEE conversion (nearest-even).
 */
#ifndef WK_SYNTH_CORE_H
#define WK_SYNTH_CORE_H

#include <stdint.h>
#if !defined(__CUDACC__)
#include <math.h>
#endif

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

/* storage types of a generated tensor */
enum { SYNTH_F32 = 0, SYNTH_BF16 = 1 };

SYNTH_HD uint64_t synth_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

SYNTH_HD uint64_t synth_key(uint64_t seed, uint64_t tensor_id) {
  return synth_mix(synth_mix(seed) ^ (tensor_id * 0xD1B54A32D192ED03ull));
}

SYNTH_HD uint64_t synth_bits(uint64_t key, uint64_t counter) {
  return synth_mix(key + counter * 0x9E3779B97F4A7C15ull);
}

SYNTH_HD double synth_u64_as_f64(uint64_t b) {
  union { uint64_t u; double d; } v;
  v.u = b;
  return v.d;
}

SYNTH_HD uint64_t synth_f64_as_u64(double d) {
  union { uint64_t u; double d; } v;
  v.d = d;
  return v.u;
}

/* 2^-53 */
#define SYNTH_TWO_M53 (1.0 / 9007199254740992.0)

SYNTH_HD double synth_u_open(uint64_t b) { return (double)((b >> 11) + 1ull) * SYNTH_TWO_M53; }
SYNTH_HD double synth_u_half(uint64_t b) { return (double)(b >> 11) * SYNTH_TWO_M53; }

/* ln 2 and pi/2 as exact binary literals */
#define SYNTH_LN2 0x1.62e42fefa39efp-1
#define SYNTH_LN10 0x1.26bb1bbb55516p+1
#define SYNTH_PI_2 0x1.921fb54442d18p+0
#define SYNTH_SQRT2 0x1.6a09e667f3bcdp+0

/* Natural log of a positive normal double x:
 * x = m * 2^e with m in (sqrt(1/2), sqrt(2)], ln m = 2 atanh(s), s = (m-1)/(m+1),
 * 2 atanh(s) = 2 s (1 + s^2/3 + s^4/5 + ... + s^22/23); |s| <= 0.1716 so the
 * dropped tail is below 1e-18 relative. The coefficients 1/(2j+1) are written
 * as exact binary literals (the nearest doubles to 1/3, 1/5, ...). */
SYNTH_HD double synth_log(double x) {
  uint64_t b = synth_f64_as_u64(x);
  int e = (int)((b >> 52) & 0x7ffull) - 1023;
  double m = synth_u64_as_f64((b & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull);
  if (m > SYNTH_SQRT2) {
    m = m * 0.5;
    e = e + 1;
  }
  double s = (m - 1.0) / (m + 1.0);
  double s2 = s * s;
  double p = 0x1.642c8590b2164p-5;     /* 1/23 */
  p = p * s2 + 0x1.8618618618618p-5;   /* 1/21 */
  p = p * s2 + 0x1.af286bca1af28p-5;   /* 1/19 */
  p = p * s2 + 0x1.e1e1e1e1e1e1ep-5;   /* 1/17 */
  p = p * s2 + 0x1.1111111111111p-4;   /* 1/15 */
  p = p * s2 + 0x1.3b13b13b13b14p-4;   /* 1/13 */
  p = p * s2 + 0x1.745d1745d1746p-4;   /* 1/11 */
  p = p * s2 + 0x1.c71c71c71c71cp-4;   /* 1/9 */
  p = p * s2 + 0x1.2492492492492p-3;   /* 1/7 */
  p = p * s2 + 0x1.999999999999ap-3;   /* 1/5 */
  p = p * s2 + 0x1.5555555555555p-2;   /* 1/3 */
  p = p * s2 + 1.0;
  return (double)e * SYNTH_LN2 + 2.0 * s * p;
}

/* cos and sin of an angle t in [0, pi/4] by their Maclaurin series, nested as
 * sin t = t (1 - t^2/(2*3) (1 - t^2/(4*5) (1 - ...))) and
 * cos t = 1 - t^2/(1*2) (1 - t^2/(3*4) (1 - ...)), ten factors each; the
 * factors 1/((2j)(2j+1)) and 1/((2j-1)(2j)) are exact binary literals. */
SYNTH_HD void synth_cos_sin_small(double t, double* c, double* s) {
  const double ks[10] = {0x1.5555555555555p-3, 0x1.999999999999ap-5, 0x1.8618618618618p-6,
                         0x1.c71c71c71c71cp-7, 0x1.29e4129e4129ep-7, 0x1.a41a41a41a41ap-8,
                         0x1.3813813813814p-8, 0x1.e1e1e1e1e1e1ep-9, 0x1.7f405fd017f40p-9,
                         0x1.3813813813814p-9};
  const double kc[10] = {0x1.0000000000000p-1, 0x1.5555555555555p-4, 0x1.1111111111111p-5,
                         0x1.2492492492492p-6, 0x1.6c16c16c16c17p-7, 0x1.f07c1f07c1f08p-8,
                         0x1.6816816816817p-8, 0x1.1111111111111p-8, 0x1.ac5701ac5701bp-9,
                         0x1.58ed2308158edp-9};
  double t2 = t * t;
  double rs = 1.0, rc = 1.0;
  for (int j = 9; j >= 0; --j) {
    rs = 1.0 - (t2 * ks[j]) * rs;
    rc = 1.0 - (t2 * kc[j]) * rc;
  }
  *s = t * rs;
  *c = rc;
}

/* cos(2 pi u), sin(2 pi u) for u in [0, 1) */
SYNTH_HD void synth_cos_sin_2pi(double u, double* c, double* s) {
  double v = 4.0 * u;          /* exact */
  int q = (int)v;              /* quadrant 0..3 */
  double f = v - (double)q;    /* exact, in [0, 1) */
  int swap = f > 0.5;
  if (swap) f = 1.0 - f;       /* exact (Sterbenz) */
  double c0, s0;
  synth_cos_sin_small(f * SYNTH_PI_2, &c0, &s0);
  if (swap) {                  /* cos(pi/2 - a) = sin a, sin(pi/2 - a) = cos a */
    double tmp = c0;
    c0 = s0;
    s0 = tmp;
  }
  switch (q & 3) {
    case 0: *c = c0;  *s = s0;  break;
    case 1: *c = -s0; *s = c0;  break;
    case 2: *c = -c0; *s = -s0; break;
    default: *c = s0; *s = -c0; break;
  }
}

/* exp(x) for |x| < 700: x = k ln2 + r, |r| <= ln2/2, exp(r) = 1 + r(1 + r/2(1 + r/3(...)))
 * to 18 terms (factors 1/j as exact binary literals), then scaled by 2^k
 * through the exponent bits (exact). */
SYNTH_HD double synth_exp(double x) {
  const double inv[18] = {0x1.0000000000000p+0, 0x1.0000000000000p-1, 0x1.5555555555555p-2,
                          0x1.0000000000000p-2, 0x1.999999999999ap-3, 0x1.5555555555555p-3,
                          0x1.2492492492492p-3, 0x1.0000000000000p-3, 0x1.c71c71c71c71cp-4,
                          0x1.999999999999ap-4, 0x1.745d1745d1746p-4, 0x1.5555555555555p-4,
                          0x1.3b13b13b13b14p-4, 0x1.2492492492492p-4, 0x1.1111111111111p-4,
                          0x1.0000000000000p-4, 0x1.e1e1e1e1e1e1ep-5, 0x1.c71c71c71c71cp-5};
  double kf = x / SYNTH_LN2;
  int k = (int)(kf < 0.0 ? kf - 0.5 : kf + 0.5);
  double r = x - (double)k * SYNTH_LN2;
  double p = 1.0;
  for (int j = 17; j >= 0; --j) p = 1.0 + (r * inv[j]) * p;
  uint64_t scale_bits = (uint64_t)(1023 + k) << 52;
  return p * synth_u64_as_f64(scale_bits);
}

SYNTH_HD double synth_normal(uint64_t key, uint64_t i) {
  uint64_t pair = i >> 1;
  double u1 = synth_u_open(synth_bits(key, 2ull * pair));
  double u2 = synth_u_half(synth_bits(key, 2ull * pair + 1ull));
  double r = sqrt(-2.0 * synth_log(u1));
  double c, s;
  synth_cos_sin_2pi(u2, &c, &s);
  return (i & 1ull) ? r * s : r * c;
}

/* LogUniform(lo=0.1, hi=10): exp(U(ln 0.1, ln 10)) = exp((2u - 1) ln 10) */
SYNTH_HD double synth_log_uniform_01_10(uint64_t key, uint64_t i) {
  double u = synth_u_half(synth_bits(key, i));
  return synth_exp((2.0 * u - 1.0) * SYNTH_LN10);
}

/* double -> bf16 bits, round to nearest, ties to even, straight from the double.
 * Magnitudes below the smallest normal bf16 flush to a signed zero; the generator
 * never produces them in practice (|x| < 2^-126). */
SYNTH_HD uint16_t synth_f64_to_bf16(double x) {
  uint64_t b = synth_f64_as_u64(x);
  uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  int e = (int)((b >> 52) & 0x7ffull) - 1023 + 127;
  uint64_t mant = b & 0x000FFFFFFFFFFFFFull;
  if (e <= 0) return sign;
  if (e >= 255) return (uint16_t)(sign | 0x7F80u);
  uint64_t keep = mant >> 45;
  uint64_t rem = mant & ((1ull << 45) - 1ull);
  uint64_t half = 1ull << 44;
  if (rem > half || (rem == half && (keep & 1ull))) keep += 1ull;
  if (keep == 128ull) {
    keep = 0ull;
    e += 1;
    if (e >= 255) return (uint16_t)(sign | 0x7F80u);
  }
  return (uint16_t)(sign | (uint16_t)(e << 7) | (uint16_t)keep);
}

#endif /* WK_SYNTH_CORE_H */
