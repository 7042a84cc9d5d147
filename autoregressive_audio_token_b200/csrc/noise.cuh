// noise.cuh -- counter-based Gumbel noise for the Gumbel-argmax draw.
//
// The diffusers issue "MiniMax Music 3 modular pipeline: 2.9x consumer-GPU
// speedup" (finding 3) replaces softmax + multinomial by Gumbel-argmax,
// which draws from the same distribution.  The noise is a pure function of
// (seed, frame, row key, vocab index), so a frame's draw is reproducible
// and resumable from the KV cache alone.
//
// Definition (every step an IEEE-754 operation with a single rounding):
//   mix(z)  : one SplitMix64 step from state z (Steele, Lea, Flood 2014;
//             public-domain form by S. Vigna)
//   b       = mix(mix(mix(mix(seed) ^ frame) ^ row) ^ index)
//   u       = ((b >> 40) + 0.5) * 2^-24                (fp64, exact)
//   G       = -ln(-ln u)                               (fp64, then fp32 RNE)
//   ln(x)   : x = m 2^e, m in [1/sqrt2, sqrt2), t = (m-1)/(m+1),
//             ln m = 2t * sum_{k=0..12} t^(2k) / (2k+1)  (Horner with fma),
//             ln x = fma(e, ln2, ln m)
// The ln is the classical atanh series, not a library routine, so that any
// IEEE implementation reproduces G bit for bit.
#pragma once

#include <stdint.h>

namespace m3 {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t noise_bits(uint64_t seed, uint64_t frame, uint64_t row,
                                               uint64_t index) {
  uint64_t b = mix64(seed);
  b = mix64(b ^ frame);
  b = mix64(b ^ row);
  return mix64(b ^ index);
}

__device__ __forceinline__ double series_ln(double x) {
  const unsigned long long bits = (unsigned long long)__double_as_longlong(x);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;
  double m = __longlong_as_double((long long)((bits & 0x000FFFFFFFFFFFFFull) |
                                              0x3FF0000000000000ull));
  if (m >= 1.4142135623730951) {
    m = __dmul_rn(m, 0.5);
    e += 1;
  }
  const double t = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
  const double t2 = __dmul_rn(t, t);
  double p = __ddiv_rn(1.0, 25.0);
#pragma unroll
  for (int k = 11; k >= 0; --k) p = __fma_rn(p, t2, __ddiv_rn(1.0, (double)(2 * k + 1)));
  const double lnm = __dmul_rn(__dmul_rn(2.0, t), p);
  return __fma_rn((double)e, 0.6931471805599453, lnm);
}

__device__ __forceinline__ float gumbel_noise(uint64_t seed, uint64_t frame, uint64_t row,
                                              uint64_t index) {
  const uint64_t b = noise_bits(seed, frame, row, index);
  const double u = __dmul_rn(__dadd_rn((double)(b >> 40), 0.5), 0x1p-24);
  const double a = -series_ln(u);
  return __double2float_rn(-series_ln(a));
}

}  // namespace m3
