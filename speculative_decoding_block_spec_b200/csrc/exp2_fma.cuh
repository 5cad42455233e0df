// 2^y on the FMA pipe, for the row-statistics hot loop.
//
// The softmax normaliser needs one base-2 exponential per logit. The
// hardware exp2 (MUFU ex2.approx) runs on the SM's narrow transcendental
// unit, whose rate caps the streaming kernels just below the HBM bandwidth;
// computing a fixed share of the exponentials with fused multiply-adds
// instead moves that work to the wide FP32 pipe.
//
// Method (written from the mathematics):
//  1. Range reduction in base 2 (as in Cody and Waite, "Software Manual for
//     the Elementary Functions", 1980, here exact): y = n + f with n the
//     integer nearest y and f in [-1/2, 1/2]. Adding 1.5 * 2^23 rounds y to
//     an integer held in the low mantissa bits of the sum, so n and f come
//     out exactly with three additions.
//  2. 2^f by the degree-5 polynomial of minimax relative error on
//     [-1/2, 1/2] (Remez exchange; the coefficients and their error are
//     produced by exp2_poly.py beside this file), in Horner form with fused
//     multiply-adds. Relative error of the polynomial with float32
//     coefficients: 1.55e-7.
//  3. 2^n * 2^f by adding n to the exponent field of 2^f (an integer add of
//     n << 23 to its bits; n << 23 is the sum's low bits shifted up).
// Domain: y <= 0 (the kernels pass (x - max) * log2(e) / T). Arguments
// below -125 give 2^-125 (a term below 1e-37 of the row's largest, which is
// 1); a NaN argument gives NaN. The function compiles for the device and
// for the host alike (the host copy is what the CPU tests measure; both use
// IEEE round-to-nearest float arithmetic and a fused multiply-add, so they
// produce the same bits).
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>

#if defined(__CUDACC__)
#define SPECV_HD __host__ __device__ __forceinline__
#else
#define SPECV_HD inline
#endif

namespace specv {

SPECV_HD int32_t f32_bits(float x) {
#if defined(__CUDA_ARCH__)
  return __float_as_int(x);
#else
  int32_t i;
  std::memcpy(&i, &x, sizeof i);
  return i;
#endif
}

SPECV_HD float bits_f32(int32_t i) {
#if defined(__CUDA_ARCH__)
  return __int_as_float(i);
#else
  float x;
  std::memcpy(&x, &i, sizeof x);
  return x;
#endif
}

SPECV_HD float fma_f32(float a, float b, float c) {
#if defined(__CUDA_ARCH__)
  return __fmaf_rn(a, b, c);
#else
  return std::fma(a, b, c);
#endif
}

SPECV_HD float exp2_fma(float y) {
  // minimax coefficients of 2^f on [-1/2, 1/2], degree 5 (exp2_poly.py)
  constexpr float c0 = 1.000000119e+00f, c1 = 6.931469440e-01f, c2 = 2.402212024e-01f;
  constexpr float c3 = 5.550713092e-02f, c4 = 9.675540961e-03f, c5 = 1.327647245e-03f;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float yc = y > -125.0f ? y : -125.0f;  // NaN takes the clamp here and is restored below
  const float t = yc + kRound;
  const float n = t - kRound;
  const float f = yc - n;
  float p = c5;
  p = fma_f32(p, f, c4);
  p = fma_f32(p, f, c3);
  p = fma_f32(p, f, c2);
  p = fma_f32(p, f, c1);
  p = fma_f32(p, f, c0);
  const float r = bits_f32(f32_bits(p) + static_cast<int32_t>(static_cast<uint32_t>(f32_bits(t)) << 23));
  return y == y ? r : y;
}

}  // namespace specv
