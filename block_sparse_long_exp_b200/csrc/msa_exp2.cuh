// msa_exp2.cuh — 2^x on the FMA and integer pipes, without the special
// function unit.
//
// The softmax of a 128 x 128 score tile needs 16384 exponentials; at 16 per
// clock on an SM's special function units that is as long as the tile's two
// MMAs.  Computing part of a row's exponentials with this function moves them
// to the FMA pipe (128 lanes per clock), so both pipes share the work.
//
// Method (textbook range reduction plus a polynomial):
//   1. x is clamped below at -125 (so the result stays a normal float);
//   2. n = rint(x) by adding and subtracting 1.5 * 2^23 (round to nearest
//      even is the hardware rounding of the addition; the sum's low mantissa
//      bits then hold n), f = x - n lies in [-1/2, 1/2] and is exact;
//   3. 2^f = p(f), a degree-3 polynomial with the smallest largest relative
//      error on [-1/2, 1/2] (Remez exchange; coefficients from
//      exp2_poly_fit.py in this directory, rounded to fp32), evaluated by
//      Horner's rule with fused multiply-adds;
//   4. 2^x = p(f) * 2^n by adding n to p's exponent field.
// Largest relative error 7.5e-5 (the fit's 7.48e-5 plus fp32 rounding),
// far below bf16's half unit in the last place (2^-9), the precision P is
// stored in for the PV product.
// Domain: x in [-125, 127] gives the value above; x < -125 (-inf included)
// gives exactly 0; NaN gives 0.  Callers pass x = (s - m) * scale * log2(e)
// <= 8 (the lazily rescaled running maximum is at most 8 below the true one).
//
// Plain fp32 arithmetic with explicitly rounded operations: the same code
// compiled for the host gives bit-identical results, which is how its error
// is tested without a GPU.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>
#ifndef __CUDACC__
#define MSA_HD inline
#else
#define MSA_HD __host__ __device__ __forceinline__
#endif

namespace msa {

namespace exp2_detail {

MSA_HD float add_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fadd_rn(a, b);  // never contracted or reassociated
#else
  volatile float s = a + b;
  return s;
#endif
}

MSA_HD float fma_rn(float a, float b, float c) {
#ifdef __CUDA_ARCH__
  return __fmaf_rn(a, b, c);
#else
  return std::fmaf(a, b, c);
#endif
}

MSA_HD uint32_t bits(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(x);
#else
  uint32_t u;
  std::memcpy(&u, &x, 4);
  return u;
#endif
}

MSA_HD float from_bits(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float x;
  std::memcpy(&x, &u, 4);
  return x;
#endif
}

}  // namespace exp2_detail

// 2^x without the special function unit (see the file comment).
MSA_HD float exp2_fma(float x) {
  using namespace exp2_detail;
  const float kRound = 12582912.0f;            // 1.5 * 2^23
  const float c0 = 0x1.fff692p-1f, c1 = 0x1.62f31ap-1f, c2 = 0x1.f0de1ap-3f, c3 = 0x1.c3f76p-5f;
  const bool live = x >= -125.0f;              // false for -inf and NaN
  const float xc = live ? x : -125.0f;
  const float j = add_rn(xc, kRound);          // 1.5 * 2^23 + rint(x), exact
  const float n = add_rn(j, -kRound);
  const float f = add_rn(xc, -n);              // in [-1/2, 1/2], exact
  float p = fma_rn(c3, f, c2);
  p = fma_rn(p, f, c1);
  p = fma_rn(p, f, c0);
  const uint32_t shift = (bits(j) - bits(kRound)) << 23;   // n in the exponent field (mod 2^32)
  const float r = from_bits(bits(p) + shift);
  return live ? r : 0.0f;
}

}  // namespace msa

#undef MSA_HD
