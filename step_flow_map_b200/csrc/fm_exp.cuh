// exp(e) in fp64 for e <= 0, the argument of every softmax weight
// exp((l - max) / T) the stochastic verify sums over a vocabulary row.
//
// Table-driven method of P. T. P. Tang ("Table-driven implementation of the
// exponential function in IEEE floating-point arithmetic", ACM TOMS 15(2),
// 1989): e = (32 q + j) ln2/32 + r with |r| <= ln2/64, so
//   exp(e) = 2^q * 2^(j/32) * exp(r),
// with 2^(j/32) from a 32-entry table (each entry the double nearest to the
// exact value) and exp(r) from its Taylor series through r^6 (the remainder
// is below 4e-18 relative for |r| <= ln2/64).  ln2/32 is split into a
// 37-bit head (k * head is exact for |k| < 2^16) and a tail, so r keeps full
// precision; k is rounded with the 1.5 * 2^52 shifter (Cody and Waite's
// trick) instead of conversion instructions.  Below e = -700 the weight (< 1e-304) is returned as 0: it
// cannot change a row sum that holds exp(0) = 1.  -inf gives 0, NaN gives
// NaN.  About a dozen fp64 operations instead of a general exp's range
// handling; the GPU tests compare it with CUDA's exp over [-700, 0].
#pragma once
#include "fm_common.cuh"

namespace fm {

// global memory read through the read-only cache: lanes of a warp index
// different entries, which constant memory would serialise
__device__ const double g_exp2_32[32] = {
    0x1.0000000000000p+0, 0x1.059b0d3158574p+0, 0x1.0b5586cf9890fp+0, 0x1.11301d0125b51p+0,
    0x1.172b83c7d517bp+0, 0x1.1d4873168b9aap+0, 0x1.2387a6e756238p+0, 0x1.29e9df51fdee1p+0,
    0x1.306fe0a31b715p+0, 0x1.371a7373aa9cbp+0, 0x1.3dea64c123422p+0, 0x1.44e086061892dp+0,
    0x1.4bfdad5362a27p+0, 0x1.5342b569d4f82p+0, 0x1.5ab07dd485429p+0, 0x1.6247eb03a5585p+0,
    0x1.6a09e667f3bcdp+0, 0x1.71f75e8ec5f74p+0, 0x1.7a11473eb0187p+0, 0x1.82589994cce13p+0,
    0x1.8ace5422aa0dbp+0, 0x1.93737b0cdc5e5p+0, 0x1.9c49182a3f090p+0, 0x1.a5503b23e255dp+0,
    0x1.ae89f995ad3adp+0, 0x1.b7f76f2fb5e47p+0, 0x1.c199bdd85529cp+0, 0x1.cb720dcef9069p+0,
    0x1.d5818dcfba487p+0, 0x1.dfc97337b9b5fp+0, 0x1.ea4afa2a490dap+0, 0x1.f50765b6e4540p+0};

__device__ __forceinline__ double exp_nonpos(double e) {
  if (!(e > -700.0)) return (e == e) ? 0.0 : e;
  // k = round(e * 32 / ln2) by adding 1.5 * 2^52 (the sum's unit in the last
  // place is 1, so the addition rounds to the nearest integer and its low
  // word holds k in two's complement): no conversion instructions
  const double t = fma(e, 0x1.71547652b82fep+5, 0x1.8p52);
  const double kf = t - 0x1.8p52;
  const int k = __double2loint(t);
  const double r = fma(-kf, 0x1.cf79abc9e3b3ap-45, fma(-kf, 0x1.62e42fefa0000p-6, e));
  double p = 1.0 / 720.0;
  p = fma(p, r, 1.0 / 120.0);
  p = fma(p, r, 1.0 / 24.0);
  p = fma(p, r, 1.0 / 6.0);
  p = fma(p, r, 0.5);
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  const int j = k & 31, q = k >> 5;                                 // q = floor(k / 32)
  // scale by 2^q through the exponent field (the result stays normal)
  return __longlong_as_double(__double_as_longlong(p * __ldg(&g_exp2_32[j])) + ((long long)q << 52));
}

}  // namespace fm
