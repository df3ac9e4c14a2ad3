// softmax_sm100.cuh -- the per-tile online-softmax step of the attention
// kernels: one thread owns one query row of a 128-key S tile held in
// registers; it finds the row maximum, turns S into P = 2^(S*scale*log2(e) - m)
// in bf16 over the front of the S row in TMEM, and returns the fp32 row sum.
//
// Throughput notes (sm_100a):
//  * the row maximum uses 3-input max instructions in eight independent
//    chains, so it is not one 128-long dependency chain;
//  * scaling, sums and the polynomial use packed f32x2 FMA/ADD instructions;
//  * exponentials run on the MUFU ex2 unit; an FMA-pipe alternative,
//    2^j * p(f) with j = round(y), f = y - j and p the degree-3 minimax fit of
//    2^f on [-1/2, 1/2] (coefficients from fit_exp2.py, relative error 7.5e-5,
//    far below bf16's 2^-8), can take a share of them (SWATTN_POLY_SEL).
#pragma once

#include <stdint.h>

#include "ptx_sm100.cuh"

namespace swattn {

// Degree-3 fit of 2^f on [-1/2, 1/2]; see fit_exp2.py.
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
// Adding 1.5 * 2^23 rounds a float of magnitude < 2^22 to the nearest integer,
// which then sits in the low mantissa bits of the sum.
constexpr float kRoundMagic = 12582912.0f;
// Which element pairs (index i of 16 per 32-column chunk) take the FMA-pipe
// exponential instead of MUFU ex2.  Measured on B200 the softmax is bound by
// instruction issue, not by MUFU throughput, so the cheaper MUFU path is used
// for every pair; the polynomial stays available (and tested) for a kernel
// that is MUFU-bound, e.g. by defining this as ((i) & 3) == 3.
#ifndef SWATTN_POLY_SEL
#define SWATTN_POLY_SEL(i) false
#endif

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) in one packed instruction.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                      float c0, float c1) {
  const float2 d = __ffma2_rn(make_float2(a0, a1), make_float2(b0, b1), make_float2(c0, c1));
  d0 = d.x;
  d1 = d.y;
}

// (d0, d1) = (a0 + b0, a1 + b1) in one packed instruction.
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  const float2 d = __fadd2_rn(make_float2(a0, a1), make_float2(b0, b1));
  d0 = d.x;
  d1 = d.y;
}

// 2^y for a pair, on the FMA and integer pipes.  y is clamped below at -125
// (results under 2^-125 are far below what bf16 P can hold next to the row
// maximum's 1); y may be as large as the rescale threshold.
__device__ __forceinline__ void exp2_poly2(float y0, float y1, float& e0, float& e1) {
  y0 = fmaxf(y0, -125.0f);
  y1 = fmaxf(y1, -125.0f);
  float t0, t1, jn0, jn1, f0, f1;
  fadd2(t0, t1, y0, y1, kRoundMagic, kRoundMagic);            // t = y + M, rounds y to j
  ffma2(jn0, jn1, t0, t1, -1.0f, -1.0f, kRoundMagic, kRoundMagic);   // M - t = -j
  fadd2(f0, f1, y0, y1, jn0, jn1);                            // f = y - j in [-1/2, 1/2]
  float p0, p1;
  ffma2(p0, p1, f0, f1, kExp2C3, kExp2C3, kExp2C2, kExp2C2);
  ffma2(p0, p1, p0, p1, f0, f1, kExp2C1, kExp2C1);
  ffma2(p0, p1, p0, p1, f0, f1, kExp2C0, kExp2C0);
  // 2^j * p: add j to the exponent field.  bits(t) = bits(M) + j and
  // bits(M) << 23 vanishes modulo 2^32, so bits(t) << 23 = j << 23.
  e0 = __int_as_float(__float_as_int(p0) + __float_as_int(t0) * 8388608);
  e1 = __int_as_float(__float_as_int(p1) + __float_as_int(t1) * 8388608);
}

// Maximum of 128 values: eight independent chains of 3-input maxima.
__device__ __forceinline__ float row_max128(const float (&x)[128]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmax3f(x[k], x[k + 8], x[k + 16]);
#pragma unroll
  for (int i = 24; i < 120; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmax3f(m[k], x[i + k], x[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], x[120 + k]);
  return fmax3f(fmax3f(m[0], m[1], m[2]), fmax3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// P for half h of a 128-column S row in registers (columns 64h .. 64h+63):
// 32 packed bf16 pairs in pk (pk[i] holds columns 64h+2i, 64h+2i+1), for one
// 32-column TMEM store.  Returns the fp32 sum.  kPartial: columns >= kv_valid
// are padding keys (P = 0).
template <bool kPartial, int kHalf>
__device__ __forceinline__ float softmax_half_to_pk(const float (&x)[128], int kv_valid, float sl2,
                                                    float neg_m, uint32_t (&pk)[32]) {
  float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int col = 64 * kHalf + 2 * i;
    float y0, y1, p0, p1;
    ffma2(y0, y1, x[col], x[col + 1], sl2, sl2, neg_m, neg_m);
    if (SWATTN_POLY_SEL(i & 15)) {
      exp2_poly2(y0, y1, p0, p1);
    } else {
      p0 = ex2_approx(y0);
      p1 = ex2_approx(y1);
    }
    if (kPartial) {
      p0 = col < kv_valid ? p0 : 0.0f;
      p1 = col + 1 < kv_valid ? p1 : 0.0f;
    }
    if (i & 1)
      fadd2(s2, s3, s2, s3, p0, p1);
    else
      fadd2(s0, s1, s0, s1, p0, p1);
    pk[i] = pack_bf16x2(p0, p1);
  }
  return (s0 + s1) + (s2 + s3);
}

}  // namespace swattn
