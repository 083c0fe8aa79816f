// sq_quant.cuh -- the per-token activation quantizer shared by the activation
// split kernel and the fused quantize + linear kernel, so that both take the
// same rounding decisions.
//
// Symmetric absmax INT8: s = float(absmax / 127) with a binary64 divide,
// q = round_half_away(v / s) clipped to [-127, 127] (2048ai.net section 三.1;
// rounding half away from zero).  Every step below is one IEEE operation
// given by an intrinsic (or an explicit fused multiply-add), so the result
// does not depend on multiply-add contraction.
#pragma once

#include <cuda_runtime.h>

namespace sq {

// The scale of a token from the absmax of its non-outlier channels:
// float(a / 127) with the quotient rounded once, to binary32.  This equals
// rounding the binary64 quotient to binary32: a/127 has a binary expansion
// of period 7 (127 = 2^7 - 1), so the binary64 rounding can never land on a
// binary32 midpoint.
__device__ __forceinline__ float act_scale(float absmax) { return __fdiv_rn(absmax, 127.0f); }

// 1/s for quantize_exact: any value within far less than 1/2 code of the
// true reciprocal serves (0 for s == 0).
__device__ __forceinline__ float act_rinv(float s) { return s != 0.0f ? __frcp_rn(s) : 0.0f; }

// round_half_away(|v| / s) decided exactly.  t = |v| * (1/s) is within far
// less than 0.5 of the true quotient Q, so with k = floor(t) the exact test
// Q >= k + 1/2 yields the correctly rounded code whether Q lies in [k, k+1)
// or just outside it (round(Q) is k or k + 1 in every case).  The test:
//   common case (2^-100 < s, |v| < 2^100):  (k + 1/2) * s - |v| <= 0 by one
//     binary32 fused multiply-add: it rounds the exact value once, and that
//     value is a multiple of 2^-149, so its sign survives the rounding;
//   otherwise, in binary64:  2|v| >= (2k+1) * s (both sides exact: 2k+1 has
//     at most 9 bits, s 24), with k from a binary64 quotient.
// Identical to rounding the exactly rounded binary64 quotient v/s, which for
// float v and s never lands on the wrong side of a midpoint.
// The common case of quantize_exact without its range test: valid when the
// token's scale is above 2^-100 and every |v| quantized is below 2^100 (the
// caller decides once per token from the scale and the absmax).
__device__ __forceinline__ bool quantize_fast_ok(float s, float absmax) {
  return s > 0x1p-100f && absmax < 0x1p100f;
}
// floor(t) for 0 <= t < 2^22 without a conversion instruction: t + 2^23
// rounded down is 2^23 + floor(t) exactly, whose low mantissa bits are the
// integer.
__device__ __forceinline__ int quantize_fast(float v, float s, float rinv) {
  const float av = fabsf(v);
  const float f = __fadd_rd(__fmul_rn(av, rinv), 8388608.0f);  // 2^23 + k
  const float k = __fsub_rn(f, 8388608.0f);
  int q = (__float_as_int(f) - 0x4B000000) + (fmaf(k + 0.5f, s, -av) <= 0.0f ? 1 : 0);
  q = min(q, 127);
  return v < 0.0f ? -q : q;
}

__device__ __forceinline__ int quantize_exact(float v, float s, float rinv) {
  if (s == 0.0f) return 0;
  const float av = fabsf(v);
  float q;
  if (s > 0x1p-100f && av < 0x1p100f) {
    const float k = floorf(__fmul_rn(av, rinv));
    q = fmaf(k + 0.5f, s, -av) <= 0.0f ? k + 1.0f : k;
  } else {
    const double ad = (double)av, sd = (double)s;
    const double k = floor(__ddiv_rn(ad, sd));
    const double rhs = __dmul_rn(__dadd_rn(__dadd_rn(k, k), 1.0), sd);
    q = (float)(__dadd_rn(ad, ad) >= rhs ? __dadd_rn(k, 1.0) : k);
  }
  q = q < 127.0f ? q : 127.0f;
  const int qi = (int)q;
  return v < 0.0f ? -qi : qi;
}

// ---- four channels at a time (K % 4 == 0): the outlier bits of channels
// 4 j4 .. 4 j4 + 3 from a bitmap (bit j % 32 of word j / 32), their absmax
// and their four codes packed into one word (channel 4 j4 in the low byte).
__device__ __forceinline__ uint32_t omask_nibble(const uint32_t* omask, int j4) {
  return (omask[j4 >> 3] >> ((j4 & 7) * 4)) & 0xFu;  // outlier bits of channels 4*j4 .. 4*j4+3
}

template <bool FAST>
__device__ __forceinline__ int qcode(float v, float s, float rinv) {
  return FAST ? quantize_fast(v, s, rinv) : quantize_exact(v, s, rinv);
}
template <bool FAST>
__device__ __forceinline__ uint32_t pack_codes(float4 v, uint32_t om, float s, float rinv) {
  const int q0 = (om & 1u) ? 0 : qcode<FAST>(v.x, s, rinv);
  const int q1 = (om & 2u) ? 0 : qcode<FAST>(v.y, s, rinv);
  const int q2 = (om & 4u) ? 0 : qcode<FAST>(v.z, s, rinv);
  const int q3 = (om & 8u) ? 0 : qcode<FAST>(v.w, s, rinv);
  return (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
         ((uint32_t)(q3 & 0xFF) << 24);
}

__device__ __forceinline__ float absmax4(float4 v, uint32_t om, float a, bool& nonfinite) {
  nonfinite |= !isfinite(v.x) || !isfinite(v.y) || !isfinite(v.z) || !isfinite(v.w);
  if (!(om & 1u)) a = fmaxf(a, fabsf(v.x));
  if (!(om & 2u)) a = fmaxf(a, fabsf(v.y));
  if (!(om & 4u)) a = fmaxf(a, fabsf(v.z));
  if (!(om & 8u)) a = fmaxf(a, fabsf(v.w));
  return a;
}

}  // namespace sq
