// sq_quant.cuh -- the per-token activation quantizer shared by the activation
// split kernel and the fused quantize + linear kernel, so that both take the
// same rounding decisions.
//
// Symmetric absmax INT8: s = float(absmax / 127) with a binary64 divide,
// q = round_half_away(v / s) clipped to [-127, 127] (2048ai.net section 三.1;
// rounding half away from zero).  Every step below is one IEEE binary64
// operation given by an intrinsic, so the result does not depend on
// multiply-add contraction.
#pragma once

#include <cuda_runtime.h>

namespace sq {

// The scale of a token from the absmax of its non-outlier channels.
__device__ __forceinline__ float act_scale(float absmax) {
  return __double2float_rn(__ddiv_rn((double)absmax, 127.0));
}

// 1/s for quantize_exact (any value within far less than 1/2 code of the
// true reciprocal serves; 0 for s == 0).
__device__ __forceinline__ double act_rinv(float s) {
  return s != 0.0f ? __ddiv_rn(1.0, (double)s) : 0.0;
}

// round_half_away(|v| / s) decided exactly.  t = |v| * (1/s) is within far
// less than 0.5 of the true quotient Q, so with k = floor(t) the exact test
// Q >= k + 1/2 yields the correctly rounded code whether Q lies in [k, k+1)
// or just outside it (round(Q) is k or k + 1 in every case).  The test:
//   fast path (2^-100 < s, |v| < 2^100):  (k + 1/2) * s - |v| <= 0 by one
//     fused multiply-add in binary32: it rounds the exact value once, and
//     that value is a multiple of 2^-149, so its sign survives the rounding;
//   otherwise, in binary64:  2|v| >= (2k+1) * s (both sides exact: 2k+1 has
//     at most 9 bits, s 24).
// Identical to rounding the exactly rounded binary64 quotient v/s, which for
// float v and s never lands on the wrong side of a midpoint.
__device__ __forceinline__ int quantize_exact(float v, float s, double rinv) {
  if (s == 0.0f) return 0;
  const float av = fabsf(v);
  float q;
  if (s > 0x1p-100f && av < 0x1p100f) {
    const float k = floorf(__fmul_rn(av, __double2float_rn(rinv)));
    q = fmaf(k + 0.5f, s, -av) <= 0.0f ? k + 1.0f : k;
  } else {
    const double ad = (double)av;
    const double k = floor(__dmul_rn(ad, rinv));
    const double rhs = __dmul_rn(__dadd_rn(__dadd_rn(k, k), 1.0), (double)s);
    q = (float)(__dadd_rn(ad, ad) >= rhs ? __dadd_rn(k, 1.0) : k);
  }
  q = q < 127.0f ? q : 127.0f;
  const int qi = (int)q;
  return v < 0.0f ? -qi : qi;
}

}  // namespace sq
