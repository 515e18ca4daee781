// The NVFP4 quantizer of one 16-element group, shared by the activation pass (kernel 1) and
// the fused MLP epilogue (kernel 6): E4M3 block scale S = RNE(amax / (6 g)), E2M1 codes
// RNE(clamp(x / (S g), -6, 6)), both rounded from exact or correctly rounded quotients.
//
// Rounding.  amax/6 is formed by a Markstein-corrected multiplication by the rounded
// reciprocal of 6 (P. Markstein's correction: with y = RN(1/b) and q0 = RN(a y),
// q0 + RN(a - b q0) y rounds to RN(a/b)), then scaled by 1/g (a power of two) and converted
// with cvt.rn.satfinite.e4m3x2.  A code quotient x / (S g) is q0 = x r with r = rcp.approx(S g)
// followed by the same correction step; because x has at most 16 significant bits (a product
// of two bf16 values) and the E2M1 midpoints times S g at most 7, a quotient is either exactly
// a midpoint -- and then the corrected value is that midpoint exactly -- or at least 2^-16
// (relative) away from one, far beyond the few-ulp error of q.  cvt.rn.satfinite.e2m1x2 then
// rounds to nearest even.  The callers hold -x (negated smoothing factors) and the residual is
// formed as e' = q0 D - x, the quotient as q0 - e' r; the values are those of the textbook
// form, and a zero x keeps its sign in q (for x = -0: q0 = -0, e' = +0, q = -0 + -0 = -0).
#pragma once

#include "ptx.cuh"

namespace svdq {

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// RN(a / 6) for a >= 0 (Markstein correction of a * RN(1/6)).
__device__ __forceinline__ float div6(float a) {
  const float y = 0.16666667163372039794921875f;      // RN(1/6) in binary32
  const float q0 = a * y;
  const float e = fmaf(-q0, 6.0f, a);
  return fmaf(e, y, q0);
}

// Quantizes one group of 16 smoothed values given as 8 pairs of -x (see the
// rounding note above): returns the E4M3 scale code and writes 8 code bytes.
__device__ __forceinline__ uint32_t quantize_group(const uint64_t (&nx)[8], float g, float inv_g, uint2& out) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) f32x2_unpack(nx[i], a[2 * i], a[2 * i + 1]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) amax = fmax3(amax, fabsf(a[i]), fabsf(a[i + 1]));
  const uint32_t sc = cvt_e4m3x2(div6(amax) * inv_g, 0.f) & 0xFFu;
  float S, unused;
  e4m3x2_to_f32(sc, S, unused);
  const float D = S * g;
  if (D == 0.f) {
    out = make_uint2(0u, 0u);
    return 0u;
  }
  const float rn = -rcp_approx(D);
  const uint64_t rn2 = f32x2_pack(rn, rn), D2 = f32x2_pack(D, D);
  float q[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t q0 = f32x2_mul(nx[i], rn2);            // x_hat r
    const uint64_t e = f32x2_fma(q0, D2, nx[i]);          // q0 D - x_hat, exact
    f32x2_unpack(f32x2_fma(e, rn2, q0), q[2 * i], q[2 * i + 1]);   // q0 - e r
  }
  out.x = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
  out.y = cvt_e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  return sc;
}

}  // namespace svdq
