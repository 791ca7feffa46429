// exp2_poly.cuh -- software 2^x on the FMA pipe, and the hardware ex2.
//
// FlashAttention-4 ("The Technical Edge": exponentials approximated with cubic
// polynomials on CUDA cores to relieve the SFU; "B. Remplacer le Couteau
// Lourd") gives neither coefficients nor a range reduction; this one is ours:
//
//   x <- max(x, -126)              (keeps the result a normal fp32 number)
//   j  = floor(x)                  (add of 1.5 * 2^23 rounded toward -inf)
//   f  = x - j  in [0, 1)          (exact)
//   p  = ((c3 f + c2) f + c1) f + 1   ~ 2^f, p >= 1   (3 FMA)
//   2^x ~= p * 2^j                 (integer add of j into the exponent field)
//
// c1..c3 minimise the maximum relative error of p(f) / 2^f on [0, 1) with
// p(0) = 1 pinned (Remez exchange, derive_exp2_poly.py): 8.6e-5, far below
// the bf16 half-ulp (2^-9) that P is rounded to.  Valid for x in [-126, 64);
// x < -126 returns 2^-126 instead of 0, so masked (-inf) logits must go
// through the hardware path.
#pragma once

#define FA_EXP2_C0 1.000000000e+00f
#define FA_EXP2_C1 6.951167583e-01f
#define FA_EXP2_C2 2.276449949e-01f
#define FA_EXP2_C3 7.706703991e-02f

namespace fa {

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float kShift = 12582912.0f;  // 1.5 * 2^23: x + kShift rounded down is floor(x) + kShift
  const float t = __fadd_rd(x, kShift);
  const float j = __fsub_rn(t, kShift);
  const float f = __fsub_rn(x, j);
  float p = fmaf(FA_EXP2_C3, f, FA_EXP2_C2);
  p = fmaf(p, f, FA_EXP2_C1);
  p = fmaf(p, f, FA_EXP2_C0);
  const int ji = __float_as_int(t) - 0x4B400000;
  return __int_as_float(__float_as_int(p) + (ji << 23));
}

// exp2_poly on two values at once with packed fp32x2 arithmetic; the result is
// bit for bit that of exp2_poly on each lane (every operation rounds the same
// exact value: x - j is computed as fma(j, -1, x), and adding t << 23 to the
// bits of p equals adding j << 23 because 0x4B400000 << 23 vanishes mod 2^32).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rd(x, make_float2(12582912.0f, 12582912.0f));
  const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(FA_EXP2_C3, FA_EXP2_C3), f, make_float2(FA_EXP2_C2, FA_EXP2_C2));
  p = __ffma2_rn(p, f, make_float2(FA_EXP2_C1, FA_EXP2_C1));
  p = __ffma2_rn(p, f, make_float2(FA_EXP2_C0, FA_EXP2_C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Hardware 2^x on the SFU (MUFU): ex2.approx, flush-to-zero; ex2(-inf) = +0.
__device__ __forceinline__ float exp2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace fa
