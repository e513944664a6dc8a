// Device-side helpers shared by the selective-scan kernels (sm_100a only).
//
// Element-wise math used on the hot path:
//   * bf16 <-> f32 conversion of packed pairs,
//   * packed f32x2 arithmetic (sm_100 FFMA2/FMUL2/FADD2: one issue slot for two lanes of work),
//   * 2^x on the MUFU unit (ex2.approx.ftz) and, alternatively, on the FMA pipe:
//       Cody-Waite style range reduction x = i + f with i = rint(x), |f| <= 1/2, then
//       2^f ~= 1 + f*q(f) with a cubic q fitted by the Remez exchange algorithm to minimise the
//       maximum RELATIVE error of (2^f - 1) on [-1/2, 1/2] (1.5e-5), and 2^i inserted by an
//       integer add into the exponent field.  p(0) == 1 exactly, so a step with Δ*A == 0
//       leaves the state unchanged, and the decay rate 1 - 2^x keeps a relative error of
//       1.5e-5 even when x -> 0 (long memories), which a plain absolute-error fit would not.
//   * softplus and the logistic sigmoid for the step size and the silu gate.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- bf16 packing
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }
// round-to-nearest-even of two floats into one word: low half <- lo, high half <- hi
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t f32_to_bf16(float x) {
  return (uint16_t)(pack_bf16x2(x, 0.f) & 0xffffu);
}

// ---------------------------------------------------------------- packed f32x2
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---------------------------------------------------------------- MUFU transcendental
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_mufu(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_mufu(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- 2^x on the FMA pipe
// Remez coefficients of q(f) ~ (2^f - 1)/f on [-1/2, 1/2] (max rel. error 1.5e-5).
constexpr float kQ0 = 0.6931368708610535f;
constexpr float kQ1 = 0.24023252725601196f;
constexpr float kQ2 = 0.05583728849887848f;
constexpr float kQ3 = 0.009618110954761505f;
// 1.5 * 2^23: adding it rounds |x| < 2^22 to an integer held in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;

// Two lanes of 2^(d*a) for |d*a| <= 126 (no range checks: the caller guarantees the range).
// The product d*a is folded into the range reduction: t = fma(d, a, M) rounds it to an integer,
// f = fma(d, a, -rint) recovers the fraction exactly.
__device__ __forceinline__ float2 exp2_fma_prod_x2(float2 d, float2 a) {
  const float2 t = fma2(d, a, f2(kRoundMagic));         // t = M + rint(d*a)
  const float2 r = add2(t, f2(-kRoundMagic));           // rint(d*a), exact
  const float2 f = fma2(d, a, mul2(r, f2(-1.f)));       // d*a - rint(d*a), |f| <= 1/2
  float2 q = fma2(f2(kQ3), f, f2(kQ2));
  q = fma2(q, f, f2(kQ1));
  q = fma2(q, f, f2(kQ0));
  const float2 p = fma2(q, f, f2(1.f));                 // 2^f, p(0) == 1
  // 2^i * p: add i to the exponent field.  The low bits of t's encoding are rint(d*a) offset by
  // a constant whose bits vanish when shifted left by 23.
  float2 out;
  out.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  out.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return out;
}

// Zero-order-hold input coefficient, two lanes: Ā = e^{ΔA} and g = (e^{ΔA} - 1)/A, from
// x = Δ a with a = A log2 e and ra = 1/A.  With x = i + f (i = rint(x), |f| <= 1/2) and
// 2^f = 1 + f q(f) (the cubic above), e^{ΔA} - 1 = 2^i f q(f) + (2^i - 1): as ΔA -> 0 the
// relative accuracy of f q(f) carries over, where Ā - 1 would cancel.  2^i is built in the
// exponent field.  CLAMP limits x to [-126, 126] (Ā -> 0 and g -> -1/A below; above, the true
// values overflow f32 anyway); otherwise the caller guarantees |x| <= 126.
template <bool CLAMP>
__device__ __forceinline__ void zoh_coef_x2(float2 d, float2 a, float2 ra, float2& abar, float2& g) {
  float2 t, f;
  if (CLAMP) {
    float2 x = mul2(d, a);
    x = make_float2(fminf(fmaxf(x.x, -126.f), 126.f), fminf(fmaxf(x.y, -126.f), 126.f));
    t = add2(x, f2(kRoundMagic));                           // M + rint(x)
    const float2 rn = add2(f2(kRoundMagic), make_float2(-t.x, -t.y));  // -rint(x), exact
    f = add2(x, rn);
  } else {
    t = fma2(d, a, f2(kRoundMagic));
    const float2 rn = add2(f2(kRoundMagic), make_float2(-t.x, -t.y));
    f = fma2(d, a, rn);                                     // Δ a - rint(Δ a), exact
  }
  float2 q = fma2(f2(kQ3), f, f2(kQ2));
  q = fma2(q, f, f2(kQ1));
  q = fma2(q, f, f2(kQ0));
  const float2 fq = mul2(f, q);                             // 2^f - 1
  float2 s;                                                 // 2^i: i added to the exponent of 1
  s.x = __int_as_float(0x3f800000 + (__float_as_int(t.x) << 23));
  s.y = __int_as_float(0x3f800000 + (__float_as_int(t.y) << 23));
  abar = fma2(fq, s, s);
  g = mul2(fma2(fq, s, add2(s, f2(-1.f))), ra);
}

// A rate that the zero-order-hold coefficient divides by: |A| below 1e-20 is taken as -1e-20
// (then Ā = 1 and g = Δ to f32 precision, the A -> 0 limit, with no division by zero).
__device__ __forceinline__ float zoh_rate(float A) { return fabsf(A) < 1e-20f ? -1e-20f : A; }

// ---------------------------------------------------------------- step size and gate
// softplus(v) = log(1 + e^v) to ~5e-6 relative error, for the bf16 path.
//   v > 15          : v (the remainder e^-v < 3.1e-7 of v)
//   e^v < 1/32      : series e - e^2/2 + e^3/3 - e^4/4 (truncation < 2e-7 relative)
//   otherwise       : log2(1 + e^v) * ln 2 on the MUFU unit (absolute error ~1e-7 against a
//                     result >= 0.03)
__device__ __forceinline__ float softplus_fast(float v) {
  const float e = ex2_mufu(v * kLog2e);
  const float big = lg2_mufu(1.f + e) * kLn2;
  const float small = e * fmaf(e, fmaf(e, fmaf(e, -0.25f, 0.33333334f), -0.5f), 1.f);
  const float r = e < 0.03125f ? small : big;
  return v > 15.f ? v : r;
}
// accurate softplus for the fp32 path (library log1pf/expf, ~1 ulp)
__device__ __forceinline__ float softplus_precise(float v) {
  return v > 0.f ? v + log1pf(expf(-v)) : log1pf(expf(v));
}

// two lanes of softplus_fast (same arithmetic, packed f32x2 where it applies)
__device__ __forceinline__ float2 softplus_fast_x2(float2 v) {
  const float2 s = mul2(v, f2(kLog2e));
  const float2 e = make_float2(ex2_mufu(s.x), ex2_mufu(s.y));
  const float2 onep = add2(e, f2(1.f));
  const float2 big = mul2(make_float2(lg2_mufu(onep.x), lg2_mufu(onep.y)), f2(kLn2));
  float2 sm = fma2(e, f2(-0.25f), f2(0.33333334f));
  sm = fma2(e, sm, f2(-0.5f));
  sm = fma2(e, sm, f2(1.f));
  sm = mul2(e, sm);
  return make_float2(v.x > 15.f ? v.x : (e.x < 0.03125f ? sm.x : big.x),
                     v.y > 15.f ? v.y : (e.y < 0.03125f ? sm.y : big.y));
}

// logistic sigmoid 1/(1+e^-z): MUFU ex2 + rcp (relative error ~1e-7 over the whole range;
// tanh-based forms lose relative accuracy for negative z).
__device__ __forceinline__ float sigmoid_fast(float z) { return rcp_mufu(1.f + ex2_mufu(-z * kLog2e)); }
__device__ __forceinline__ float sigmoid_precise(float z) { return 1.f / (1.f + expf(-z)); }
__device__ __forceinline__ float2 sigmoid_fast_x2(float2 z) {
  const float2 s = mul2(z, f2(-kLog2e));
  const float2 d = add2(make_float2(ex2_mufu(s.x), ex2_mufu(s.y)), f2(1.f));
  return make_float2(rcp_mufu(d.x), rcp_mufu(d.y));
}

}  // namespace ssm
