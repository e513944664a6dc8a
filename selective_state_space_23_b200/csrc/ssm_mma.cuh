// Warp-level bf16 tensor-core helpers and the B/C tile ring shared by the chunked matrix form of
// the scalar-decay scan (ssm_ssd.cu) and its backward (ssm_ssd_bwd.cu), sm_100a.
#pragma once

#include <stdint.h>

#include "ssm_device.cuh"

namespace ssm {
namespace ssd {

constexpr int kT = 16;       // steps per chunk (one MMA k-step)
constexpr int kLdS = 24;     // bf16 per shared tile row: 16 steps + 8 pad (48-byte rows)
constexpr int kStages = 4;   // B/C ring depth (chunks)

template <int N>
struct SsdStage {
  uint16_t Bs[N * kLdS];  // B of the chunk as [n][t]
  uint16_t Cs[N * kLdS];  // C of the chunk as [n][t]
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two floats as a pair of bf16 words with a + b ~= hi + lo to about 16 significant bits: hi the
// nearest bf16 values, lo the nearest bf16 values of the remainders.  A product whose operand
// is not a bf16 input takes two MMAs (hi and lo against an exact bf16 operand), or three when
// both operands are split (hi.hi + hi.lo + lo.hi; the lo.lo term is below f32 rounding).
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  // (a, b) - hi as one packed f32x2 operation; the differences are exact either way
  const float2 r = fma2(make_float2(bf16_lo(hi), bf16_hi(hi)), make_float2(-1.f, -1.f),
                        make_float2(a, b));
  lo = pack_bf16x2(r.x, r.y);
}

// Zero-order-hold input coefficient of a step Δ with one rate A per channel (the chunked form):
// c = (e^{ΔA} - 1)/A (library expm1f; Δ as A -> 0), its derivatives dc/dΔ = e^{ΔA} and
// dc/dA = Δ² φ'(ΔA) with φ(z) = (e^z - 1)/z: the series 1/2 + z/3 + z²/8 + z³/30 + z⁴/144 for
// |z| < 1/8 (truncation below 4e-8 relative), else (Δ e^{ΔA} - c)/A, which no longer cancels.
__device__ __forceinline__ float zoh_c(float d, float A) {
  return fabsf(A) < 1e-20f ? d : expm1f(d * A) / A;
}
__device__ __forceinline__ float zoh_dc_da(float d, float A, float c) {
  const float z = d * A;
  if (fabsf(z) < 0.125f)
    return d * d * fmaf(z, fmaf(z, fmaf(z, fmaf(z, 1.f / 144.f, 1.f / 30.f), 0.125f), 1.f / 3.f), 0.5f);
  return (d * expf(z) - c) / A;
}

// The transpose of an 8x8 b16 matrix held one pair per lane (lane l: row l / 4, cols 2 (l % 4),
// +1), returned in the same layout.
__device__ __forceinline__ uint32_t movt(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}
// A 16x16 tile held as an A fragment ({rows 0-7 | 8-15} x {cols 0-7 | 8-15}: a[0] rows lo cols
// lo, a[1] rows hi cols lo, a[2] rows lo cols hi, a[3] rows hi cols hi) -> the A fragment of
// its transpose (what ldmatrix .trans of the tile in shared memory would give).
__device__ __forceinline__ void frag_t(uint32_t (&r)[4], const uint32_t (&a)[4]) {
  r[0] = movt(a[0]);
  r[1] = movt(a[2]);
  r[2] = movt(a[1]);
  r[3] = movt(a[3]);
}

// Four 8x8 bf16 matrices from shared memory; lane i gives the address of row i % 8 of matrix
// i / 8.  Plain: lane l receives (row l / 4, cols 2 (l % 4), +1) of each; .trans: the transpose.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
// The lane's row address for the four 8x8 blocks (rows n0 .. n0+7 | n0+8 .., cols 0..7 | 8..15)
// of a [n][t] tile: matrix m = lane / 8 covers rows n0 + 8 (m / 2) .., cols 8 (m % 2) ..
__device__ __forceinline__ const uint16_t* blk(const uint16_t* tile, int n0, int lane, int ld = kLdS) {
  return tile + (n0 + ((lane >> 4) << 3) + (lane & 7)) * ld + (((lane >> 3) & 1) << 3);
}

__device__ __forceinline__ void cp16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int K>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(K) : "memory"); }

}  // namespace ssd
}  // namespace ssm
