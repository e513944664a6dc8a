// Backward pass of the selective scan with state recomputation, sm_100a.
//
// The pages say only that the intermediate states are recomputed on chip in the backward pass
// instead of being stored ("Mamba: ..." summary page, "Donanım Duyarlı Durum Genişletme").
// The gradient formulas are the chain rule through the forward recurrence (see the forward
// kernel for the notation):
//   g_t  = dout_t * silu(z_t)                                   (dL/dy_t)
//   λ_t  = g_t C_t + Ā_{t+1} λ_{t+1},  λ_{L-1} = g_{L-1} C_{L-1} + dhL
//   dB_t = Σ_d λ_t Δ_t x_t        dC_t = Σ_d g_t h_t
//   du_t = g_t D + Δ_t Σ_n λ_t B_t
//   dΔ_t = Σ_n λ_t (A Ā_t h_{t-1} + B_t x_t),   ddelta_t = dΔ_t * sigmoid(delta_t + dt_bias)
//   dA   = Σ_{b,t} λ_t Δ_t Ā_t h_{t-1},  dD = Σ_{b,t} g_t x_t,  ddt_bias = Σ_{b,t} ddelta_t
//   dz_t = dout_t y_t silu'(z_t),  dh0 = Ā_0 λ_0
// with Ā_t h_{t-1} = h_t - Δ_t B_t x_t, so the reverse sweep needs only h_t.  With the
// zero-order-hold input term ("Yöntem": B̄ = (ΔA)^{-1}(e^{ΔA} - I) ΔB) the coefficient of B_t x_t
// is c = (e^{ΔA} - 1)/A per state instead of Δ: dB_t = Σ_d λ_t c x_t, du_t = g_t D + Σ_n λ_t c B_t,
// dΔ_t = Σ_n λ_t Ā_t (A h_{t-1} + B_t x_t) (dc/dΔ = Ā) and dA gains λ_t (dc/dA) B_t x_t with
// dc/dA = (Δ Ā - c)/A, or Δ^2 (1/2 + y/3 + y^2/8) for |y = ΔA| < 0.01 where that form cancels.
//
// Mapping: two lanes per channel, 8 states each in registers; a warp holds 16 consecutive d of
// one batch row.  Time is walked backwards in 16-step blocks; each block is handled in two halves
// (upper then lower 8 steps): the lanes reload the state entering the block (a checkpoint written
// by the forward pass, or by a state-only replay pass), replay forward to the end of the half,
// parking h_t of the half's 8 steps in shared memory, then run the adjoint recurrence backwards
// over the half, recomputing Ā_t.  Per-step scalars (Δ, Δx, g) are computed once per (channel,
// step) and shared through shared memory; the two half-lanes combine their sums with one shuffle.
// dB and dC (sums over the channel axis) are transposed through shared memory two steps at a
// time, summed with vector loads and one shuffle level, and written as one partial per
// (CTA, b, n, t); a finishing kernel adds the partials in a fixed order (deterministic).
#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"
#include "ssm_rows.cuh"

namespace ssm {
namespace {

constexpr int kHB = 8;                  // steps per half block = states per lane
constexpr int kCW = 16;                 // channels per warp (two lanes per channel)
constexpr int kTS = kCW + 1;            // padded step stride of the per-step tables
constexpr int kParkS = kHB * kHB + 4;   // per-lane parked states: 8 steps x 8 states (+4: banks)
constexpr int kRedS = 36;               // per-lane row of the dB/dC transpose: 2 steps x 16 (+4)

// Per-warp shared memory of one 16-step block.
struct BwdTile {
  float4 sB[kBlk * kNS / 4];   // B_t,n as f32 [step][state]
  float4 sC[kBlk * kNS / 4];   // C_t,n
  float2 sd[kBlk * kTS];       // (Δ_t, Δ_t x_t) per [step][channel slot]
  float sg[kBlk * kTS];        // g_t = dout_t silu(z_t)
  float ys[kBlk * kTS];        // y_t = C_t.h_t + D x_t without D x_t (for dz)
  float2 sS[kBlk * kTS];       // (Σ_n λ B, Σ_n A λ Ā h_{t-1}) of each step
  float park[32 * kParkS];     // per lane: h_t of the 8 steps of the current half block
  float red[32 * kRedS];       // dB/dC values of two steps, transposed to sum over channels
  float wres[kBlk * 32];       // the warp's channel sums [step][half * 16 + (dB n | dC n)]
};
static_assert(sizeof(BwdTile) % 16 == 0, "per-warp tiles keep 16-byte alignment");

// Ā and the ZOH coefficient c = (e^{ΔA} - 1)/A of two states: library expf/expm1f on the fp32
// path, the FMA-pipe form (zoh_coef_x2) on the bf16 path.  al = A (fp32) or A log2 e (bf16).
template <bool PRECISE, bool CLAMP>
__device__ __forceinline__ void zoh_pair(float2 d2, float2 al, float2 ra, float2& av, float2& c) {
  if (PRECISE) {
    const float2 y = mul2(d2, al);
    av = make_float2(expf(y.x), expf(y.y));
    c = mul2(make_float2(expm1f(y.x), expm1f(y.y)), ra);
  } else {
    zoh_coef_x2<CLAMP>(d2, al, ra, av, c);
  }
}

__device__ __forceinline__ float2 dx2_of(float2 dd) { return f2(dd.y); }

// One replayed step for one lane (8 states): h <- Ā h + Δ x B.  KP of the 4 state pairs take 2^x
// from MUFU, the rest from the FMA-pipe polynomial (only used in range-checked blocks).  Returns
// the partial readout Σ C h over the lane's states when READOUT.
template <bool PRECISE, bool READOUT, int KP>
__device__ __forceinline__ float replay_step(float2 (&hh)[4], const float2 (&al)[4],
                                             const float2 (&ra)[4], float2 dd, const float4* bq,
                                             const float4* cq) {
  constexpr bool kZoh = KP == kKpZoh || KP == kKpZohClamped;
  const float2 d2 = f2(dd.x), dx2 = f2(dd.y);  // (Δ, Δx), or (Δ, x) with the ZOH term
  const float4 b0 = bq[0], b1 = bq[1];
  float4 c0 = make_float4(0.f, 0.f, 0.f, 0.f), c1 = c0;
  if (READOUT) {
    c0 = cq[0];
    c1 = cq[1];
  }
  float2 ya = make_float2(0.f, 0.f), yb = ya;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 bb = j < 2 ? b0 : b1;
    const float2 bp = (j & 1) ? make_float2(bb.z, bb.w) : make_float2(bb.x, bb.y);
    float2 av, bx = dx2;
    if (kZoh) {
      float2 c;
      zoh_pair<PRECISE, KP == kKpZohClamped>(d2, al[j], ra[j], av, c);
      bx = mul2(c, dx2);
    } else if (PRECISE) {
      av = make_float2(expf(dd.x * al[j].x), expf(dd.x * al[j].y));
    } else if (j < KP) {
      const float2 x = mul2(d2, al[j]);
      av = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
    } else {
      av = exp2_fma_prod_x2(d2, al[j]);
    }
    hh[j] = fma2(av, hh[j], mul2(bx, bp));
    if (READOUT) {
      const float4 cc = j < 2 ? c0 : c1;
      const float2 cp = (j & 1) ? make_float2(cc.z, cc.w) : make_float2(cc.x, cc.y);
      if (j & 1) yb = fma2(cp, hh[j], yb);
      else ya = fma2(cp, hh[j], ya);
    }
  }
  const float2 ys = add2(ya, yb);
  return ys.x + ys.y;
}

// One adjoint step for one lane: completes λ_t, forms the dB/dC contributions (into `vals`),
// accumulates dA, Σ λB and Σ A λ Ā h_{t-1}, and advances λ <- Ā_t λ_t.
template <bool PRECISE, int KP>
__device__ __forceinline__ void adjoint_step(float2 (&lam)[4], float2 (&dA)[4], const float2 (&al)[4],
                                             const float2 (&ra)[4], float aback,
                                             const float2 (&hk)[4], float2 dd, float g, float live,
                                             const float4* bq, const float4* cq, float2 (&vals)[8],
                                             float& S1, float& S2, float& S3) {
  constexpr bool kZoh = KP == kKpZoh || KP == kKpZohClamped;
  const float2 d2 = f2(dd.x), ndx2 = f2(-dd.y), g2 = f2(g);
  const float2 dxl = f2(dd.y * live), gl = f2(g * live);
  const float4 b0 = bq[0], b1 = bq[1], c0 = cq[0], c1 = cq[1];
  float2 s1 = make_float2(0.f, 0.f), s2 = s1, s3 = s1;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 bb = j < 2 ? b0 : b1;
    const float4 cc = j < 2 ? c0 : c1;
    const float2 bp = (j & 1) ? make_float2(bb.z, bb.w) : make_float2(bb.x, bb.y);
    const float2 cp = (j & 1) ? make_float2(cc.z, cc.w) : make_float2(cc.x, cc.y);
    float2 av;
    if (kZoh) {
      // (Δ, x) in dd; c = (e^{ΔA} - 1)/A per state
      float2 c;
      zoh_pair<PRECISE, KP == kKpZohClamped>(d2, al[j], ra[j], av, c);
      lam[j] = fma2(g2, cp, lam[j]);                        // λ_t complete
      const float2 cx = mul2(c, dx2_of(dd));
      vals[j] = mul2(lam[j], mul2(cx, f2(live)));           // dB_t contribution: λ c x
      vals[4 + j] = mul2(gl, hk[j]);                        // dC_t contribution: g h_t
      const float2 qv = fma2(make_float2(-cx.x, -cx.y), bp, hk[j]);  // Ā h_{t-1} = h_t - c x B
      const float2 lq = mul2(lam[j], qv);
      s1 = fma2(mul2(lam[j], c), bp, s1);                   // Σ λ c B        (du)
      s2 = fma2(al[j], lq, s2);                             // Σ A λ Ā h_{t-1} (dΔ, / aback)
      s3 = fma2(mul2(lam[j], av), bp, s3);                  // Σ λ Ā B        (dΔ, times x)
      // dc/dA: direct form, or its series where |ΔA| < 0.01
      const float2 y = mul2(mul2(d2, al[j]), f2(aback));
      const float2 ser = mul2(mul2(d2, d2), fma2(fma2(y, f2(0.125f), f2(1.f / 3.f)), y, f2(0.5f)));
      const float2 dir = mul2(fma2(d2, av, make_float2(-c.x, -c.y)), ra[j]);
      const float2 dcda = make_float2(fabsf(y.x) < 1e-2f ? ser.x : dir.x, fabsf(y.y) < 1e-2f ? ser.y : dir.y);
      dA[j] = fma2(d2, lq, fma2(mul2(lam[j], mul2(dcda, dx2_of(dd))), bp, dA[j]));
      lam[j] = mul2(lam[j], av);                            // Ā_t λ_t, for step t-1
      continue;
    }
    if (PRECISE) {
      av = make_float2(expf(dd.x * al[j].x), expf(dd.x * al[j].y));
    } else if (j < KP) {
      const float2 x = mul2(d2, al[j]);
      av = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
    } else {
      av = exp2_fma_prod_x2(d2, al[j]);
    }
    lam[j] = fma2(g2, cp, lam[j]);              // λ_t complete
    vals[j] = mul2(lam[j], dxl);                // dB_t contribution: λ Δ x
    vals[4 + j] = mul2(gl, hk[j]);              // dC_t contribution: g h_t
    const float2 qv = fma2(ndx2, bp, hk[j]);    // Ā_t h_{t-1} = h_t - Δ x B
    const float2 lq = mul2(lam[j], qv);
    s1 = fma2(lam[j], bp, s1);
    s2 = fma2(al[j], lq, s2);
    dA[j] = fma2(d2, lq, dA[j]);
    lam[j] = mul2(lam[j], av);                  // Ā_t λ_t, for step t-1
  }
  S1 = s1.x + s1.y;
  S2 = s2.x + s2.y;
  S3 = s3.x + s3.y;
}

// Sum the dB/dC values of two steps over the warp's 16 channels.  Row `lane` of `red` holds the
// lane's 32 values (step slot s = 0, 1; 8 dB then 8 dC of its half of the states).  Lane j sums
// one 4-value quad of one step over 8 channels with vector loads, one shuffle adds the other 8,
// and lanes 0..15 store the warp sums.
__device__ __forceinline__ void reduce_two_steps(BwdTile& tl, int lane, int k0, int k1) {
  __syncwarp();
  const int quad = lane & 3, s = (lane >> 2) & 1, qq = (lane >> 3) & 1, rg = lane >> 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 2 * (8 * rg + i) + qq;
    const float4 v = *reinterpret_cast<const float4*>(tl.red + r * kRedS + s * 16 + quad * 4);
    const float2 lo = add2(make_float2(acc.x, acc.y), make_float2(v.x, v.y));
    const float2 hi = add2(make_float2(acc.z, acc.w), make_float2(v.z, v.w));
    acc = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
  acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
  acc.z += __shfl_xor_sync(0xffffffffu, acc.z, 16);
  acc.w += __shfl_xor_sync(0xffffffffu, acc.w, 16);
  const int kk = s == 0 ? k0 : k1;
  if (rg == 0 && kk >= 0) *reinterpret_cast<float4*>(tl.wres + kk * 32 + qq * 16 + quad * 4) = acc;
  __syncwarp();
}

// Replay a block from its entering state and run the adjoint over steps [lo, hi).
template <bool PRECISE, int KP>
__device__ __forceinline__ void half_pass(BwdTile& tl, const float2 (&hstart)[4], float2 (&lam)[4],
                                          float2 (&dA)[4], const float2 (&al)[4],
                                          const float2 (&ra)[4], float aback,
                                          float live, int lane, int slot, int q, int lo, int hi) {
  constexpr bool kZoh = KP == kKpZoh || KP == kKpZohClamped;
  const float4* bq = tl.sB + 2 * q;
  const float4* cq = tl.sC + 2 * q;
  float* prow = tl.park + lane * kParkS;
  float2 hh[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) hh[j] = hstart[j];
#pragma unroll 1
  for (int k = 0; k < lo; ++k)
    replay_step<PRECISE, false, KP>(hh, al, ra, tl.sd[k * kTS + slot], bq + k * 4, cq);
#pragma unroll 1
  for (int k = lo; k < hi; ++k) {
    float y = replay_step<PRECISE, true, KP>(hh, al, ra, tl.sd[k * kTS + slot], bq + k * 4, cq + k * 4);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    if (q == 0) tl.ys[k * kTS + slot] = y;
    float4* pk = reinterpret_cast<float4*>(prow + (k - lo) * kHB);
    pk[0] = make_float4(hh[0].x, hh[0].y, hh[1].x, hh[1].y);
    pk[1] = make_float4(hh[2].x, hh[2].y, hh[3].x, hh[3].y);
  }
  // adjoint, two steps at a time (hi-1, hi-2), ..., down to lo
  float* rrow = tl.red + lane * kRedS;
#pragma unroll 1
  for (int k = hi - 1; k >= lo; k -= 2) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int kk = k - s;
      float2 vals[8];
      if (kk >= lo) {
        const float4* pk = reinterpret_cast<const float4*>(prow + (kk - lo) * kHB);
        const float4 h0 = pk[0], h1 = pk[1];
        const float2 hk[4] = {make_float2(h0.x, h0.y), make_float2(h0.z, h0.w),
                              make_float2(h1.x, h1.y), make_float2(h1.z, h1.w)};
        float S1, S2, S3;
        const float2 dd = tl.sd[kk * kTS + slot];
        adjoint_step<PRECISE, KP>(lam, dA, al, ra, aback, hk, dd, tl.sg[kk * kTS + slot],
                                  live, bq + kk * 4, cq + kk * 4, vals, S1, S2, S3);
        // Euler: (Σ λ B, Σ A λ Ā h_{t-1}); ZOH: (Σ λ c B, x Σ λ Ā B + Σ A λ Ā h_{t-1})
        float T = kZoh ? fmaf(dd.y, S3, S2 * aback) : S2 * aback;
        S1 += __shfl_xor_sync(0xffffffffu, S1, 1);
        T += __shfl_xor_sync(0xffffffffu, T, 1);
        if (q == 0) tl.sS[kk * kTS + slot] = make_float2(S1, T);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) vals[j] = make_float2(0.f, 0.f);
      }
      float4* rv = reinterpret_cast<float4*>(rrow + s * 16);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        rv[j] = make_float4(vals[2 * j].x, vals[2 * j].y, vals[2 * j + 1].x, vals[2 * j + 1].y);
    }
    reduce_two_steps(tl, lane, k, k - 1 >= lo ? k - 1 : -1);
  }
}

// ---- channels-last tiles (the kernel's VEC = false forms): lane l moves step l/2 of 8 consecutive
// channels (or B/C states) with one 16-byte access (two for fp32), and a per-warp 16 x 16 scratch
// tile, reused for every operand, turns the warp's [16 steps][16 columns] tile into per-lane rows
// (column l/2, steps 8 (l & 1) .. + 7) and back.
constexpr int kClTile = 256;  // elements of the scratch tile, [column][step]

template <typename IO>
__device__ __forceinline__ void cl_load_piece(Row<IO, kHB>& w, const IO* base, long long stride,
                                              long long tr, bool ok) {
  if (!ok) {
    w.zero();
    return;
  }
  const uint4* p = reinterpret_cast<const uint4*>(base + tr * stride);
#pragma unroll
  for (int i = 0; i < Row<IO, kHB>::kWords / 4; ++i) {
    const uint4 v = __ldcs(p + i);
    w.w[4 * i] = v.x; w.w[4 * i + 1] = v.y; w.w[4 * i + 2] = v.z; w.w[4 * i + 3] = v.w;
  }
}

template <typename IO>
__device__ __forceinline__ void cl_transpose_in(Row<IO, kHB>& w, IO* T, int lane) {
  const int st = lane >> 1, h = lane & 1;
#pragma unroll
  for (int e = 0; e < kHB; ++e) {
    if (sizeof(IO) == 4) reinterpret_cast<uint32_t*>(T)[(8 * h + e) * 16 + st] = w.w[e];
    else reinterpret_cast<uint16_t*>(T)[(8 * h + e) * 16 + st] = (uint16_t)(w.w[e >> 1] >> (16 * (e & 1)));
  }
  __syncwarp();
  const uint4* p = reinterpret_cast<const uint4*>(T + st * 16 + 8 * h);
#pragma unroll
  for (int i = 0; i < Row<IO, kHB>::kWords / 4; ++i) {
    const uint4 v = p[i];
    w.w[4 * i] = v.x; w.w[4 * i + 1] = v.y; w.w[4 * i + 2] = v.z; w.w[4 * i + 3] = v.w;
  }
  __syncwarp();  // the tile is free for the next operand
}

// The lane's row (column lane/2, steps 8 (lane & 1) .. + 7) goes out as step `st` of its 8
// columns; ok: that step exists; tr: its time row.
template <typename IO>
__device__ __forceinline__ void cl_store_piece(IO* base, long long stride, const float (&o)[kHB],
                                               IO* T, int lane, long long tr, bool ok) {
  const int st = lane >> 1, h = lane & 1;
  __syncwarp();  // the scratch's previous reads are done
  {
    uint32_t rw[Row<IO, kHB>::kWords];
#pragma unroll
    for (int i = 0; i < Row<IO, kHB>::kWords; ++i)
      rw[i] = sizeof(IO) == 4 ? __float_as_uint(o[i]) : pack_bf16x2(o[2 * i], o[2 * i + 1]);
    uint4* p = reinterpret_cast<uint4*>(T + st * 16 + 8 * h);
#pragma unroll
    for (int i = 0; i < Row<IO, kHB>::kWords / 4; ++i)
      p[i] = make_uint4(rw[4 * i], rw[4 * i + 1], rw[4 * i + 2], rw[4 * i + 3]);
  }
  __syncwarp();
  uint32_t wv[Row<IO, kHB>::kWords];
#pragma unroll
  for (int e = 0; e < kHB; ++e) {
    uint32_t v;
    if (sizeof(IO) == 4) v = reinterpret_cast<const uint32_t*>(T)[(8 * h + e) * 16 + st];
    else v = reinterpret_cast<const uint16_t*>(T)[(8 * h + e) * 16 + st];
    if (sizeof(IO) == 4) wv[e] = v;
    else if (e & 1) wv[e >> 1] |= v << 16;
    else wv[e >> 1] = v;
  }
  if (!ok) return;
  uint4* p = reinterpret_cast<uint4*>(base + tr * stride);
#pragma unroll
  for (int i = 0; i < Row<IO, kHB>::kWords / 4; ++i)
    __stcs(p + i, make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]));
}

__device__ __forceinline__ bool al16p(const void* p) {
  return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0;
}

template <typename IO, bool VEC, int KP>
__global__ void __launch_bounds__(128) bwd_kernel(const BwdArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  extern __shared__ float4 smem4[];
  BwdTile* tiles = reinterpret_cast<BwdTile*>(smem4);
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  BwdTile& tl = tiles[wib];
  const int slot = lane >> 1, q = lane & 1;
  const int b = blockIdx.x / a.ngroups, grp = blockIdx.x % a.ngroups;
  const int d = (grp * a.wpb + wib) * kCW + slot;
  const bool act = d < a.dim;
  const int dd = act ? d : a.dim - 1;
  const float live = act ? 1.f : 0.f;  // idle lanes contribute nothing to the channel sums
  const long long ch = (long long)b * a.dim + dd;
  const int L = a.L, N = a.N;
  const int nblk = (L + kBlk - 1) / kBlk;
  const float ascale = kPrecise ? 1.f : kLog2e;
  const float aback = kPrecise ? 1.f : kLn2;  // al * aback == A

  // ZOH: ra = 1/A, with |A| < 1e-20 taken as -1e-20 (the A -> 0 limit, c = Δ)
  constexpr bool kZoh = KP == kKpZoh;
  float2 al[4], ra[4], lam[4], dA[4];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n0 = kHB * q + 2 * j, n1 = n0 + 1;
    float2 av = make_float2(n0 < N ? a.A[(long long)dd * N + n0] : 0.f,
                            n1 < N ? a.A[(long long)dd * N + n1] : 0.f);
    if (kZoh) av = make_float2(zoh_rate(av.x), zoh_rate(av.y));
    al[j] = mul2(av, f2(ascale));
    ra[j] = kZoh ? make_float2(1.f / av.x, 1.f / av.y) : f2(0.f);
    lam[j] = make_float2((a.dhL && n0 < N) ? a.dhL[ch * N + n0] : 0.f,
                         (a.dhL && n1 < N) ? a.dhL[ch * N + n1] : 0.f);
    dA[j] = make_float2(0.f, 0.f);
    amax = fmaxf(amax, fmaxf(fabsf(al[j].x), fabsf(al[j].y)));
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
  const float Dd = a.D ? a.D[dd] : 0.f;
  const float bias = a.dt_bias ? a.dt_bias[dd] : 0.f;
  float dD_acc = 0.f, dbias_acc = 0.f;

  // time rows at step 0 in scan order (mirrored for a reverse scan); the lane owns steps
  // [8 q, 8 q + 8) of each block
  const bool cl = a.channels_last != 0;  // [batch][L][dim] rows: element stride dim
  const long long row = cl ? (long long)b * L * a.dim + dd : ch * (long long)L;
  const long long ts_x = cl ? a.dim : 1, ts_bc = cl ? (long long)a.bc_groups * N : 1;
  const bool rev = a.reverse != 0;
  const IO* up = reinterpret_cast<const IO*>(a.u) + row;
  const IO* dp = reinterpret_cast<const IO*>(a.delta) + row;
  const IO* zp = a.z ? reinterpret_cast<const IO*>(a.z) + row : nullptr;
  const IO* gp = reinterpret_cast<const IO*>(a.dout) + row;
  const bool bc_live = slot < N;  // the lane also stages B/C row `slot`, steps [8 q, 8 q + 8)
  // the warp's B/C group (a warp wholly past dim shadows the last channel's)
  const int gbc = min((grp * a.wpb + wib) * kCW, a.dim - 1) / (a.dim / a.bc_groups);
  const long long bcrow = cl ? ((long long)b * L * a.bc_groups + gbc) * N + (bc_live ? slot : 0)
                             : (((long long)b * a.bc_groups + gbc) * N + (bc_live ? slot : 0)) * L;
  const IO* Bp = reinterpret_cast<const IO*>(a.B) + bcrow;
  const IO* Cp = reinterpret_cast<const IO*>(a.C) + bcrow;
  // channels-last tiles: the warp's 16 channels all exist, N == 16, every time row 16-byte aligned
  const bool clt = !VEC && cl && a.dim % kCW == 0 && (grp * a.wpb + wib + 1) * kCW <= a.dim &&
                   N == kNS && (a.dim * sizeof(IO)) % 16 == 0 &&
                   al16p(a.u) && al16p(a.delta) && al16p(a.z) && al16p(a.dout) && al16p(a.du) &&
                   al16p(a.ddelta) && al16p(a.dz) && al16p(a.B) && al16p(a.C);
  IO* xs = VEC ? nullptr
               : reinterpret_cast<IO*>(tiles + (blockDim.x >> 5)) + (size_t)wib * kClTile;
  const long long xrow = (long long)b * L * a.dim + (grp * a.wpb + wib) * kCW + 8 * (lane & 1);
  const long long xbc = ((long long)b * L * a.bc_groups + gbc) * N + 8 * (lane & 1);
  float* sBw = reinterpret_cast<float*>(tl.sB);
  float* sCw = reinterpret_cast<float*>(tl.sC);

  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * kBlk;
    const int nvalid = min(kBlk, L - t0);
    const int nown = max(0, min(kHB, nvalid - kHB * q));
    Row<IO, kHB> ru, rd, rz, rg, rb, rc;
    const int tq = t0 + kHB * q;
    if (VEC && nown == kHB) {
      load_steps<IO, kHB, true>(ru, up, L, tq, kHB, rev);
      load_steps<IO, kHB, true>(rd, dp, L, tq, kHB, rev);
      load_steps<IO, kHB, true>(rg, gp, L, tq, kHB, rev);
      if (zp) load_steps<IO, kHB, true>(rz, zp, L, tq, kHB, rev);
    } else if (clt) {
      const int st = lane >> 1;
      const bool ok = st < nvalid;
      const long long tr = rev ? (long long)L - 1 - (t0 + st) : (long long)(t0 + st);
      cl_load_piece<IO>(ru, reinterpret_cast<const IO*>(a.u) + xrow, a.dim, tr, ok);
      cl_load_piece<IO>(rd, reinterpret_cast<const IO*>(a.delta) + xrow, a.dim, tr, ok);
      cl_load_piece<IO>(rg, reinterpret_cast<const IO*>(a.dout) + xrow, a.dim, tr, ok);
      if (zp) cl_load_piece<IO>(rz, reinterpret_cast<const IO*>(a.z) + xrow, a.dim, tr, ok);
      cl_load_piece<IO>(rb, reinterpret_cast<const IO*>(a.B) + xbc, ts_bc, tr, ok);
      cl_load_piece<IO>(rc, reinterpret_cast<const IO*>(a.C) + xbc, ts_bc, tr, ok);
      __syncwarp();  // the scratch's previous reads are done
      cl_transpose_in<IO>(ru, xs, lane);
      cl_transpose_in<IO>(rd, xs, lane);
      cl_transpose_in<IO>(rg, xs, lane);
      if (zp) cl_transpose_in<IO>(rz, xs, lane);
      cl_transpose_in<IO>(rb, xs, lane);
      cl_transpose_in<IO>(rc, xs, lane);
    } else {
      load_steps<IO, kHB, false>(ru, up, L, tq, nown, rev, ts_x);
      load_steps<IO, kHB, false>(rd, dp, L, tq, nown, rev, ts_x);
      load_steps<IO, kHB, false>(rg, gp, L, tq, nown, rev, ts_x);
      if (zp) load_steps<IO, kHB, false>(rz, zp, L, tq, nown, rev, ts_x);
    }
    if (clt) {
      // B/C rows came with the tile
    } else if (!bc_live) {
      rb.zero();
      rc.zero();
    } else if (VEC && nown == kHB) {
      load_steps<IO, kHB, true>(rb, Bp, L, tq, kHB, rev);
      load_steps<IO, kHB, true>(rc, Cp, L, tq, kHB, rev);
    } else {
      load_steps<IO, kHB, false>(rb, Bp, L, tq, nown, rev, ts_bc);
      load_steps<IO, kHB, false>(rc, Cp, L, tq, nown, rev, ts_bc);
    }
    // the state entering the block
    float2 hstart[4];
    const float* cp = a.ckpt + (ch * nblk + blk) * N;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n0 = kHB * q + 2 * j;
      hstart[j] = make_float2(n0 < N ? cp[n0] : 0.f, n0 + 1 < N ? cp[n0 + 1] : 0.f);
    }

    __syncwarp();  // the previous block's tables are no longer read
#pragma unroll
    for (int j = 0; j < kHB; ++j) {
      sBw[(kHB * q + j) * kNS + slot] = rb.get(j);
      sCw[(kHB * q + j) * kNS + slot] = rc.get(j);
    }
    // per-step scalars of this lane's 8 steps
    float sv[kHB], dzf[kHB];
    float dabs = 0.f;
#pragma unroll
    for (int j = 0; j < kHB; j += 2) {
      const float2 v = add2(make_float2(rd.get(j), rd.get(j + 1)), f2(bias));
      float2 dl = v, sp = make_float2(1.f, 1.f);
      if (a.softplus) {
        if (kPrecise) {
          dl = make_float2(softplus_precise(v.x), softplus_precise(v.y));
          sp = make_float2(sigmoid_precise(v.x), sigmoid_precise(v.y));
        } else {
          dl = softplus_fast_x2(v);
          sp = sigmoid_fast_x2(v);
        }
      }
      // (Δ, Δx), or (Δ, x) with the ZOH term (its coefficient is per state)
      const float2 xv = make_float2(ru.get(j), ru.get(j + 1));
      const float2 dx = kZoh ? xv : mul2(dl, xv);
      const float2 go = make_float2(rg.get(j), rg.get(j + 1));
      float2 g = go, zf = make_float2(0.f, 0.f);
      if (zp) {
        const float2 z2 = make_float2(rz.get(j), rz.get(j + 1));
        const float2 sg = kPrecise ? make_float2(sigmoid_precise(z2.x), sigmoid_precise(z2.y))
                                   : sigmoid_fast_x2(z2);
        g = mul2(go, mul2(z2, sg));
        // silu'(z) = σ(z) (1 + z (1 - σ(z)))
        zf = mul2(mul2(go, sg), fma2(z2, add2(f2(1.f), mul2(sg, f2(-1.f))), f2(1.f)));
      }
      tl.sd[(kHB * q + j) * kTS + slot] = make_float2(dl.x, dx.x);
      tl.sd[(kHB * q + j + 1) * kTS + slot] = make_float2(dl.y, dx.y);
      tl.sg[(kHB * q + j) * kTS + slot] = g.x;
      tl.sg[(kHB * q + j + 1) * kTS + slot] = g.y;
      sv[j] = sp.x; sv[j + 1] = sp.y;
      dzf[j] = zf.x; dzf[j + 1] = zf.y;
      dabs = fmaxf(dabs, fmaxf(fabsf(dl.x), fabsf(dl.y)));
      if (dl.x != dl.x || dl.y != dl.y) dabs = __int_as_float(0x7f800000);
    }
    __syncwarp();
    const bool safe = !__any_sync(0xffffffffu, !(amax * dabs <= 126.f));
    for (int half = 1; half >= 0; --half) {
      const int lo = kHB * half, hi = min(nvalid, lo + kHB);
      if (lo >= hi) continue;
      // blocks that fail the range vote: MUFU exponentials, or the clamped ZOH form
      constexpr int KS = kZoh ? kKpZohClamped : 4;
      if (!safe || (kPrecise && !kZoh))
        half_pass<kPrecise, KS>(tl, hstart, lam, dA, al, ra, aback, live, lane, slot, q, lo, hi);
      else
        half_pass<kPrecise, KP>(tl, hstart, lam, dA, al, ra, aback, live, lane, slot, q, lo, hi);
    }
    __syncwarp();

    // outputs of this lane's 8 steps
    float odu[kHB], odd[kHB], odz[kHB];
#pragma unroll
    for (int j = 0; j < kHB; ++j) {
      const int k = kHB * q + j;
      const float2 S = tl.sS[k * kTS + slot];
      const float2 dlx = tl.sd[k * kTS + slot];
      const float g = tl.sg[k * kTS + slot];
      const float x = ru.get(j);
      odz[j] = (tl.ys[k * kTS + slot] + Dd * x) * dzf[j];
      odu[j] = (kZoh ? S.x : dlx.x * S.x) + g * Dd;
      odd[j] = (kZoh ? S.y : x * S.x + S.y) * sv[j];
      if (j < nown) {
        dD_acc += g * x;
        dbias_acc += odd[j];
      }
    }
    if (clt) {  // every lane takes part: the tiles go out through the scratch
      const int st = lane >> 1;
      const bool ok = st < nvalid;
      const long long tr = rev ? (long long)L - 1 - (t0 + st) : (long long)(t0 + st);
      IO* T = xs;
      if (a.du) cl_store_piece<IO>(reinterpret_cast<IO*>(a.du) + xrow, a.dim, odu, T, lane, tr, ok);
      if (a.ddelta) cl_store_piece<IO>(reinterpret_cast<IO*>(a.ddelta) + xrow, a.dim, odd, T, lane, tr, ok);
      if (a.dz && zp) cl_store_piece<IO>(reinterpret_cast<IO*>(a.dz) + xrow, a.dim, odz, T, lane, tr, ok);
    } else if (act && nown > 0) {
      const auto put = [&](void* base, const float (&v)[kHB]) {
        IO* o = reinterpret_cast<IO*>(base) + row;
        if (VEC && nown == kHB) store_steps<IO, kHB, true>(o, v, L, tq, kHB, rev);
        else store_steps<IO, kHB, false>(o, v, L, tq, nown, rev, ts_x);
      };
      if (a.du) put(a.du, odu);
      if (a.ddelta) put(a.ddelta, odd);
      if (a.dz && zp) put(a.dz, odz);
    }

    // CTA partial of dB, dC for this block: add the warps' sums, one value per (step, n, which)
    __syncthreads();
    for (int p = threadIdx.x; p < kBlk * 32; p += blockDim.x) {
      const int k = p & (kBlk - 1), e = p >> 4;    // e = half * 16 + (v < 8 ? dB : dC) * 8 + n
      if (k < nvalid) {
        float sum = 0.f;
        for (int w = 0; w < a.wpb; ++w) sum += tiles[w].wres[k * 32 + e];
        const int n = 8 * (e >> 4) + (e & 7), which = (e >> 3) & 1;
        const long long prow = ((long long)(grp * a.batch + b) * 2 + which) * kNS + n;
        a.part_bc[prow * L + t0 + k] = sum;
      }
    }
    __syncthreads();
  }

  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
  if (!act) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n0 = kHB * q + 2 * j;
    if (a.dh0) {
      if (n0 < N) a.dh0[ch * N + n0] = lam[j].x;
      if (n0 + 1 < N) a.dh0[ch * N + n0 + 1] = lam[j].y;
    }
    float* pa = a.part_adt + ch * (kNS + 2);
    pa[n0] = dA[j].x;  // Σ λ Δ Ā h_{t-1}: no A factor, so no log2(e) rescale
    pa[n0 + 1] = dA[j].y;
  }
  if (q == 0) {
    float* pa = a.part_adt + ch * (kNS + 2);
    pa[kNS] = dD_acc;
    pa[kNS + 1] = dbias_acc;
  }
}

// dB, dC: sum the partials of the CTAs of one B/C group in a fixed order; dA, dD, ddt_bias: sum
// over batch.
template <typename IO>
__global__ void bwd_finish_bc(const BwdArgs a, IO* dB, IO* dC) {
  const long long total = (long long)a.batch * a.bc_groups * 2 * a.N * a.L;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int t = (int)(i % a.L);
  long long r = i / a.L;
  const int n = (int)(r % a.N);
  r /= a.N;
  const int which = (int)(r % 2);
  r /= 2;
  const int gb = (int)(r % a.bc_groups);
  const int b = (int)(r / a.bc_groups);
  const int per = a.ngroups / a.bc_groups;  // CTAs per B/C group (whole groups of channels)
  float s = 0.f;
  for (int g = gb * per; g < (gb + 1) * per; ++g)
    s += a.part_bc[(((long long)(g * a.batch + b) * 2 + which) * kNS + n) * a.L + t];
  IO* dst = which == 0 ? dB : dC;
  if (!dst) return;
  const long long tm = a.reverse ? a.L - 1 - t : t;  // time index of scan step t
  const long long o = a.channels_last ? (((long long)b * a.L + tm) * a.bc_groups + gb) * a.N + n
                                      : (((long long)b * a.bc_groups + gb) * a.N + n) * a.L + tm;
  if (sizeof(IO) == 2) reinterpret_cast<uint16_t*>(dst)[o] = f32_to_bf16(s);
  else reinterpret_cast<float*>(dst)[o] = s;
}

__global__ void bwd_finish_adt(const BwdArgs a, float* dA, float* dD, float* ddt_bias) {
  const long long total = (long long)a.dim * (kNS + 2);
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int d = (int)(i / (kNS + 2)), j = (int)(i % (kNS + 2));
  if (j < kNS && j >= a.N) return;
  float s = 0.f;
  const int nsplit = a.nsplit > 1 ? a.nsplit : 1;  // chunks of a time-split backward
  for (int c = 0; c < nsplit; ++c)
    for (int b = 0; b < a.batch; ++b)
      s += a.part_adt[(((long long)c * a.batch + b) * a.dim + d) * (kNS + 2) + j];
  if (j < kNS) { if (dA) dA[(long long)d * a.N + j] = s; }
  else if (j == kNS) { if (dD) dD[d] = s; }
  else if (ddt_bias) ddt_bias[d] = s;
}

template <typename IO, bool VEC>
cudaError_t launch_bwd_io(const BwdArgs& a, cudaStream_t s) {
  const dim3 grid((unsigned)(a.batch * a.ngroups)), block(32 * a.wpb);
  // the channels-last scratch tile exists only in channels-last launches (the kernel's tile test
  // requires the layout flag)
  const size_t smem =
      (sizeof(BwdTile) + (!VEC && a.channels_last ? kClTile * sizeof(IO) : 0)) * a.wpb;
  auto k = bwd_kernel<IO, VEC, 2>;
  if (a.zoh) {
    k = bwd_kernel<IO, VEC, kKpZoh>;  // ZOH coefficient on the FMA pipe
  } else if constexpr (!std::is_same<IO, float>::value) {
    if (a.kmufu == 3) k = bwd_kernel<IO, VEC, 3>;
    else if (a.kmufu == 4) k = bwd_kernel<IO, VEC, 4>;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, block, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, int io, bool vec, cudaStream_t s) {
  if (io == 1) return vec ? launch_bwd_io<uint16_t, true>(a, s) : launch_bwd_io<uint16_t, false>(a, s);
  return vec ? launch_bwd_io<float, true>(a, s) : launch_bwd_io<float, false>(a, s);
}

cudaError_t launch_bwd_finish(const BwdArgs& a, int io, void* dB, void* dC, float* dA, float* dD,
                              float* ddt_bias, cudaStream_t s) {
  const int tpb = 256;
  const long long nbc = (long long)a.batch * a.bc_groups * 2 * a.N * a.L;
  if (io == 1)
    bwd_finish_bc<uint16_t><<<(unsigned)((nbc + tpb - 1) / tpb), tpb, 0, s>>>(
        a, reinterpret_cast<uint16_t*>(dB), reinterpret_cast<uint16_t*>(dC));
  else
    bwd_finish_bc<float><<<(unsigned)((nbc + tpb - 1) / tpb), tpb, 0, s>>>(
        a, reinterpret_cast<float*>(dB), reinterpret_cast<float*>(dC));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_bwd_finish_adt(a, dA, dD, ddt_bias, s);
}

cudaError_t launch_bwd_finish_adt(const BwdArgs& a, float* dA, float* dD, float* ddt_bias,
                                  cudaStream_t s) {
  const int tpb = 256;
  const long long nadt = (long long)a.dim * (kNS + 2);
  bwd_finish_adt<<<(unsigned)((nadt + tpb - 1) / tpb), tpb, 0, s>>>(a, dA, dD, ddt_bias);
  return cudaGetLastError();
}

}  // namespace ssm
