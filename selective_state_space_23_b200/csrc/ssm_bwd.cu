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
// with Ā_t h_{t-1} = h_t - Δ_t B_t x_t, so the reverse sweep needs only h_t.
//
// Mapping: one lane per channel, 16 states in registers, time walked backwards in 16-step
// blocks.  For each block the lane reloads the state entering the block (a checkpoint written
// by the forward pass or by a checkpoint-only forward pass), replays the 16 steps forward and
// parks h_t in shared memory, then runs the adjoint recurrence backwards over the block.  dB
// and dC are sums over the channel axis: each warp transposes its 32 lanes' per-step values
// through shared memory and sums columns; the CTA sums its warps and writes one partial per
// (CTA, b, n, t); a finishing kernel adds the partials in a fixed order (deterministic).
#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace {

constexpr int kHsStride = kBlk * kNS + 4;  // per-lane row of parked states (+4: no bank conflicts)
constexpr int kRedStride = 36;             // per-lane row of the transpose buffer

struct WarpSmem {
  float sB[kBlk * kNS];
  float sC[kBlk * kNS];
  float hs[32 * kHsStride];
  float red[32 * kRedStride];
  float wsum[kBlk * 32];
};

__device__ __forceinline__ uint32_t wd(const uint4& q, int j) {
  return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w;
}
template <typename IO> struct Row { uint4 v[sizeof(IO) * kBlk / 16]; };
template <typename IO> __device__ __forceinline__ float el(const Row<IO>& r, int k);
template <> __device__ __forceinline__ float el<float>(const Row<float>& r, int k) {
  return __uint_as_float(wd(r.v[k >> 2], k & 3));
}
template <> __device__ __forceinline__ float el<uint16_t>(const Row<uint16_t>& r, int k) {
  const uint32_t w = wd(r.v[k >> 3], (k >> 1) & 3);
  return (k & 1) ? bf16_hi(w) : bf16_lo(w);
}

template <typename IO, bool VEC>
__device__ __forceinline__ void load_row(Row<IO>& r, const IO* p, int nvalid) {
  if (VEC && nvalid == kBlk) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < (int)(sizeof(r.v) / 16); ++i) r.v[i] = __ldcs(q + i);
    return;
  }
  uint32_t w[sizeof(r.v) / 4];
#pragma unroll
  for (int i = 0; i < (int)(sizeof(r.v) / 4); ++i) w[i] = 0u;
  if (sizeof(IO) == 4) {
    const uint32_t* s = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int e = 0; e < kBlk; ++e)
      if (e < nvalid) w[e] = s[e];
  } else {
    const unsigned short* s = reinterpret_cast<const unsigned short*>(p);
#pragma unroll
    for (int e = 0; e < kBlk; ++e)
      if (e < nvalid) w[e >> 1] |= ((uint32_t)s[e]) << (16 * (e & 1));
  }
#pragma unroll
  for (int i = 0; i < (int)(sizeof(r.v) / 16); ++i)
    r.v[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

template <typename IO, bool VEC>
__device__ __forceinline__ void store_row(IO* p, const float (&o)[kBlk], int nvalid) {
  if (sizeof(IO) == 2) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
    if (VEC && nvalid == kBlk) {
      uint4* q = reinterpret_cast<uint4*>(p);
      __stcs(q, make_uint4(w[0], w[1], w[2], w[3]));
      __stcs(q + 1, make_uint4(w[4], w[5], w[6], w[7]));
    } else {
      unsigned short* s = reinterpret_cast<unsigned short*>(p);
#pragma unroll
      for (int e = 0; e < kBlk; ++e)
        if (e < nvalid) s[e] = (unsigned short)(w[e >> 1] >> (16 * (e & 1)));
    }
  } else {
    float* s = reinterpret_cast<float*>(p);
    if (VEC && nvalid == kBlk) {
      float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
      for (int i = 0; i < 4; ++i) __stcs(q + i, make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
    } else {
#pragma unroll
      for (int e = 0; e < kBlk; ++e)
        if (e < nvalid) s[e] = o[e];
    }
  }
}

template <typename IO, bool VEC>
__global__ void __launch_bounds__(128, 1) bwd_kernel(const BwdArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  extern __shared__ float4 smem4[];
  WarpSmem* all = reinterpret_cast<WarpSmem*>(smem4);
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  WarpSmem& sm = all[wib];
  const int b = blockIdx.x / a.ngroups, g = blockIdx.x % a.ngroups;
  const int d = (g * a.wpb + wib) * 32 + lane;
  const bool act = d < a.dim;
  const int dd = act ? d : a.dim - 1;
  const float live = act ? 1.f : 0.f;  // idle lanes contribute nothing to the channel sums
  const long long ch = (long long)b * a.dim + dd;
  const int L = a.L, N = a.N;
  const int nblk = (L + kBlk - 1) / kBlk;

  const float ascale = kPrecise ? 1.f : kLog2e;
  const float aback = kPrecise ? 1.f : kLn2;  // al * aback == A
  float2 al[8], lam[8], dA[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int n0 = 2 * j, n1 = 2 * j + 1;
    al[j] = make_float2(n0 < N ? a.A[(long long)dd * N + n0] * ascale : 0.f,
                        n1 < N ? a.A[(long long)dd * N + n1] * ascale : 0.f);
    lam[j] = make_float2((a.dhL && n0 < N) ? a.dhL[ch * N + n0] : 0.f,
                         (a.dhL && n1 < N) ? a.dhL[ch * N + n1] : 0.f);
    dA[j] = make_float2(0.f, 0.f);
  }
  const float Dd = a.D ? a.D[dd] : 0.f;
  const float bias = a.dt_bias ? a.dt_bias[dd] : 0.f;
  float dD_acc = 0.f, dbias_acc = 0.f;

  const IO* up = reinterpret_cast<const IO*>(a.u) + ch * (long long)L;
  const IO* dp = reinterpret_cast<const IO*>(a.delta) + ch * (long long)L;
  const IO* zp = a.z ? reinterpret_cast<const IO*>(a.z) + ch * (long long)L : nullptr;
  const IO* gp = reinterpret_cast<const IO*>(a.dout) + ch * (long long)L;
  const int bc_n = lane >> 1, bc_half = lane & 1;
  const bool bc_live = bc_n < N;
  const IO* Bp = reinterpret_cast<const IO*>(a.B) + ((long long)b * N + (bc_live ? bc_n : 0)) * L;
  const IO* Cp = reinterpret_cast<const IO*>(a.C) + ((long long)b * N + (bc_live ? bc_n : 0)) * L;
  float* hrow = sm.hs + lane * kHsStride;
  float* rrow = sm.red + lane * kRedStride;

  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * kBlk;
    const int nvalid = min(kBlk, L - t0);
    Row<IO> ru, rd, rz, rg;
    load_row<IO, VEC>(ru, up + t0, nvalid);
    load_row<IO, VEC>(rd, dp + t0, nvalid);
    load_row<IO, VEC>(rg, gp + t0, nvalid);
    if (zp) load_row<IO, VEC>(rz, zp + t0, nvalid);

    // B, C rows of this block -> shared memory as f32 [step][state]
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t = t0 + 8 * bc_half + j;
      const bool ok = bc_live && t < L;
      float bv = 0.f, cv = 0.f;
      if (ok) {
        if (sizeof(IO) == 2) {
          bv = bf16_to_f32(reinterpret_cast<const uint16_t*>(Bp)[t]);
          cv = bf16_to_f32(reinterpret_cast<const uint16_t*>(Cp)[t]);
        } else {
          bv = reinterpret_cast<const float*>(Bp)[t];
          cv = reinterpret_cast<const float*>(Cp)[t];
        }
      }
      sm.sB[(8 * bc_half + j) * kNS + bc_n] = bv;
      sm.sC[(8 * bc_half + j) * kNS + bc_n] = cv;
    }
    __syncwarp();

    // state entering the block
    float2 hh[8];
    const float* cp = a.ckpt + (ch * nblk + blk) * N;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      hh[j] = make_float2(2 * j < N ? cp[2 * j] : 0.f, 2 * j + 1 < N ? cp[2 * j + 1] : 0.f);

    // per-step scalars
    float dl[kBlk], dxu[kBlk], gg[kBlk];
#pragma unroll
    for (int k = 0; k < kBlk; ++k) {
      const float v = el<IO>(rd, k) + bias;
      dl[k] = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
      dxu[k] = dl[k] * el<IO>(ru, k);
      float gk = el<IO>(rg, k);
      if (zp) {
        const float zk = el<IO>(rz, k);
        gk *= zk * (kPrecise ? sigmoid_precise(zk) : sigmoid_fast(zk));
      }
      gg[k] = gk;
    }

    // replay the block forward, parking h_t; y_t for dz
    float odz[kBlk];
#pragma unroll
    for (int k = 0; k < kBlk; ++k) {
      if (k < nvalid) {
        const float2 d2 = f2(dl[k]), du2 = f2(dxu[k]);
        float2 y2 = make_float2(Dd * el<IO>(ru, k), 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float2 av;
          if (kPrecise) {
            av = make_float2(expf(dl[k] * al[j].x), expf(dl[k] * al[j].y));
          } else {
            const float2 x = mul2(d2, al[j]);
            av = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
          }
          const float2 bp = *reinterpret_cast<const float2*>(sm.sB + k * kNS + 2 * j);
          const float2 cq = *reinterpret_cast<const float2*>(sm.sC + k * kNS + 2 * j);
          hh[j] = fma2(av, hh[j], mul2(du2, bp));
          y2 = fma2(cq, hh[j], y2);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<float4*>(hrow + k * kNS)[q] =
              make_float4(hh[2 * q].x, hh[2 * q].y, hh[2 * q + 1].x, hh[2 * q + 1].y);
        float dzk = 0.f;
        if (zp) {
          const float zk = el<IO>(rz, k);
          const float sg = kPrecise ? sigmoid_precise(zk) : sigmoid_fast(zk);
          dzk = el<IO>(rg, k) * (y2.x + y2.y) * sg * (1.f + zk * (1.f - sg));
        }
        odz[k] = dzk;
      } else {
        odz[k] = 0.f;
      }
    }
    if (a.dz && zp && act) store_row<IO, VEC>(reinterpret_cast<IO*>(a.dz) + ch * (long long)L + t0, odz, nvalid);

    // adjoint sweep, backwards over the block
#pragma unroll
    for (int k = kBlk - 1; k >= 0; --k) {
      if (k < nvalid) {
        float2 hk[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v = reinterpret_cast<const float4*>(hrow + k * kNS)[q];
          hk[2 * q] = make_float2(v.x, v.y);
          hk[2 * q + 1] = make_float2(v.z, v.w);
        }
        const float2 g2 = f2(gg[k]), du2 = f2(dxu[k]), d2 = f2(dl[k]);
        const float2 gl = f2(gg[k] * live), dul = f2(dxu[k] * live);
        float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
        float2 vB[8], vC[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 bp = *reinterpret_cast<const float2*>(sm.sB + k * kNS + 2 * j);
          const float2 cq = *reinterpret_cast<const float2*>(sm.sC + k * kNS + 2 * j);
          lam[j] = fma2(g2, cq, lam[j]);                       // λ_t complete
          vB[j] = mul2(lam[j], dul);                           // dB contribution
          vC[j] = mul2(gl, hk[j]);                             // dC contribution
          const float2 qv = fma2(du2, make_float2(-bp.x, -bp.y), hk[j]);  // Ā_t h_{t-1}
          const float2 lq = mul2(lam[j], qv);
          s1 = fma2(lam[j], bp, s1);
          s2 = fma2(al[j], lq, s2);
          dA[j] = fma2(d2, lq, dA[j]);
          float2 av;
          if (kPrecise) {
            av = make_float2(expf(dl[k] * al[j].x), expf(dl[k] * al[j].y));
          } else {
            const float2 x = mul2(d2, al[j]);
            av = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
          }
          lam[j] = mul2(lam[j], av);                           // Ā_t λ_t, for step t-1
        }
        const float S1 = s1.x + s1.y, S2 = (s2.x + s2.y) * aback;
        const float xk = el<IO>(ru, k);
        const float duk = dl[k] * S1 + gg[k] * Dd;
        const float ddt = xk * S1 + S2;
        float ddl = ddt;
        if (a.softplus) {
          const float v = el<IO>(rd, k) + bias;
          ddl = ddt * (kPrecise ? sigmoid_precise(v) : sigmoid_fast(v));
        }
        dD_acc += gg[k] * xk;
        dbias_acc += ddl;
        // park du, ddelta in the (already consumed) state slot of step k
        hrow[k * kNS + 0] = duk;
        hrow[k * kNS + 1] = ddl;

        // channel sums of dB, dC for this step: transpose through shared memory
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          reinterpret_cast<float4*>(rrow)[q] = make_float4(vB[2 * q].x, vB[2 * q].y, vB[2 * q + 1].x, vB[2 * q + 1].y);
          reinterpret_cast<float4*>(rrow)[4 + q] = make_float4(vC[2 * q].x, vC[2 * q].y, vC[2 * q + 1].x, vC[2 * q + 1].y);
        }
        __syncwarp();
        float colsum = 0.f;
#pragma unroll
        for (int l = 0; l < 32; ++l) colsum += sm.red[l * kRedStride + lane];
        sm.wsum[k * 32 + lane] = colsum;
        __syncwarp();
      } else {
        sm.wsum[k * 32 + lane] = 0.f;
      }
    }
    float odu[kBlk], odd[kBlk];
#pragma unroll
    for (int k = 0; k < kBlk; ++k) {
      odu[k] = hrow[k * kNS + 0];
      odd[k] = hrow[k * kNS + 1];
    }
    if (act) {
      if (a.du) store_row<IO, VEC>(reinterpret_cast<IO*>(a.du) + ch * (long long)L + t0, odu, nvalid);
      if (a.ddelta) store_row<IO, VEC>(reinterpret_cast<IO*>(a.ddelta) + ch * (long long)L + t0, odd, nvalid);
    }

    // CTA partial of dB, dC for this block: sum the warps, one value per (n, which, step)
    __syncthreads();
    for (int p = threadIdx.x; p < kBlk * 32; p += blockDim.x) {
      const int k = p & (kBlk - 1), j = p >> 4;   // j < 16: dB state j; j >= 16: dC state j-16
      if (k < nvalid) {
        float s = 0.f;
        for (int w = 0; w < a.wpb; ++w) s += all[w].wsum[k * 32 + j];
        const long long row = ((long long)(g * a.batch + b) * 2 + (j >> 4)) * kNS + (j & 15);
        a.part_bc[row * L + t0 + k] = s;
      }
    }
    __syncthreads();
  }

  if (!act) return;
  if (a.dh0)
#pragma unroll
    for (int n = 0; n < kNS; ++n)
      if (n < N) a.dh0[ch * N + n] = (n & 1) ? lam[n >> 1].y : lam[n >> 1].x;
  float* pa = a.part_adt + ch * (kNS + 2);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    pa[2 * j] = dA[j].x;        // Σ λ Δ Ā h_{t-1}: no A factor, so no log2(e) rescale
    pa[2 * j + 1] = dA[j].y;
  }
  pa[kNS] = dD_acc;
  pa[kNS + 1] = dbias_acc;
}

// dB, dC: sum the CTA partials over groups in a fixed order; dA, dD, ddt_bias: sum over batch.
template <typename IO>
__global__ void bwd_finish_bc(const BwdArgs a, IO* dB, IO* dC) {
  const long long total = (long long)a.batch * 2 * a.N * a.L;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int t = (int)(i % a.L);
  long long r = i / a.L;
  const int n = (int)(r % a.N);
  r /= a.N;
  const int which = (int)(r % 2);
  const int b = (int)(r / 2);
  float s = 0.f;
  for (int g = 0; g < a.ngroups; ++g)
    s += a.part_bc[(((long long)(g * a.batch + b) * 2 + which) * kNS + n) * a.L + t];
  IO* dst = which == 0 ? dB : dC;
  if (!dst) return;
  const long long o = ((long long)b * a.N + n) * a.L + t;
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
  for (int b = 0; b < a.batch; ++b) s += a.part_adt[((long long)b * a.dim + d) * (kNS + 2) + j];
  if (j < kNS) { if (dA) dA[(long long)d * a.N + j] = s; }
  else if (j == kNS) { if (dD) dD[d] = s; }
  else if (ddt_bias) ddt_bias[d] = s;
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, int io, bool vec, cudaStream_t s) {
  dim3 grid((unsigned)(a.batch * a.ngroups));
  dim3 block(32 * a.wpb);
  const size_t smem = sizeof(WarpSmem) * a.wpb;
  if (io == 1) {
    auto k = vec ? bwd_kernel<uint16_t, true> : bwd_kernel<uint16_t, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, block, smem, s>>>(a);
  } else {
    auto k = vec ? bwd_kernel<float, true> : bwd_kernel<float, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, block, smem, s>>>(a);
  }
  return cudaGetLastError();
}

size_t bwd_smem_per_warp() { return sizeof(WarpSmem); }

cudaError_t launch_bwd_finish(const BwdArgs& a, int io, void* dB, void* dC, float* dA, float* dD,
                              float* ddt_bias, cudaStream_t s) {
  const int tpb = 256;
  const long long nbc = (long long)a.batch * 2 * a.N * a.L;
  if (io == 1)
    bwd_finish_bc<uint16_t><<<(unsigned)((nbc + tpb - 1) / tpb), tpb, 0, s>>>(
        a, reinterpret_cast<uint16_t*>(dB), reinterpret_cast<uint16_t*>(dC));
  else
    bwd_finish_bc<float><<<(unsigned)((nbc + tpb - 1) / tpb), tpb, 0, s>>>(
        a, reinterpret_cast<float*>(dB), reinterpret_cast<float*>(dC));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long nadt = (long long)a.dim * (kNS + 2);
  bwd_finish_adt<<<(unsigned)((nadt + tpb - 1) / tpb), tpb, 0, s>>>(a, dA, dD, ddt_bias);
  return cudaGetLastError();
}

}  // namespace ssm
