// Selective scan with B, C per channel (bc_groups == dim), sm_100a: forward and backward.
//
// The selection mechanism makes B_t, C_t functions of the input ("Mamba: ..." summary page,
// "Seçim Mekanizması (S6)"); computed per channel they are [batch][dim][N][L] tensors, so every
// (channel, step) reads 2 N values of its own instead of sharing one B_t, C_t per batch row.
// The recurrence and readout are those of the shared case:
//   h_t,n = exp(Δ_t A_dn) h_{t-1},n + Δ_t B_{c,t,n} x_t,  y_t = Σ_n C_{c,t,n} h_t,n + D x_t,
//   out_t = y_t silu(z_t),
// and the backward is the chain rule through it with per-channel dB, dC (no sum over d):
//   dB_{c,t} = λ_t Δ_t x_t,  dC_{c,t} = g_t h_t,  the other gradients as in ssm_bwd.cu.
//
// B200 mapping: the work per (channel, step) is dominated by reading its own B and C rows, so
// one LANE owns one STATE: 16 lanes per channel, two channels per warp.  Each lane streams its
// state's B and C rows with 16-byte loads (8 bf16 steps each) and keeps its single state in a
// register.  Per-step scalars (Δ, Δx, the gate) are computed by one lane per step and broadcast
// to the channel's 16 lanes with shuffles; the readout Σ_n C h is a shuffle reduction over the
// 16 lanes that leaves the total of step j in lanes 2 j and 2 j + 1.  The backward keeps the
// 16 states and Ā of a 16-step block in registers (one state per lane), so each exponential is
// computed once, and writes dB, dC rows directly.
#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"
#include "ssm_rows.cuh"

namespace ssm {
namespace {

template <typename IO>
__device__ __forceinline__ float ld1(const void* p, long long i) {
  if constexpr (sizeof(IO) == 2) return bf16_to_f32(reinterpret_cast<const uint16_t*>(p)[i]);
  else return reinterpret_cast<const float*>(p)[i];
}
template <typename IO>
__device__ __forceinline__ void st1(void* p, long long i, float v) {
  if constexpr (sizeof(IO) == 2) reinterpret_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

// E values of one row at t0 (E = 8 or 16): 16-byte pieces when VEC (row pieces aligned and
// all E valid), else element loads; steps at or beyond nv read as zero.
template <typename IO, int E, bool VEC>
__device__ __forceinline__ void load_seg(Row<IO, E>& r, const IO* p, int nv) {
  if (VEC && nv == E) load_row<IO, E, true>(r, p, E);
  else load_row<IO, E, false>(r, p, nv);
}

// Sum over the channel's 16 lanes of v[k] for k < 8 (lane bits 0..3 = state): afterwards lanes
// 2 j and 2 j + 1 of the group hold the total of v[j].
__device__ __forceinline__ float reduce8(float (&v)[8], int n) {
  const bool b3 = (n >> 3) & 1, b2 = (n >> 2) & 1, b1 = (n >> 1) & 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b3 ? v[i + 4] : v[i], send = b3 ? v[i] : v[i + 4];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b2 ? v[i + 2] : v[i], send = b2 ? v[i] : v[i + 2];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const float keep = b1 ? v[1] : v[0], send = b1 ? v[0] : v[1];
  float t = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  return t + __shfl_xor_sync(0xffffffffu, t, 1);
}

// Sum over the channel's 16 lanes of v[k] for k < 16: afterwards lane n of the group holds the
// total of v[n].
__device__ __forceinline__ float reduce16(float (&v)[16], int n) {
  const bool b3 = (n >> 3) & 1, b2 = (n >> 2) & 1, b1 = (n >> 1) & 1, b0 = n & 1;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float keep = b3 ? v[i + 8] : v[i], send = b3 ? v[i] : v[i + 8];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b2 ? v[i + 4] : v[i], send = b2 ? v[i] : v[i + 4];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b1 ? v[i + 2] : v[i], send = b1 ? v[i] : v[i + 2];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  const float keep = b0 ? v[1] : v[0], send = b0 ? v[0] : v[1];
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

// Forward.  MODE kFwdOut: gated output (+ optional checkpoints, final state); kFwdCkpt: the
// states entering every 16-step block only (the backward's replay input).
template <typename IO, int MODE, bool VEC>
__global__ void __launch_bounds__(128) fwd_pcbc_kernel(const __grid_constant__ FwdArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  constexpr bool kOut = MODE == kFwdOut;
  const int lane = threadIdx.x & 31, n = lane & 15, base = lane & 16;
  const long long nch = (long long)a.batch * a.dim;
  const long long cg = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  if (((long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) >> 4 >= nch) return;  // whole warps
  const bool act = cg < nch;
  const long long ch = act ? cg : nch - 1;  // idle lanes shadow a valid channel, store nothing
  const int L = a.L, N = a.N, d = (int)(ch % a.dim);
  const bool live = n < N;
  const IO* up = reinterpret_cast<const IO*>(a.u) + ch * L;
  const IO* dp = reinterpret_cast<const IO*>(a.delta) + ch * L;
  const IO* zp = (kOut && a.z) ? reinterpret_cast<const IO*>(a.z) + ch * L : nullptr;
  const IO* Bp = reinterpret_cast<const IO*>(a.B) + (ch * N + (live ? n : 0)) * (long long)L;
  const IO* Cp = reinterpret_cast<const IO*>(a.C) + (ch * N + (live ? n : 0)) * (long long)L;
  const float An = live ? a.A[(long long)d * N + n] * (kPrecise ? 1.f : kLog2e) : 0.f;
  float h = (a.h0 && live) ? a.h0[ch * N + n] : 0.f;
  const float bias = a.dt_bias ? a.dt_bias[d] : 0.f;
  const float Dd = (kOut && a.D) ? a.D[d] : 0.f;
  const int nblk16 = (L + 15) / 16;
  const int j = n >> 1;  // the step whose scalars (and output) this lane pair handles

  for (int t0 = 0; t0 < L; t0 += 8) {
    const int nv = min(8, L - t0);
    if ((t0 & 15) == 0 && a.ckpt && act && live) a.ckpt[(ch * nblk16 + t0 / 16) * N + n] = h;
    Row<IO, 8> rb, rc;
    load_seg<IO, 8, VEC>(rb, Bp + t0, live ? nv : 0);
    if (kOut) load_seg<IO, 8, VEC>(rc, Cp + t0, live ? nv : 0);
    float dl = 0.f, dx = 0.f, uj = 0.f, gate = 1.f;
    if (j < nv) {
      uj = ld1<IO>(up, t0 + j);
      const float v = ld1<IO>(dp, t0 + j) + bias;
      dl = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
      dx = dl * uj;
      if (zp) {
        const float zj = ld1<IO>(zp, t0 + j);
        gate = zj * (kPrecise ? sigmoid_precise(zj) : sigmoid_fast(zj));
      }
    }
    float yk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {  // steps past the end have Δ = 0: the state is unchanged
      const float dk = __shfl_sync(0xffffffffu, dl, base + 2 * k);
      const float xk = __shfl_sync(0xffffffffu, dx, base + 2 * k);
      const float abar = kPrecise ? expf(dk * An) : ex2_mufu(dk * An);
      h = fmaf(abar, h, xk * rb.get(k));
      yk[k] = kOut ? rc.get(k) * h : 0.f;
    }
    if (kOut) {
      const float y = reduce8(yk, n);
      if (act && (n & 1) == 0 && j < nv)
        st1<IO>(a.out, ch * L + t0 + j, fmaf(Dd, uj, y) * gate);
    }
  }
  if (kOut && a.hL && act && live) a.hL[ch * N + n] = h;
}

// Backward over 16-step blocks from the checkpoints.
template <typename IO, bool VEC>
__global__ void __launch_bounds__(128) bwd_pcbc_kernel(const __grid_constant__ BwdArgs a,
                                                      void* dB, void* dC) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  const int lane = threadIdx.x & 31, n = lane & 15, base = lane & 16;
  const long long nch = (long long)a.batch * a.dim;
  const long long cg = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  if (((long long)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) >> 4 >= nch) return;
  const bool act = cg < nch;
  const long long ch = act ? cg : nch - 1;
  const int L = a.L, N = a.N, d = (int)(ch % a.dim);
  const bool live = n < N;
  const float lv = (act && live) ? 1.f : 0.f;
  const long long xrow = ch * L;
  const long long brow = (ch * N + (live ? n : 0)) * (long long)L;
  const IO* Bp = reinterpret_cast<const IO*>(a.B) + brow;
  const IO* Cp = reinterpret_cast<const IO*>(a.C) + brow;
  const float ascale = kPrecise ? 1.f : kLog2e, aback = kPrecise ? 1.f : kLn2;
  const float An = live ? a.A[(long long)d * N + n] * ascale : 0.f;
  const float bias = a.dt_bias ? a.dt_bias[d] : 0.f;
  const float Dd = a.D ? a.D[d] : 0.f;
  float lam = (a.dhL && live) ? a.dhL[ch * N + n] : 0.f;
  float dA = 0.f, dD_acc = 0.f, db_acc = 0.f;
  const int nblk = (L + 15) / 16;

  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = 16 * blk, nv = min(16, L - t0);
    Row<IO, 16> rb, rc;
    load_seg<IO, 16, VEC>(rb, Bp + t0, live ? nv : 0);
    load_seg<IO, 16, VEC>(rc, Cp + t0, live ? nv : 0);
    // scalars of step n (one lane per step)
    float dl = 0.f, dx = 0.f, g = 0.f, gz = 0.f, sv = 1.f, un = 0.f;
    if (n < nv) {
      un = ld1<IO>(a.u, xrow + t0 + n);
      const float v = ld1<IO>(a.delta, xrow + t0 + n) + bias;
      if (a.softplus) {
        dl = kPrecise ? softplus_precise(v) : softplus_fast(v);
        sv = kPrecise ? sigmoid_precise(v) : sigmoid_fast(v);
      } else {
        dl = v;
      }
      dx = dl * un;
      const float go = ld1<IO>(a.dout, xrow + t0 + n);
      g = go;
      if (a.z) {
        const float zn = ld1<IO>(a.z, xrow + t0 + n);
        const float sg = kPrecise ? sigmoid_precise(zn) : sigmoid_fast(zn);
        g = go * zn * sg;
        gz = go * sg * fmaf(zn, 1.f - sg, 1.f);  // dout silu'(z)
      }
    }
    // replay the block from its checkpoint: states and decays of its 16 steps
    float h = live ? a.ckpt[(ch * nblk + blk) * N + n] : 0.f;
    float hist[16], ab[16], dk[16], xk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      dk[k] = __shfl_sync(0xffffffffu, dl, base + k);
      xk[k] = __shfl_sync(0xffffffffu, dx, base + k);
      ab[k] = kPrecise ? expf(dk[k] * An) : ex2_mufu(dk[k] * An);
      h = fmaf(ab[k], h, xk[k] * rb.get(k));
      hist[k] = h;
    }
    // adjoint, steps 15 .. 0
    float s1[16], s2[16], yv[16], vb[16], vc[16];
#pragma unroll
    for (int k = 15; k >= 0; --k) {
      const float gk = __shfl_sync(0xffffffffu, g, base + k);
      lam = fmaf(gk, rc.get(k), lam);                     // λ_t complete
      const float xv = fmaf(-xk[k], rb.get(k), hist[k]);  // Ā_t h_{t-1}
      const float qv = lam * xv;
      dA = fmaf(dk[k], qv, dA);
      s2[k] = An * qv;
      s1[k] = lam * rb.get(k);
      yv[k] = rc.get(k) * hist[k];
      vb[k] = lam * xk[k];                                // dB: λ Δ x
      vc[k] = gk * hist[k];                               // dC: g h
      lam *= ab[k];                                       // Ā_t λ_t for step t-1
    }
    const float S1 = reduce16(s1, n), S2 = reduce16(s2, n), Y = reduce16(yv, n);
    if (act && n < nv) {  // lane n owns step n
      const float du = fmaf(g, Dd, dl * S1);
      const float dd = fmaf(un, S1, S2 * aback);
      const float ddl = a.softplus ? dd * sv : dd;
      if (a.du) st1<IO>(a.du, xrow + t0 + n, du);
      if (a.ddelta) st1<IO>(a.ddelta, xrow + t0 + n, ddl);
      if (a.dz && a.z) st1<IO>(a.dz, xrow + t0 + n, gz * fmaf(Dd, un, Y));
      dD_acc = fmaf(g, un, dD_acc);
      db_acc += ddl;
    }
    if (act && live) {  // this lane's rows of dB, dC
      float ob[16], oc[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        ob[k] = vb[k];
        oc[k] = vc[k];
      }
      if (dB) {
        IO* p = reinterpret_cast<IO*>(dB) + brow + t0;
        if (VEC && nv == 16) store_row<IO, 16, true>(p, ob, 16);
        else store_row<IO, 16, false>(p, ob, nv);
      }
      if (dC) {
        IO* p = reinterpret_cast<IO*>(dC) + brow + t0;
        if (VEC && nv == 16) store_row<IO, 16, true>(p, oc, 16);
        else store_row<IO, 16, false>(p, oc, nv);
      }
    }
  }
  // the channel's sums over its 16 lanes (steps were owned by different lanes)
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, m);
    db_acc += __shfl_xor_sync(0xffffffffu, db_acc, m);
  }
  if (!act) return;
  float* pa = a.part_adt + ch * (kNS + 2);
  if (live) {
    pa[n] = dA * lv;  // Σ λ Δ Ā h_{t-1} (no A factor)
    if (a.dh0) a.dh0[ch * N + n] = lam;
  }
  if (n == 0) {
    pa[kNS] = dD_acc;
    pa[kNS + 1] = db_acc;
  }
}

}  // namespace

cudaError_t launch_fwd_pcbc(const FwdArgs& a, int io, bool vec, int mode, cudaStream_t s) {
  const long long threads = (long long)a.batch * a.dim * 16;
  const int tpb = 128;
  const unsigned grid = (unsigned)((threads + tpb - 1) / tpb);
  const bool out = mode == kFwdOut;
  if (io == 1) {
    if (out) vec ? fwd_pcbc_kernel<uint16_t, kFwdOut, true><<<grid, tpb, 0, s>>>(a)
                 : fwd_pcbc_kernel<uint16_t, kFwdOut, false><<<grid, tpb, 0, s>>>(a);
    else vec ? fwd_pcbc_kernel<uint16_t, kFwdCkpt, true><<<grid, tpb, 0, s>>>(a)
             : fwd_pcbc_kernel<uint16_t, kFwdCkpt, false><<<grid, tpb, 0, s>>>(a);
  } else {
    if (out) vec ? fwd_pcbc_kernel<float, kFwdOut, true><<<grid, tpb, 0, s>>>(a)
                 : fwd_pcbc_kernel<float, kFwdOut, false><<<grid, tpb, 0, s>>>(a);
    else vec ? fwd_pcbc_kernel<float, kFwdCkpt, true><<<grid, tpb, 0, s>>>(a)
             : fwd_pcbc_kernel<float, kFwdCkpt, false><<<grid, tpb, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_pcbc(const BwdArgs& a, int io, bool vec, void* dB, void* dC, cudaStream_t s) {
  const long long threads = (long long)a.batch * a.dim * 16;
  const int tpb = 128;
  const unsigned grid = (unsigned)((threads + tpb - 1) / tpb);
  if (io == 1) vec ? bwd_pcbc_kernel<uint16_t, true><<<grid, tpb, 0, s>>>(a, dB, dC)
                   : bwd_pcbc_kernel<uint16_t, false><<<grid, tpb, 0, s>>>(a, dB, dC);
  else vec ? bwd_pcbc_kernel<float, true><<<grid, tpb, 0, s>>>(a, dB, dC)
           : bwd_pcbc_kernel<float, false><<<grid, tpb, 0, s>>>(a, dB, dC);
  return cudaGetLastError();
}

}  // namespace ssm
