// Scalar-decay selective scan for large state sizes (N = 32, 64, 128) in its chunked matrix form,
// on the tensor cores, sm_100a, bf16 io.
//
// With one decay rate A_d per channel (the Mamba-2 restriction noted on the "2024 Reading List:
// Neural Network" page, section on state-space models, where the scalar transition is what lets
// the state grow to N = 64..128), the scan h_t = e^{Δ_t A_d} h_{t-1} + Δ_t x_t B_t,
// y_t = C_t . h_t + D_d x_t, out_t = y_t silu(z_t) has, over a chunk of T steps with cumulative
// steps S_t = Σ_{r <= t} Δ_r (from the chunk start) and state h_in entering the chunk,
//   y_t   = Σ_{s <= t} (C_t . B_s) e^{A (S_t - S_s)} Δ_s x_s  +  e^{A S_t} (C_t . h_in)  +  D x_t
//   h_out = e^{A S_{T-1}} h_in + Σ_s e^{A (S_{T-1} - S_s)} Δ_s x_s B_s,
// the masked-matrix ("state-space duality") form of the scan, whose products over states and
// steps are dense contractions.  Because A is a scalar per channel, the decay factor is rank one
// in (t, s) for every channel: e^{A (S_t - S_s)} = P_t Q_s with P_t = e^{A (S_t - S_m)},
// Q_s = 1 / P_s about the chunk's middle step m.  So with B, C shared by the channels of a batch
// row the chunk is four matrix products over a tile of 64 channels:
//   G  = C B^T                  [T x T]   (K = N)
//   Y1 = mask(G) X',  X'[s][d]  = Q_s Δ_s x_s                 [T x 64]  (K = T)
//   Y2 = C H_in                                                 [T x 64]  (K = N)
//   U  = B^T X'',  X''[s][d] = e^{A (S_{T-1} - S_s)} Δ_s x_s  [N x 64]  (K = T)
// and y = P Y1 + e^{A S_t} Y2 + D x,  h_out = e^{A S_{T-1}} h_in + U.  The products run as
// warp-level bf16 tensor-core MMAs (m16n8k16, f32 accumulation); the state H stays in shared
// memory in f32 (a bf16 copy feeds Y2).  P_t and Q_s grow as e^{|A| S} inside a chunk: a channel
// whose chunk would leave the safe range (|A| S_{T-1} > 80, or a non-finite step) is computed for
// that chunk by an exact sequential pass instead (its columns of the products are ignored).
#include <stdint.h>

#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace {

constexpr int kT = 16;        // steps per chunk (one MMA k-step)
constexpr int kDB = 64;       // channels per CTA
constexpr int kThreads = 128; // 4 warps, 16 channels each in the products
constexpr int kPadH = 8;      // bf16 row padding of the [*][N] and [*][T] operand tiles

__device__ __forceinline__ uint32_t ld32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ uint16_t to_bf16(float x) { return f32_to_bf16(x); }

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16 x 8 output tile: D += A[16 x K] B[K x 8].  A row-major at a (row stride lda elements);
// B given as its transpose [8][K] at b (row stride ldb), i.e. the MMA's column-major operand.
template <int K>
__device__ __forceinline__ void mma_tile(float (&d)[4], const uint16_t* a, int lda,
                                         const uint16_t* b, int ldb, int lane) {
  const int g = lane >> 2, tg = lane & 3;
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    const uint16_t* ar = a + g * lda + k0 + 2 * tg;
    const uint16_t* br = b + g * ldb + k0 + 2 * tg;
    mma16816(d, ld32(ar), ld32(ar + 8 * lda), ld32(ar + 8), ld32(ar + 8 * lda + 8), ld32(br),
             ld32(br + 8));
  }
}

template <int N>
struct SsdSmem {
  static constexpr int kLdN = N + kPadH;    // [*][N] tiles
  static constexpr int kLdT = kT + kPadH;   // [*][T] tiles
  float H[kDB * N];              // state, [d][n], f32
  uint16_t Hb[kDB * kLdN];       // bf16 copy of H (B operand of Y2: [d][n])
  uint16_t Ct[kT * kLdN];        // C as [t][n] (A operand of G and Y2)
  uint16_t Bt[kT * kLdN];        // B as [s][n] (B operand of G)
  uint16_t Bn[N * kLdT];         // B as [n][s] (A operand of U)
  uint16_t Gm[kT * kLdT];        // mask(G) as [t][s] (A operand of Y1)
  uint16_t X1[kDB * kLdT];       // X'  as [d][s]
  uint16_t X2[kDB * kLdT];       // X'' as [d][s]
  float P[kDB * kT], E[kDB * kT], Ux[kDB * kT], Gt[kDB * kT], Dl[kDB * kT], Xs[kDB * kT];
  float Eend[kDB], Dskip[kDB];
  int fb[kDB];
  uint16_t Y[kDB * kT];          // gated outputs of the chunk, [d][t]
};

template <int N>
__global__ void __launch_bounds__(kThreads) ssd_fwd_kernel(const __grid_constant__ FwdArgs a) {
  using SM = SsdSmem<N>;
  extern __shared__ float4 smem_ssd[];
  SM& sm = *reinterpret_cast<SM*>(smem_ssd);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nblk_d = (a.dim + kDB - 1) / kDB;
  const int b = blockIdx.x / nblk_d;
  const int d0 = (blockIdx.x % nblk_d) * kDB;
  const int L = a.L;
  const int gbc = d0 / (a.dim / a.bc_groups);
  const uint16_t* Bg = reinterpret_cast<const uint16_t*>(a.B) + ((long long)b * a.bc_groups + gbc) * N * (long long)L;
  const uint16_t* Cg = reinterpret_cast<const uint16_t*>(a.C) + ((long long)b * a.bc_groups + gbc) * N * (long long)L;

  // per-channel constants (threads 0..63 own channel d0 + tid in the elementwise phases)
  const int dl = tid & (kDB - 1);
  const bool own = tid < kDB;
  const int d = min(d0 + dl, a.dim - 1);
  const bool dact = d0 + dl < a.dim;
  const long long row = ((long long)b * a.dim + d) * L;
  const float Ad = a.A[d];
  const float bias = a.dt_bias ? a.dt_bias[d] : 0.f;
  const float Dd = a.D ? a.D[d] : 0.f;

  // initial state
  for (int i = tid; i < kDB * N; i += kThreads) {
    const int dd = i / N, n = i % N;
    const int dg = d0 + dd;
    sm.H[i] = (a.h0 && dg < a.dim) ? a.h0[((long long)b * a.dim + dg) * N + n] : 0.f;
  }

  for (int t0 = 0; t0 < L; t0 += kT) {
    const int nv = min(kT, L - t0);
    __syncthreads();  // the previous chunk's reads of every table are done
    // ---- phase A: channel scalars (threads 0..63) and the B/C tiles (threads 64..127)
    if (own) {
      // the chunk's 16 steps of u, delta, z: two 16-byte pieces per row when aligned
      uint32_t uw[8], dw[8], zw[8];
      const auto load16 = [&](const void* base, uint32_t (&w)[8]) {
        const uint16_t* p = reinterpret_cast<const uint16_t*>(base) + row + t0;
        if (nv == kT && a.rows16) {
          const uint4 v0 = reinterpret_cast<const uint4*>(p)[0], v1 = reinterpret_cast<const uint4*>(p)[1];
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
          w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = 0u;
          for (int e = 0; e < nv; ++e) w[e >> 1] |= (uint32_t)p[e] << (16 * (e & 1));
        }
      };
      load16(a.u, uw);
      load16(a.delta, dw);
      if (a.z) load16(a.z, zw);
      float S = 0.f;
      float mx = 0.f;
      bool bad = false;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        float Dv = 0.f, xv = 0.f, gv = 1.f;
        if (t < nv) {
          const float u = (t & 1) ? bf16_hi(uw[t >> 1]) : bf16_lo(uw[t >> 1]);
          const float v = ((t & 1) ? bf16_hi(dw[t >> 1]) : bf16_lo(dw[t >> 1])) + bias;
          Dv = a.softplus ? softplus_fast(v) : v;
          xv = Dv * u;
          if (a.z) {
            const float zv = (t & 1) ? bf16_hi(zw[t >> 1]) : bf16_lo(zw[t >> 1]);
            gv = zv * sigmoid_fast(zv);
          }
          sm.Ux[dl * kT + t] = u;  // x_t for the D skip
        } else {
          sm.Ux[dl * kT + t] = 0.f;
        }
        S += Dv;
        bad = bad || !(Dv == Dv) || fabsf(Dv) > 3.0e38f;
        sm.Dl[dl * kT + t] = S;   // cumulative step S_t
        sm.Xs[dl * kT + t] = xv;  // Δ_t x_t
        sm.Gt[dl * kT + t] = gv;  // silu(z_t)
        mx = fmaxf(mx, fabsf(S));
      }
      sm.fb[dl] = (bad || fabsf(Ad) * mx > 80.f) ? 1 : 0;
      sm.Dskip[dl] = Dd;
    } else {
      const int i0 = tid - kDB;  // 64 threads load N rows x 16 steps of B and of C
      for (int i = i0; i < N * 2; i += kThreads - kDB) {
        const int n = i >> 1, h = i & 1;  // steps 8 h .. 8 h + 7 of state row n
        uint32_t bw[4] = {0u, 0u, 0u, 0u}, cw[4] = {0u, 0u, 0u, 0u};
        const long long off = (long long)n * L + t0 + 8 * h;
        if (8 * h + 8 <= nv && ((off & 7) == 0) && a.rows16) {  // aligned 16-byte pieces
          const uint4 vb = *reinterpret_cast<const uint4*>(Bg + off);
          const uint4 vc = *reinterpret_cast<const uint4*>(Cg + off);
          bw[0] = vb.x; bw[1] = vb.y; bw[2] = vb.z; bw[3] = vb.w;
          cw[0] = vc.x; cw[1] = vc.y; cw[2] = vc.z; cw[3] = vc.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (8 * h + e < nv) {
              bw[e >> 1] |= (uint32_t)Bg[off + e] << (16 * (e & 1));
              cw[e >> 1] |= (uint32_t)Cg[off + e] << (16 * (e & 1));
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint16_t vb = (uint16_t)(bw[e >> 1] >> (16 * (e & 1)));
          const uint16_t vc = (uint16_t)(cw[e >> 1] >> (16 * (e & 1)));
          const int s = 8 * h + e;
          sm.Bn[n * SM::kLdT + s] = vb;
          sm.Bt[s * SM::kLdN + n] = vb;
          sm.Ct[s * SM::kLdN + n] = vc;
        }
      }
    }
    __syncthreads();
    // ---- phase B: decay factors and scaled inputs (threads 0..63); bf16 copy of the state
    if (own) {
      const float Sm = sm.Dl[dl * kT + kT / 2 - 1], Send = sm.Dl[dl * kT + kT - 1];
      const bool fbk = sm.fb[dl] != 0;
      const float eAm = expf(Ad * Sm), eEnd_m = expf(Ad * (Send - Sm));
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const float S = sm.Dl[dl * kT + t];
        const float P = expf(Ad * (S - Sm));                 // e^{A (S_t - S_m)}
        const float Q = expf(Ad * (Sm - S));                 // 1 / P_t
        const float x = sm.Xs[dl * kT + t];
        sm.P[dl * kT + t] = P;
        sm.E[dl * kT + t] = eAm * P;                         // e^{A S_t}
        sm.X1[dl * SM::kLdT + t] = to_bf16(fbk ? 0.f : Q * x);
        sm.X2[dl * SM::kLdT + t] = to_bf16(fbk ? 0.f : eEnd_m * Q * x);  // e^{A (S_end - S_t)} x
      }
      sm.Eend[dl] = expf(Ad * Send);
    }
    for (int i = tid; i < kDB * N; i += kThreads) {
      const int dd = i / N, n = i % N;
      sm.Hb[dd * SM::kLdN + n] = to_bf16(sm.H[i]);
    }
    __syncthreads();
    // ---- phase C: the products.  Warps 0, 1: G; every warp: its 16 channels of Y2 and U
    if (warp < 2) {
      float g[4] = {0.f, 0.f, 0.f, 0.f};
      mma_tile<N>(g, sm.Ct, SM::kLdN, sm.Bt + (8 * warp) * SM::kLdN, SM::kLdN, lane);
      const int r = lane >> 2, c = 8 * warp + 2 * (lane & 3);
      // mask: s <= t
      sm.Gm[r * SM::kLdT + c] = to_bf16(c <= r ? g[0] : 0.f);
      sm.Gm[r * SM::kLdT + c + 1] = to_bf16(c + 1 <= r ? g[1] : 0.f);
      sm.Gm[(r + 8) * SM::kLdT + c] = to_bf16(c <= r + 8 ? g[2] : 0.f);
      sm.Gm[(r + 8) * SM::kLdT + c + 1] = to_bf16(c + 1 <= r + 8 ? g[3] : 0.f);
    }
    float y2[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      y2[j][0] = y2[j][1] = y2[j][2] = y2[j][3] = 0.f;
      mma_tile<N>(y2[j], sm.Ct, SM::kLdN, sm.Hb + (16 * warp + 8 * j) * SM::kLdN, SM::kLdN, lane);
    }
    // U = B^T X'': rows n (N / 16 tiles), columns the warp's 16 channels; h_out = e^{A S_end} h + U
#pragma unroll
    for (int mt = 0; mt < N / 16; ++mt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float u4[4] = {0.f, 0.f, 0.f, 0.f};
        mma_tile<kT>(u4, sm.Bn + (16 * mt) * SM::kLdT, SM::kLdT,
                     sm.X2 + (16 * warp + 8 * j) * SM::kLdT, SM::kLdT, lane);
        const int n = 16 * mt + (lane >> 2), dd = 16 * warp + 8 * j + 2 * (lane & 3);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int nn = n + (e >> 1) * 8, dc = dd + (e & 1);
          if (!sm.fb[dc]) sm.H[dc * N + nn] = fmaf(sm.Eend[dc], sm.H[dc * N + nn], u4[e]);
        }
      }
    }
    __syncthreads();  // Gm is complete
    // Y1 = mask(G) X' and the outputs of the warp's 16 channels
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float y1[4] = {0.f, 0.f, 0.f, 0.f};
      mma_tile<kT>(y1, sm.Gm, SM::kLdT, sm.X1 + (16 * warp + 8 * j) * SM::kLdT, SM::kLdT, lane);
      const int t = lane >> 2, dd = 16 * warp + 8 * j + 2 * (lane & 3);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tt = t + (e >> 1) * 8, dc = dd + (e & 1);
        if (sm.fb[dc]) continue;
        const int k = dc * kT + tt;
        const float y = fmaf(sm.P[k], y1[e], fmaf(sm.E[k], y2[j][e], sm.Dskip[dc] * sm.Ux[k]));
        sm.Y[k] = to_bf16(y * sm.Gt[k]);
      }
    }
    __syncthreads();
    // ---- phase D: channels whose chunk left the factorization's range: exact sequential pass
    if (own && sm.fb[dl]) {
      float prevS = 0.f;
      for (int t = 0; t < nv; ++t) {
        const float S = sm.Dl[dl * kT + t];
        const float ab = expf(Ad * (S - prevS));
        prevS = S;
        const float x = sm.Xs[dl * kT + t];
        float y = 0.f;
        for (int n = 0; n < N; ++n) {
          const float hb = fmaf(ab, sm.H[dl * N + n], x * bf16_to_f32(sm.Bt[t * SM::kLdN + n]));
          sm.H[dl * N + n] = hb;
          y = fmaf(bf16_to_f32(sm.Ct[t * SM::kLdN + n]), hb, y);
        }
        sm.Y[dl * kT + t] = to_bf16(fmaf(Dd, sm.Ux[dl * kT + t], y) * sm.Gt[dl * kT + t]);
      }
    }
    __syncthreads();
    // ---- outputs of the chunk
    if (own && dact) {
      uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + row + t0;
      if (nv == kT && ((row + t0) & 7) == 0 && a.rows16) {
        const uint4* src = reinterpret_cast<const uint4*>(sm.Y + dl * kT);
        reinterpret_cast<uint4*>(o)[0] = src[0];
        reinterpret_cast<uint4*>(o)[1] = src[1];
      } else {
        for (int t = 0; t < nv; ++t) o[t] = sm.Y[dl * kT + t];
      }
    }
  }
  __syncthreads();
  if (a.hL) {
    for (int i = tid; i < kDB * N; i += kThreads) {
      const int dd = i / N, n = i % N;
      const int dg = d0 + dd;
      if (dg < a.dim) a.hL[((long long)b * a.dim + dg) * N + n] = sm.H[i];
    }
  }
}

}  // namespace

cudaError_t launch_ssd_fwd(const FwdArgs& a, cudaStream_t s) {
  const unsigned grid = (unsigned)((long long)a.batch * ((a.dim + kDB - 1) / kDB));
  switch (a.N) {
    case 32: {
      auto k = ssd_fwd_kernel<32>;
      const size_t sm = sizeof(SsdSmem<32>);
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      k<<<grid, kThreads, sm, s>>>(a);
      break;
    }
    case 64: {
      auto k = ssd_fwd_kernel<64>;
      const size_t sm = sizeof(SsdSmem<64>);
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      k<<<grid, kThreads, sm, s>>>(a);
      break;
    }
    case 128: {
      auto k = ssd_fwd_kernel<128>;
      const size_t sm = sizeof(SsdSmem<128>);
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      k<<<grid, kThreads, sm, s>>>(a);
      break;
    }
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ssm
