// Forward selective scan (S6), sm_100a: one lane per channel.
//
// What is computed is the scan of ssm_fwd_impl.cuh (per channel c = (b, d), time t, state n):
//   Δ_t = softplus(delta_t + dt_bias_d),  h_t,n = exp(Δ_t A_dn) h_{t-1},n + Δ_t B_t,n x_t,
//   y_t = Σ_n C_t,n h_t,n + D_d x_t,  out_t = y_t * silu(z_t)
// ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces", summary page, sections
// "Yöntem" and "Seçim Mekanizması (S6)"; the state never leaves the chip, "Donanım Duyarlı Durum
// Genişletme").  This file is the kernel for the default variant (per-state decay, Euler input
// term, forward direction, [batch][dim][L] rows that allow 16-byte copies, B/C shared by at least
// 32 consecutive channels); every other variant runs in ssm_fwd_impl.cuh.
//
// B200 mapping:
//   * lane l of a warp owns channel d0 + l completely: its 16 states live in its registers, it
//     computes its own step size, input term, readout and gated output, so no per-step value
//     crosses lanes.  The warp's 32 channels share B_t and C_t, which every lane reads as
//     warp-uniform 16-byte shared-memory broadcasts (8 per step);
//   * all streamed inputs (the lane's u, delta, z rows and the warp's B/C tile) are copied by
//     cp.async into a 4-slot shared-memory ring, 16-step blocks up to three ahead of the block
//     being computed, so no register holds data in flight and no load latency reaches the loop;
//     the B/C tile of the next block is turned into f32 [step][state] once per block;
//   * the per-element work (Δ A, 2^x, Δ x B, the state FMA and the C readout) runs as packed
//     f32x2 instructions; KE / KO of the 8 state pairs take 2^x from the MUFU unit at even / odd
//     steps and the rest from the FMA-pipe polynomial (ssm_device.cuh), which needs
//     |Δ A log2 e| <= 126: a warp vote per block selects that body, or one with every
//     exponential on MUFU when some lane's block leaves the range;
//   * the step sizes of block i+1 are computed in the same straight-line body as block i's
//     recurrence, so their MUFU work (softplus) interleaves with the state updates.
#pragma once

#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace lane {

constexpr int kT = 16;                   // steps per block
constexpr int kStages = 4;               // blocks held in the shared-memory ring
constexpr int kBCStride = kT * kNS + 16;  // f32 [step][state] tile; steps 8..15 shifted 16 floats

// Offset of (step k, state n) in a B/C tile.  Steps 8..15 are shifted by 16 floats so that the
// two half-warps staging steps k and k + 8 of the same state write different banks.
__device__ __forceinline__ int bc_off(int k, int n) { return k * kNS + n + (k >= 8 ? 16 : 0); }

template <typename IO>
struct Geo {
  static constexpr int kES = (int)sizeof(IO);
  static constexpr int kRowBytes = kT * kES;          // one 16-step row segment
  static constexpr int kRowStride = kRowBytes + 16;   // padded: conflict-free 16-byte reads
  static constexpr int kPieces = kRowBytes / 16;      // 16-byte pieces per row segment
  static constexpr int kStepsPerPiece = 16 / kES;
  static constexpr int kRowsBytes = 32 * kRowStride;  // one tensor's rows for 32 lanes
  static constexpr int kSlotBytes = 3 * kRowsBytes + 2 * kNS * kRowBytes;
  static constexpr int kRingBytes = kStages * kSlotBytes;
  static constexpr int kWarpBytes = kRingBytes + 2 * 2 * kBCStride * 4;
};

// ---------------------------------------------------------------- cp.async (16-byte pieces)
// src_bytes < 16 zero-fills the rest of the piece (0: nothing is read).
__device__ __forceinline__ void cp16(void* smem, const void* gmem, int src_bytes) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Eight io values of a 16-byte piece (bf16) or two pieces (f32) as floats.
template <typename IO>
__device__ __forceinline__ void unpack8(const unsigned char* p, float (&v)[8]) {
  if constexpr (sizeof(IO) == 2) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// One step of the lane's 16 states: h <- Ā h + Δ x B, returns Σ C h.  KP of the 8 state pairs
// take 2^x from MUFU, the others from the FMA-pipe polynomial (range checked by the caller's
// vote); PRECISE (fp32 io) uses the library expf for every state.
template <bool PRECISE, bool READOUT, int KP>
__device__ __forceinline__ float lane_step(float2 (&h)[8], const float2 (&al)[8], float dl, float du,
                                           const float* __restrict__ bk,
                                           const float* __restrict__ ck) {
  float4 bq[4], cq[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    bq[q] = reinterpret_cast<const float4*>(bk)[q];
    if (READOUT) cq[q] = reinterpret_cast<const float4*>(ck)[q];
  }
  const float2 d2 = f2(dl), du2 = f2(du);
  float2 ya = make_float2(0.f, 0.f), yb = ya;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float2 av;
    if (PRECISE) {
      av = make_float2(expf(dl * al[j].x), expf(dl * al[j].y));
    } else if (j < KP) {
      const float2 x = mul2(d2, al[j]);
      av = make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
    } else {
      av = exp2_fma_prod_x2(d2, al[j]);
    }
    const float4 bb = bq[j >> 1];
    const float2 bp = (j & 1) ? make_float2(bb.z, bb.w) : make_float2(bb.x, bb.y);
    h[j] = fma2(av, h[j], mul2(du2, bp));
    if (READOUT) {
      const float4 cc = cq[j >> 1];
      const float2 cp = (j & 1) ? make_float2(cc.z, cc.w) : make_float2(cc.x, cc.y);
      if (j & 1) yb = fma2(cp, h[j], yb);
      else ya = fma2(cp, h[j], ya);
    }
  }
  const float2 ys = add2(ya, yb);
  return ys.x + ys.y;
}

template <typename IO, int MODE>
struct LaneScan {
  using G = Geo<IO>;
  static constexpr bool kPrecise = std::is_same<IO, float>::value;
  static constexpr bool kOut = MODE == kFwdOut;

  const FwdArgs& a;
  unsigned char* ring;
  float* bcf;  // [2 buffers][B, C][kBCStride]
  const IO* up;
  const IO* dp;
  const IO* zp;
  IO* op;
  const IO* Bp;
  const IO* Cp;
  long long ch;
  int lane, t_begin, t_end, nblk, N, L;
  bool act;
  float bias, Dd;

  __device__ __forceinline__ unsigned char* slot(int blk) const {
    return ring + (blk % kStages) * G::kSlotBytes;
  }

  // Copies of block blk (index within the chunk) into its ring slot; one commit group per
  // block index (empty past the last block), so the wait counts stay uniform.
  __device__ __forceinline__ void issue(int blk) const {
    if (blk < nblk) {
      unsigned char* s = slot(blk);
      const int t0 = t_begin + blk * kT;
#pragma unroll
      for (int c = 0; c < G::kPieces; ++c) {
        const int tc = t0 + c * G::kStepsPerPiece;
        const int nb = max(0, min(16, (t_end - tc) * G::kES));
        const long long off = nb > 0 ? tc : t_begin;  // an in-bounds address when nothing is read
        unsigned char* dst = s + lane * G::kRowStride + c * 16;
        cp16(dst, up + off, nb);
        cp16(dst + G::kRowsBytes, dp + off, nb);
        if (zp) cp16(dst + 2 * G::kRowsBytes, zp + off, nb);
      }
      unsigned char* raw = s + 3 * G::kRowsBytes;
#pragma unroll
      for (int p0 = 0; p0 < kNS * G::kPieces; p0 += 32) {
        const int p = p0 + lane;
        const int n = p / G::kPieces, c = p % G::kPieces;
        const int tc = t0 + c * G::kStepsPerPiece;
        const int nb = n < N ? max(0, min(16, (t_end - tc) * G::kES)) : 0;
        const long long off = (long long)(n < N ? n : 0) * L + (nb > 0 ? tc : t_begin);
        cp16(raw + n * G::kRowBytes + c * 16, Bp + off, nb);
        if (kOut) cp16(raw + (kNS + n) * G::kRowBytes + c * 16, Cp + off, nb);
      }
    }
    cp_commit();
  }

  // The landed B/C tile of block blk as f32 [step][state] into buffer buf: lane l turns state
  // l/2, steps 8 (l & 1) .. + 7 of each tile.
  __device__ __forceinline__ void convert_bc(int blk, int buf) const {
    const unsigned char* raw = slot(blk) + 3 * G::kRowsBytes;
    float* sb = bcf + buf * 2 * kBCStride;
    const int n = lane >> 1, hh = lane & 1;
#pragma unroll
    for (int which = 0; which < (kOut ? 2 : 1); ++which) {
      float v[8];
      unpack8<IO>(raw + (which * kNS + n) * G::kRowBytes + hh * 8 * G::kES, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) sb[which * kBCStride + bc_off(8 * hh + j, n)] = v[j];
    }
  }

  // Row segment of one tensor (0 = u, 1 = delta, 2 = z) of block blk, as 16 floats.
  __device__ __forceinline__ void row(int blk, int tensor, float (&v)[kT]) const {
    const unsigned char* p = slot(blk) + tensor * G::kRowsBytes + lane * G::kRowStride;
    float lo[8], hi[8];
    unpack8<IO>(p, lo);
    unpack8<IO>(p + 8 * G::kES, hi);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = lo[k];
      v[8 + k] = hi[k];
    }
  }

  // Step sizes Δ and input scales Δ x of block blk; steps past the end get Δ = 0 (the state is
  // then left unchanged).  m: the largest |Δ| (an infinite Δ fails the range vote; a NaN Δ
  // reaches every state through its input term Δ x B whichever body runs).
  __device__ __forceinline__ void scalars(int blk, float (&dl)[kT], float (&du)[kT], float& m,
                                          float& dsum) const {
    float dv[kT], uv[kT];
    row(blk, 1, dv);
    row(blk, 0, uv);
    const int nvalid = t_end - (t_begin + blk * kT);
    m = 0.f;
    dsum = 0.f;
#pragma unroll
    for (int k = 0; k < kT; k += 2) {
      const float2 v = add2(make_float2(dv[k], dv[k + 1]), f2(bias));
      float2 s = v;
      if (a.softplus) {
        if (kPrecise) s = make_float2(softplus_precise(v.x), softplus_precise(v.y));
        else s = softplus_fast_x2(v);
      }
      s.x = k < nvalid ? s.x : 0.f;
      s.y = k + 1 < nvalid ? s.y : 0.f;
      const float2 x = mul2(s, make_float2(uv[k], uv[k + 1]));
      dl[k] = s.x;
      dl[k + 1] = s.y;
      du[k] = x.x;
      du[k + 1] = x.y;
      m = fmaxf(m, fmaxf(fabsf(s.x), fabsf(s.y)));
      if (MODE == kFwdSummary) dsum += s.x + s.y;
    }
  }

  // Gated outputs of block blk from its readouts y.
  __device__ __forceinline__ void output(int blk, const float (&y)[kT]) const {
    float uv[kT], zv[kT], o[kT];
    row(blk, 0, uv);
    if (zp) row(blk, 2, zv);
#pragma unroll
    for (int k = 0; k < kT; k += 2) {
      float2 yy = fma2(f2(Dd), make_float2(uv[k], uv[k + 1]), make_float2(y[k], y[k + 1]));
      if (zp) {
        const float2 z2 = make_float2(zv[k], zv[k + 1]);
        const float2 sg = kPrecise ? make_float2(sigmoid_precise(z2.x), sigmoid_precise(z2.y))
                                   : sigmoid_fast_x2(z2);
        yy = mul2(yy, mul2(z2, sg));
      }
      o[k] = yy.x;
      o[k + 1] = yy.y;
    }
    if (!act) return;
    const int t0 = t_begin + blk * kT;
    const int nvalid = min(kT, t_end - t0);
#pragma unroll
    for (int c = 0; c < G::kPieces; ++c) {
      if (c * G::kStepsPerPiece >= nvalid) break;  // row lengths are whole pieces
      uint4 w;
      if constexpr (sizeof(IO) == 2) {
        w = make_uint4(pack_bf16x2(o[8 * c], o[8 * c + 1]), pack_bf16x2(o[8 * c + 2], o[8 * c + 3]),
                       pack_bf16x2(o[8 * c + 4], o[8 * c + 5]),
                       pack_bf16x2(o[8 * c + 6], o[8 * c + 7]));
      } else {
        w = make_uint4(__float_as_uint(o[4 * c]), __float_as_uint(o[4 * c + 1]),
                       __float_as_uint(o[4 * c + 2]), __float_as_uint(o[4 * c + 3]));
      }
      __stcs(reinterpret_cast<uint4*>(op + t0 + c * G::kStepsPerPiece), w);
    }
  }

  __device__ __forceinline__ void store_state(float* dst, const float2 (&h)[8], int n_out) const {
    if (n_out == kNS && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<float4*>(dst)[j] = make_float4(h[2 * j].x, h[2 * j].y, h[2 * j + 1].x,
                                                         h[2 * j + 1].y);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (2 * j < n_out) dst[2 * j] = h[j].x;
        if (2 * j + 1 < n_out) dst[2 * j + 1] = h[j].y;
      }
    }
  }

  // Block i: issue block i+3's copies, stage block i+1's B/C and step sizes, run block i's 16
  // steps and write its outputs.  One straight-line body, so the compiler interleaves the
  // next block's scalar work with this block's recurrence.
  template <int KE, int KO>
  __device__ __forceinline__ void body(int i, float2 (&h)[8], const float2 (&al)[8],
                                       float (&dl)[kT], float (&du)[kT], float& m, float& dsum) const {
    issue(i + kStages - 1);
    convert_bc(i + 1, (i + 1) & 1);
    if (a.ckpt && act) {
      const int nblk_total = (L + kT - 1) / kT;
      store_state(a.ckpt + (ch * nblk_total + (t_begin / kT + i)) * N, h, N);
    }
    float dl_n[kT], du_n[kT], m_n, ds_n;
    scalars(i + 1, dl_n, du_n, m_n, ds_n);
    const float* bk = bcf + (i & 1) * 2 * kBCStride;
    float y[kT];
#pragma unroll
    for (int k = 0; k < kT; k += 2) {
      y[k] = lane_step<kPrecise, kOut, KE>(h, al, dl[k], du[k], bk + bc_off(k, 0),
                                           bk + kBCStride + bc_off(k, 0));
      y[k + 1] = lane_step<kPrecise, kOut, KO>(h, al, dl[k + 1], du[k + 1], bk + bc_off(k + 1, 0),
                                               bk + kBCStride + bc_off(k + 1, 0));
    }
    if (kOut) output(i, y);
#pragma unroll
    for (int k = 0; k < kT; ++k) {
      dl[k] = dl_n[k];
      du[k] = du_n[k];
    }
    m = m_n;
    dsum = ds_n;
  }
};

template <typename IO, int MODE, int KE, int KO>
__global__ void __launch_bounds__(32, 1) fwd_lane_kernel(const __grid_constant__ FwdArgs a) {
  using Scan = LaneScan<IO, MODE>;
  using G = Geo<IO>;
  constexpr bool kPrecise = Scan::kPrecise;
  extern __shared__ float4 smem_lane[];
  const int lane = threadIdx.x & 31;
  const long long w = blockIdx.x;
  if (w >= a.nwarps) return;
  const int b = (int)(w / a.warps_per_b);
  const int d0 = (int)(w % a.warps_per_b) * 32;
  const int d = d0 + lane;
  const bool act = d < a.dim;
  const int dd = act ? d : a.dim - 1;  // idle lanes shadow a valid channel and store nothing
  const long long ch = (long long)b * a.dim + dd;
  const int chunk = blockIdx.y;
  const int L = a.L, N = a.N;
  const int gbc = d0 / (a.dim / a.bc_groups);  // the warp's channels share one B/C group

  Scan sc{a};
  sc.ring = reinterpret_cast<unsigned char*>(smem_lane);
  sc.bcf = reinterpret_cast<float*>(sc.ring + G::kRingBytes);
  const long long rowx = ch * (long long)L;
  sc.up = reinterpret_cast<const IO*>(a.u) + rowx;
  sc.dp = reinterpret_cast<const IO*>(a.delta) + rowx;
  sc.zp = (Scan::kOut && a.z) ? reinterpret_cast<const IO*>(a.z) + rowx : nullptr;
  sc.op = Scan::kOut ? reinterpret_cast<IO*>(a.out) + rowx : nullptr;
  const long long bcrow = ((long long)b * a.bc_groups + gbc) * N * (long long)L;
  sc.Bp = reinterpret_cast<const IO*>(a.B) + bcrow;
  sc.Cp = reinterpret_cast<const IO*>(a.C) + bcrow;
  sc.ch = ch;
  sc.lane = lane;
  sc.t_begin = chunk * a.chunk_len;
  sc.t_end = min(L, sc.t_begin + a.chunk_len);
  sc.nblk = (sc.t_end - sc.t_begin + kT - 1) / kT;
  sc.N = N;
  sc.L = L;
  sc.act = act;
  sc.bias = a.dt_bias ? a.dt_bias[dd] : 0.f;
  sc.Dd = (Scan::kOut && a.D) ? a.D[dd] : 0.f;

  // A (times log2 e on the bf16 path) and the initial state; missing states (n >= N) get A = 0,
  // B = C = 0 and stay zero
  const float ascale = kPrecise ? 1.f : kLog2e;
  const float* Ad = a.A + (long long)dd * N;
  float2 al[8], h[8];
  float amax = 0.f;
  const float* hsrc = nullptr;
  bool hs16 = false;
  if (MODE != kFwdSummary) {
    if (a.hin) {
      hsrc = a.hin + ((long long)chunk * a.batch * a.dim + ch) * kNS;
      hs16 = true;
    } else if (a.h0) {
      hsrc = a.h0 + ch * N;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int n0 = 2 * j, n1 = 2 * j + 1;
    al[j] = make_float2(n0 < N ? Ad[n0] * ascale : 0.f, n1 < N ? Ad[n1] * ascale : 0.f);
    amax = fmaxf(amax, fmaxf(fabsf(al[j].x), fabsf(al[j].y)));
    h[j] = make_float2((hsrc && (hs16 || n0 < N)) ? hsrc[n0] : 0.f,
                       (hsrc && (hs16 || n1 < N)) ? hsrc[n1] : 0.f);
  }
  // the FMA-pipe exponential needs |Δ A log2 e| <= 126: blocks whose largest |Δ| exceeds dlim
  // (in any lane) run every exponential on MUFU.  FLT_MAX when A is zero; 0 when A is infinite.
  const float dlim = amax > 0.f ? 126.f / amax : 3.402823466e38f;

  float dl[kT], du[kT], m = 0.f, dsum = 0.f;
  float acc = 0.f, comp = 0.f;  // Kahan-compensated ΣΔ of the chunk (summary pass)
  const auto kahan = [&](float x) {
    const float yk = x - comp;
    const float tk = acc + yk;
    comp = (tk - acc) - yk;
    acc = tk;
  };
  // prologue: blocks 0 .. kStages-2 in flight, block 0 staged
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) sc.issue(s);
  cp_wait<kStages - 2>();
  __syncwarp();
  sc.convert_bc(0, 0);
  sc.scalars(0, dl, du, m, dsum);
  __syncwarp();

#pragma unroll 1
  for (int i = 0; i < sc.nblk; ++i) {
    if (MODE == kFwdSummary) kahan(dsum);
    cp_wait<kStages - 3>();  // block i+1 has landed (this lane's copies)
    __syncwarp();            // ... and every other lane's
    if constexpr (kPrecise || (KE == 8 && KO == 8)) {
      sc.template body<8, 8>(i, h, al, dl, du, m, dsum);  // every exponential on MUFU: no vote
    } else {
      const bool fast = __all_sync(0xffffffffu, m <= dlim);
      if (fast) sc.template body<KE, KO>(i, h, al, dl, du, m, dsum);
      else sc.template body<8, 8>(i, h, al, dl, du, m, dsum);
    }
    __syncwarp();  // slot i-1 and B/C buffer i&1 are free for reuse
  }
  cp_wait<0>();

  if (MODE == kFwdSummary) {
    if (!act) return;
    float* sp = a.summ + ((long long)chunk * a.batch * a.dim + ch) * kNS;
    sc.store_state(sp, h, kNS);
    a.dsum[(long long)chunk * a.batch * a.dim + ch] = acc;
  } else if (sc.t_end == L && a.hL && act) {
    sc.store_state(a.hL + ch * N, h, N);
  }
}

template <typename IO, int MODE, int KE, int KO>
void launch_lane_one(const FwdArgs& a, cudaStream_t s) {
  const int nchunk_launch = MODE == kFwdSummary ? a.nchunk - 1 : a.nchunk;
  if (a.nwarps <= 0 || nchunk_launch <= 0) return;
  const size_t smem = Geo<IO>::kWarpBytes;
  auto k = fwd_lane_kernel<IO, MODE, KE, KO>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k<<<dim3((unsigned)a.nwarps, (unsigned)nchunk_launch), dim3(32), smem, s>>>(a);
}

}  // namespace lane
}  // namespace ssm
