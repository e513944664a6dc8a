// Backward pass of the default scan variant with the state history in registers, sm_100a.
//
// What is computed is the backward of ssm_bwd.cu (the chain rule through the forward recurrence;
// the pages only say that the states are recomputed in the backward pass, "Mamba: ..." summary
// page, "Donanım Duyarlı Durum Genişletme"):
//   g_t = dout_t silu(z_t);  λ_t = g_t C_t + Ā_{t+1} λ_{t+1}  (λ_{L-1} = g_{L-1} C_{L-1} + dhL)
//   du_t = g_t D + Δ_t Σ_n λ_t B_t;  dΔ_t = Σ_n λ_t (A Ā_t h_{t-1} + B_t x_t)
//   dB_t = Σ_d λ_t Δ_t x_t;  dC_t = Σ_d g_t h_t;  dA = Σ_{b,t} λ_t Δ_t Ā_t h_{t-1}
//   dD = Σ g_t x_t;  ddt_bias = Σ ddelta_t;  dz_t = dout_t y_t silu'(z_t);  dh0 = Ā_0 λ_0
// with Ā_t h_{t-1} = h_t - Δ_t B_t x_t.  This kernel serves the default variant (per-state decay,
// Euler input term, forward direction, [batch][dim][L] rows that allow 16-byte copies, N = 16);
// every other variant runs in ssm_bwd.cu.
//
// B200 mapping:
//   * two lanes own one channel (8 states each), a warp holds 16 channels of one batch row, a CTA
//     W warps.  Time is walked backwards in 16-step blocks, each in two halves: the lanes replay
//     the block forward from its checkpoint and keep the half's 8 states x 8 steps in REGISTERS,
//     then run the adjoint backwards over the half, recomputing Ā_t;
//   * the lane's rows (u, delta, z, dout), the warp's B/C tile and the checkpoint of the next
//     (earlier) block are copied by cp.async while the current block runs;
//   * per-step scalars (Δ, Δx, g, dout silu'(z)) are computed once per (channel, step) by the lane
//     that owns the step and shared through a per-warp table; the two lanes' partial sums over
//     their states (Σ λB, Σ A λ Ā h, C.h) are combined with one shuffle;
//   * dB, dC (sums over channels) are reduced over the warp's 16 channels with a shuffle
//     butterfly: lanes whose channel slot has bit 3 set hold their 8 states rotated by 4, so the
//     butterfly's first level (8 of its 15 shuffles) needs no selects; the CTA's warps are then
//     added in shared memory in a fixed order and written as one partial per (CTA, b, n, t),
//     which the finishing kernel of ssm_bwd.cu sums in a fixed order (bitwise reproducible);
//   * 16.6 KB of shared memory per warp (the step outputs reuse the step scalars' slots), so a
//     CTA of 4 warps leaves room for 3 per SM: the 320 CTAs of a 4 x 5120-channel row set run
//     in one wave.
#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace {

constexpr int kCW = 16;                   // channels per warp
constexpr int kBCS = kBlk * kNS + 16;     // f32 B/C tile [step][state], steps 8..15 shifted
__device__ __forceinline__ int bco(int k) { return k * kNS + (k >= 8 ? 16 : 0); }
// Per-step table [step][channel slot] (float4), steps 8..15 one bank group further on: the two
// lanes of a channel write and read the rows of steps j and 8 + j together, and rows 8 apart
// would otherwise share their banks.
constexpr int kTbl = kBlk * kCW + 4;
__device__ __forceinline__ int tbo(int k) { return k * kCW + (k >= 8 ? 4 : 0); }

template <typename IO>
struct HGeo {
  static constexpr int kES = (int)sizeof(IO);
  static constexpr int kSeg = 8 * kES;                 // one lane's 8 steps of one row
  static constexpr int kRowsBytes = 4 * 32 * kSeg;     // u, delta, z, dout: [tensor][lane][8]
  static constexpr int kRawBytes = 2 * kNS * kBlk * kES;  // B, C: [which][state][16 steps]
  static constexpr int kCkBytes = 32 * 32;             // checkpoint: [lane][8 states] f32
  static constexpr int kSlotBytes = kRowsBytes + kRawBytes + kCkBytes;
  static constexpr int kWarpBytes = 2 * kSlotBytes          // ring: this block and the next
                                    + 2 * kBCS * 4          // B/C tile as f32
                                    + kTbl * 16             // per-step scalars, then outputs
                                    + kBlk * 32 * 4;        // dB/dC warp sums of the block
};

// 16 bytes from global to shared; src_bytes < 16 zero-fills the rest (0: nothing is read).
__device__ __forceinline__ void cp16(void* smem, const void* gmem, int src_bytes = 16) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all_but1() {
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}

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

// The lane's 8 states of one step of a B or C tile, in the lane's (rotated) state order.
__device__ __forceinline__ void quads(const float* row, int qlo, int qhi, float2 (&v)[4]) {
  const float4 lo = *reinterpret_cast<const float4*>(row + qlo);
  const float4 hi = *reinterpret_cast<const float4*>(row + qhi);
  v[0] = make_float2(lo.x, lo.y);
  v[1] = make_float2(lo.z, lo.w);
  v[2] = make_float2(hi.x, hi.y);
  v[3] = make_float2(hi.z, hi.w);
}

// 2^(d * al) of one state pair: MUFU for pairs below KP, else the FMA-pipe polynomial (callers
// run KP < 4 only in range-checked blocks); PRECISE: library expf (al = A).
template <bool PRECISE, int KP>
__device__ __forceinline__ float2 exp_pair(int jj, float2 d2, float2 al) {
  if (PRECISE) return make_float2(expf(d2.x * al.x), expf(d2.x * al.y));
  if (jj < KP) {
    const float2 x = mul2(d2, al);
    return make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
  }
  return exp2_fma_prod_x2(d2, al);
}

template <typename IO, int W>
struct HistBwd {
  using G = HGeo<IO>;
  static constexpr bool kPrecise = std::is_same<IO, float>::value;

  const BwdArgs& a;
  unsigned char* wsm;  // this warp's shared memory
  int lane, s, q, rot, b, d0w, gbc, L, nblk;
  long long ch;
  bool act;
  int qlo, qhi;        // offsets of the lane's two state quads in a B/C tile row

  __device__ __forceinline__ unsigned char* slot(int blk) const {
    return wsm + (blk & 1) * G::kSlotBytes;
  }
  __device__ __forceinline__ float* bcf() const {
    return reinterpret_cast<float*>(wsm + 2 * G::kSlotBytes);
  }
  __device__ __forceinline__ float4* table() const {
    return reinterpret_cast<float4*>(wsm + 2 * G::kSlotBytes + 2 * kBCS * 4);
  }
  // the outputs of step k replace its scalars once both lanes of the channel have read them
  __device__ __forceinline__ float4* outs() const { return table(); }
  __device__ __forceinline__ float* red() const {
    return reinterpret_cast<float*>(table() + kTbl);
  }

  // Copies of block blk: the lane's 8 steps (8 q ..) of its channel's u, delta, z, dout; its
  // piece of the warp's B/C tile (state lane/2, steps 8 (lane & 1) ..); and its 8 checkpointed
  // states.  Each lane later reads only its own row pieces.
  __device__ __forceinline__ void issue(int blk) const {
    if (blk >= 0) {
      unsigned char* sl = slot(blk);
      // the last block may hold only its lower 8 steps (rows are whole 8-step pieces): the
      // upper half's pieces are then zero-filled from an in-bounds address and never used
      const long long t = (long long)blk * kBlk + 8 * q;
      const bool have = t < L;
      const long long row = ch * (long long)L + (have ? t : 0);
      const int nb = have ? 16 : 0;
      const void* src[4] = {reinterpret_cast<const IO*>(a.u) + row,
                            reinterpret_cast<const IO*>(a.delta) + row,
                            a.z ? reinterpret_cast<const IO*>(a.z) + row : nullptr,
                            reinterpret_cast<const IO*>(a.dout) + row};
#pragma unroll
      for (int tsr = 0; tsr < 4; ++tsr) {
        if (!src[tsr]) continue;
#pragma unroll
        for (int c = 0; c < G::kSeg / 16; ++c)
          cp16(sl + (tsr * 32 + lane) * G::kSeg + c * 16,
               reinterpret_cast<const unsigned char*>(src[tsr]) + (have ? c * 16 : 0), nb);
      }
      const int n = lane >> 1, hh = lane & 1;
      const long long tb = (long long)blk * kBlk + 8 * hh;
      const bool have_bc = tb < L;
      const long long bcrow = (((long long)b * a.bc_groups + gbc) * kNS + n) * L +
                              (have_bc ? tb : 0);
      const int nbc = have_bc ? 16 : 0;
      unsigned char* raw = sl + G::kRowsBytes;
#pragma unroll
      for (int c = 0; c < G::kSeg / 16; ++c) {
        const int off = have_bc ? c * 16 : 0;
        cp16(raw + (n * kBlk + 8 * hh) * G::kES + c * 16,
             reinterpret_cast<const unsigned char*>(reinterpret_cast<const IO*>(a.B) + bcrow) + off, nbc);
        cp16(raw + ((kNS + n) * kBlk + 8 * hh) * G::kES + c * 16,
             reinterpret_cast<const unsigned char*>(reinterpret_cast<const IO*>(a.C) + bcrow) + off, nbc);
      }
      const float* ck = a.ckpt + (ch * nblk + blk) * kNS + 8 * q;
      // halves swapped for lanes with bit 2 set: lanes 4 apart then use different bank groups
      unsigned char* cks = sl + G::kRowsBytes + G::kRawBytes + lane * 32;
      const int sw = (lane >> 2) & 1;
      cp16(cks + 16 * sw, ck);
      cp16(cks + 16 * (1 - sw), ck + 4);
    }
    cp_commit();
  }

  // B/C tile of block blk to f32 [step][state] (lane: state lane/2, steps 8 (lane & 1) ..).
  __device__ __forceinline__ void convert_bc(int blk) const {
    const unsigned char* raw = slot(blk) + G::kRowsBytes;
    float* t = bcf();
    const int n = lane >> 1, hh = lane & 1;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      float v[8];
      unpack8<IO>(raw + ((which * kNS + n) * kBlk + 8 * hh) * G::kES, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) t[which * kBCS + bco(8 * hh + j) + n] = v[j];
    }
  }

  // The checkpointed state entering block blk, in the lane's rotated order.
  __device__ __forceinline__ void entry_state(int blk, float2 (&h)[4]) const {
    const float* ck = reinterpret_cast<const float*>(slot(blk) + G::kRowsBytes + G::kRawBytes + lane * 32);
    const int sw = (lane >> 2) & 1;  // the halves as issue() placed them
    const float4 lo = *reinterpret_cast<const float4*>(ck + 4 * (rot ^ sw));
    const float4 hi = *reinterpret_cast<const float4*>(ck + 4 * ((1 - rot) ^ sw));
    h[0] = make_float2(lo.x, lo.y);
    h[1] = make_float2(lo.z, lo.w);
    h[2] = make_float2(hi.x, hi.y);
    h[3] = make_float2(hi.z, hi.w);
  }

  // One replayed step k: h <- Ā h + Δx B.
  template <int KP>
  __device__ __forceinline__ void replay(int k, float2 (&h)[4], const float2 (&al)[4]) const {
    const float4 sc = table()[tbo(k) + s];
    float2 bq[4];
    quads(bcf() + bco(k), qlo, qhi, bq);
    const float2 d2 = f2(sc.x), du2 = f2(sc.y);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      h[jj] = fma2(exp_pair<kPrecise, KP>(jj, d2, al[jj]), h[jj], mul2(du2, bq[jj]));
  }

  // One adjoint step k of the half owned by lane q == half; hk = h_k.
  template <int KP>
  __device__ __forceinline__ void adjoint(int k, int half, const float2 (&hk)[4], float2 (&lam)[4],
                                          float2 (&dA)[4], const float2 (&al)[4], float uk,
                                          float svk, float Dd, float live, float& dD_acc,
                                          float& db_acc) const {
    const float4 sc = table()[tbo(k) + s];  // (Δ, Δx, g, dout silu'(z))
    float2 bq[4], cq[4];
    quads(bcf() + bco(k), qlo, qhi, bq);
    quads(bcf() + kBCS + bco(k), qlo, qhi, cq);
    const float2 d2 = f2(sc.x), g2 = f2(sc.z), ndu2 = f2(-sc.y);
    const float2 dul = f2(sc.y * live), gl = f2(sc.z * live);
    float2 S1 = make_float2(0.f, 0.f), S2 = S1, Y = S1;
    float v[16];  // dB contributions (local states 0..7), then dC
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      lam[jj] = fma2(g2, cq[jj], lam[jj]);          // λ_t complete
      const float2 xv = fma2(ndu2, bq[jj], hk[jj]);  // Ā_t h_{t-1} = h_t - Δx B
      const float2 qv = mul2(lam[jj], xv);
      S2 = fma2(al[jj], qv, S2);
      dA[jj] = fma2(d2, qv, dA[jj]);
      S1 = fma2(lam[jj], bq[jj], S1);
      Y = fma2(cq[jj], hk[jj], Y);
      const float2 vb = mul2(lam[jj], dul), vc = mul2(gl, hk[jj]);
      v[2 * jj] = vb.x; v[2 * jj + 1] = vb.y;
      v[8 + 2 * jj] = vc.x; v[8 + 2 * jj + 1] = vc.y;
      lam[jj] = mul2(exp_pair<kPrecise, KP>(jj, d2, al[jj]), lam[jj]);  // Ā_t λ_t for step t-1
    }
    float s1 = S1.x + S1.y, s2 = S2.x + S2.y, y = Y.x + Y.y;
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    __syncwarp();  // both lanes of the channel have read the scalars of step k
    if (q == half) {
      const float aback = kPrecise ? 1.f : kLn2;  // al * aback = A
      const float du = fmaf(sc.z, Dd, sc.x * s1);
      const float dd = fmaf(uk, s1, s2 * aback);
      const float ddl = a.softplus ? dd * svk : dd;
      const float dz = sc.w * fmaf(Dd, uk, y);
      dD_acc = fmaf(sc.z * live, uk, dD_acc);
      db_acc = fmaf(live, ddl, db_acc);
      outs()[tbo(k) + s] = make_float4(du, ddl, dz, 0.f);
    }
    // dB, dC over the warp's 16 channels (lane bits 1..4 = channel slot bits 0..3)
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // slot bit 3: partners hold the same states rotated by 4
      v[i] += __shfl_xor_sync(0xffffffffu, v[i + 4], 16);
      v[8 + i] += __shfl_xor_sync(0xffffffffu, v[12 + i], 16);
    }
    const bool b2 = (s >> 2) & 1, b1 = (s >> 1) & 1, b0 = s & 1;
#pragma unroll
    for (int i = 0; i < 2; ++i) {  // slot bit 2: keep local states 2 b2 + {0, 1}
#pragma unroll
      for (int w8 = 0; w8 < 16; w8 += 8) {
        const float keep = b2 ? v[w8 + i + 2] : v[w8 + i];
        const float send = b2 ? v[w8 + i] : v[w8 + i + 2];
        v[w8 + i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
    }
#pragma unroll
    for (int w8 = 0; w8 < 16; w8 += 8) {  // slot bit 1: keep local state 2 b2 + b1
      const float keep = b1 ? v[w8 + 1] : v[w8];
      const float send = b1 ? v[w8] : v[w8 + 1];
      v[w8] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    // slot bit 0: keep dB (b0 = 0) or dC (b0 = 1)
    const float keep = b0 ? v[8] : v[0];
    const float send = b0 ? v[0] : v[8];
    const float tot = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    const int n = 8 * q + ((2 * (int)b2 + (int)b1 + 4 * rot) & 7);
    red()[k * 32 + (int)b0 * 16 + n] = tot;
  }

  int blkcur;
};

template <typename IO, int W, int KP>
__device__ __forceinline__ void half_pass(HistBwd<IO, W>& hb, int half, const float2 (&al)[4],
                                          float2 (&lam)[4], float2 (&dA)[4], const float (&uo)[8],
                                          const float (&svo)[8], float Dd, float live,
                                          float& dD_acc, float& db_acc) {
  const int lo = 8 * half;
  float2 h[4];
  hb.entry_state(hb.blkcur, h);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (half == 1) hb.template replay<KP>(k, h, al);  // steps below the half: state only
  float2 hist[8][4];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    hb.template replay<KP>(lo + k, h, al);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) hist[k][jj] = h[jj];
  }
#pragma unroll
  for (int k = 7; k >= 0; --k)
    hb.template adjoint<KP>(lo + k, half, hist[k], lam, dA, al, uo[k], svo[k], Dd, live, dD_acc,
                            db_acc);
}

template <typename IO, int W, int KP>
__global__ void __launch_bounds__(32 * W) bwd_hist_kernel(const __grid_constant__ BwdArgs a) {
  using G = HGeo<IO>;
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  extern __shared__ float4 smem_bh[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int b = blockIdx.x / a.ngroups, grp = blockIdx.x % a.ngroups;
  HistBwd<IO, W> hb{a};
  hb.wsm = reinterpret_cast<unsigned char*>(smem_bh) + (size_t)wib * G::kWarpBytes;
  hb.lane = lane;
  hb.s = lane >> 1;
  hb.q = lane & 1;
  hb.rot = (hb.s >> 3) & 1;
  hb.b = b;
  hb.d0w = (grp * W + wib) * kCW;
  // the warp's B/C group; a warp wholly past dim (last CTA of a row) shadows the last channel's
  hb.gbc = min(hb.d0w, a.dim - 1) / (a.dim / a.bc_groups);
  const int d = hb.d0w + hb.s;
  hb.act = d < a.dim;
  const int dd = hb.act ? d : a.dim - 1;
  hb.ch = (long long)b * a.dim + dd;
  hb.L = a.L;
  hb.nblk = (a.L + kBlk - 1) / kBlk;
  // time split: this CTA walks the blocks of chunk blockIdx.y only
  const int chunk = blockIdx.y;
  const bool split = a.nsplit > 1;
  const int blk_lo = split ? chunk * a.blk_per_chunk : 0;
  const int blk_hi = split ? min(hb.nblk, blk_lo + a.blk_per_chunk) : hb.nblk;
  const long long nch = (long long)a.batch * a.dim;
  // the adjoint entering the chunk from later time (dhL for the last chunk, or none)
  const float* lam0 = split ? a.lam_in + (long long)(a.nsplit - 1 - chunk) * nch * kNS : a.dhL;
  hb.qlo = 8 * hb.q + 4 * hb.rot;
  hb.qhi = 8 * hb.q + 4 * (1 - hb.rot);
  const float live = hb.act ? 1.f : 0.f;  // idle lanes add nothing to the channel sums
  const int q = hb.q, rot = hb.rot;

  // per-state parameters in the lane's rotated order: local state j <-> 8 q + ((j + 4 rot) & 7)
  const float ascale = kPrecise ? 1.f : kLog2e;
  float2 al[4], lam[4], dA[4];
  float amax = 0.f;
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int n0 = 8 * q + ((2 * jj + 4 * rot) & 7);
    al[jj] = make_float2(a.A[(long long)dd * kNS + n0] * ascale, a.A[(long long)dd * kNS + n0 + 1] * ascale);
    lam[jj] = lam0 ? make_float2(lam0[hb.ch * kNS + n0], lam0[hb.ch * kNS + n0 + 1])
                   : make_float2(0.f, 0.f);
    dA[jj] = make_float2(0.f, 0.f);
    amax = fmaxf(amax, fmaxf(fabsf(al[jj].x), fabsf(al[jj].y)));
  }
  const float Dd = a.D ? a.D[dd] : 0.f;
  const float bias = a.dt_bias ? a.dt_bias[dd] : 0.f;
  float dD_acc = 0.f, db_acc = 0.f;
  const float* redw0 = reinterpret_cast<const float*>(reinterpret_cast<unsigned char*>(smem_bh));

  hb.issue(blk_hi - 1);
  for (int blk = blk_hi - 1; blk >= blk_lo; --blk) {
    hb.blkcur = blk;
    hb.issue(blk > blk_lo ? blk - 1 : -1);  // the next (earlier) block's copies run meanwhile
    cp_wait_all_but1();  // this block's copies have landed
    __syncwarp();
    hb.convert_bc(blk);
    // per-step scalars of the lane's 8 steps (8 q ..)
    const int t0 = blk * kBlk;
    const int nvalid = min(kBlk, a.L - t0);
    float uo[8], svo[8];
    float dabs = 0.f;
    {
      const unsigned char* sl = hb.slot(blk);
      float uv[8], dv[8], zv[8], gv[8];
      unpack8<IO>(sl + (0 * 32 + lane) * G::kSeg, uv);
      unpack8<IO>(sl + (1 * 32 + lane) * G::kSeg, dv);
      if (a.z) unpack8<IO>(sl + (2 * 32 + lane) * G::kSeg, zv);
      unpack8<IO>(sl + (3 * 32 + lane) * G::kSeg, gv);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 v = add2(make_float2(dv[j], dv[j + 1]), f2(bias));
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
        const float2 xv = make_float2(uv[j], uv[j + 1]);
        const float2 dx = mul2(dl, xv);
        const float2 go = make_float2(gv[j], gv[j + 1]);
        float2 g = go, zf = make_float2(0.f, 0.f);
        if (a.z) {
          const float2 z2 = make_float2(zv[j], zv[j + 1]);
          const float2 sg = kPrecise ? make_float2(sigmoid_precise(z2.x), sigmoid_precise(z2.y))
                                     : sigmoid_fast_x2(z2);
          g = mul2(go, mul2(z2, sg));
          // silu'(z) = σ(z) (1 + z (1 - σ(z)))
          zf = mul2(mul2(go, sg), fma2(z2, add2(f2(1.f), mul2(sg, f2(-1.f))), f2(1.f)));
        }
        hb.table()[tbo(8 * q + j) + hb.s] = make_float4(dl.x, dx.x, g.x, zf.x);
        hb.table()[tbo(8 * q + j + 1) + hb.s] = make_float4(dl.y, dx.y, g.y, zf.y);
        uo[j] = xv.x; uo[j + 1] = xv.y;
        svo[j] = sp.x; svo[j + 1] = sp.y;
        dabs = fmaxf(dabs, fmaxf(fabsf(dl.x), fabsf(dl.y)));
        if (dl.x != dl.x || dl.y != dl.y) dabs = __int_as_float(0x7f800000);
      }
    }
    __syncwarp();  // tables and the B/C tile are complete
    // the polynomial exponential needs |Δ A log2 e| <= 126 in every lane of the block
    const bool safe = !kPrecise && !__any_sync(0xffffffffu, !(amax * dabs <= 126.f));
    for (int half = 1; half >= 0; --half) {
      if (8 * half >= nvalid) continue;  // rows are whole 8-step pieces: a half is all or nothing
      if (safe) half_pass<IO, W, KP>(hb, half, al, lam, dA, uo, svo, Dd, live, dD_acc, db_acc);
      else half_pass<IO, W, 4>(hb, half, al, lam, dA, uo, svo, Dd, live, dD_acc, db_acc);
    }
    __syncwarp();
    // du, ddelta, dz of the lane's 8 steps (8 q ..)
    if (hb.act && 8 * q < nvalid) {
      float odu[8], odd[8], odz[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 o = hb.outs()[tbo(8 * q + j) + hb.s];
        odu[j] = o.x; odd[j] = o.y; odz[j] = o.z;
      }
      const long long row = hb.ch * (long long)a.L + t0 + 8 * q;
      const auto put = [&](void* base, const float (&v)[8]) {
        IO* p = reinterpret_cast<IO*>(base) + row;
        if constexpr (sizeof(IO) == 2) {
          __stcs(reinterpret_cast<uint4*>(p),
                 make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7])));
        } else {
          __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
          __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
        }
      };
      if (a.du) put(a.du, odu);
      if (a.ddelta) put(a.ddelta, odd);
      if (a.dz && a.z) put(a.dz, odz);
    }
    // the CTA partial of dB, dC: add the W warps' sums in a fixed order
    __syncthreads();
    for (int p = threadIdx.x; p < 32 * 4; p += 32 * W) {
      const int e = p & 31, tq = p >> 5;  // value (which * 16 + n), steps 4 tq .. 4 tq + 3
      if (4 * tq >= nvalid) continue;
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const float* rw = reinterpret_cast<const float*>(
            reinterpret_cast<const unsigned char*>(redw0) + (size_t)w * G::kWarpBytes +
            2 * G::kSlotBytes + 2 * kBCS * 4 + kTbl * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[i] += rw[(4 * tq + i) * 32 + e];
      }
      const int which = e >> 4, n = e & 15;
      const long long prow = ((long long)(grp * a.batch + b) * 2 + which) * kNS + n;
      *reinterpret_cast<float4*>(a.part_bc + prow * a.L + t0 + 4 * tq) =
          make_float4(sum[0], sum[1], sum[2], sum[3]);
    }
    __syncthreads();  // the warps' sums are read before the next block writes them again
  }

  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  db_acc += __shfl_xor_sync(0xffffffffu, db_acc, 1);
  if (!hb.act) return;
  float* pa = a.part_adt + ((long long)(split ? chunk : 0) * nch + hb.ch) * (kNS + 2);
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int n0 = 8 * q + ((2 * jj + 4 * rot) & 7);
    if (a.dh0 && chunk == 0) {
      a.dh0[hb.ch * kNS + n0] = lam[jj].x;
      a.dh0[hb.ch * kNS + n0 + 1] = lam[jj].y;
    }
    pa[n0] = dA[jj].x;  // Σ λ Δ Ā h_{t-1}: no A factor, so no log2(e) rescale
    pa[n0 + 1] = dA[jj].y;
  }
  if (q == 0) {
    pa[kNS] = dD_acc;
    pa[kNS + 1] = db_acc;
  }
}

// 8 consecutive steps of a row from global memory (16-byte aligned).
template <typename IO>
__device__ __forceinline__ void load8(const IO* p, float (&v)[8]) {
  if constexpr (sizeof(IO) == 2) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Adjoint summary of chunk c >= 1 of a time-split backward.  The adjoint recurrence is linear in
// what enters a chunk from later time: if μ_in enters at the chunk's end, the adjoint leaving its
// first step is exp(A ΣΔ) μ_in + m, where m is what leaves when nothing enters.  This kernel walks
// the chunk backwards from zero (λ <- g_t C_t + λ, then λ <- Ā_t λ, as the history backward does)
// to get m, and sums Δ over the chunk (Kahan-compensated); the forward carry pass then chains the
// chunks' maps from the last chunk to the first, starting from dhL.  Two threads per channel (8
// states each); rows are read in 8-step pieces.
template <typename IO>
__global__ void __launch_bounds__(128) bwd_summary_kernel(const __grid_constant__ BwdArgs a,
                                                          float* __restrict__ summ,
                                                          float* __restrict__ dsum) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  const long long nch = (long long)a.batch * a.dim;
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long ch = tid >> 1;
  const int q = (int)(tid & 1);
  if (ch >= nch) return;
  const int chunk = blockIdx.y + 1;
  const long long slot = a.nsplit - 1 - chunk;
  const int b = (int)(ch / a.dim), d = (int)(ch % a.dim);
  const int gbc = d / (a.dim / a.bc_groups);
  const float ascale = kPrecise ? 1.f : kLog2e;
  float al[8], lam[8];
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    al[n] = a.A[(long long)d * kNS + 8 * q + n] * ascale;
    lam[n] = 0.f;
  }
  const float bias = a.dt_bias ? a.dt_bias[d] : 0.f;
  const long long L = a.L;
  const int t_lo = chunk * a.blk_per_chunk * kBlk;
  const int t_hi = min(a.L, t_lo + a.blk_per_chunk * kBlk);  // L % 8 == 0: whole 8-step pieces
  const IO* dp = reinterpret_cast<const IO*>(a.delta) + ch * L;
  const IO* zp = a.z ? reinterpret_cast<const IO*>(a.z) + ch * L : nullptr;
  const IO* gp = reinterpret_cast<const IO*>(a.dout) + ch * L;
  const IO* cp = reinterpret_cast<const IO*>(a.C) + (((long long)b * a.bc_groups + gbc) * kNS + 8 * q) * L;
  float dsm = 0.f, dcomp = 0.f;
  for (int t0 = t_hi - 8; t0 >= t_lo; t0 -= 8) {
    float dv[8], zv[8], gv[8], cv[8][8];
    load8<IO>(dp + t0, dv);
    if (zp) load8<IO>(zp + t0, zv);
    load8<IO>(gp + t0, gv);
#pragma unroll
    for (int n = 0; n < 8; ++n) load8<IO>(cp + n * L + t0, cv[n]);
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      const float v = dv[j] + bias;
      const float dl = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
      float g = gv[j];
      if (zp) {
        const float sg = kPrecise ? sigmoid_precise(zv[j]) : sigmoid_fast(zv[j]);
        g = g * (zv[j] * sg);
      }
      const float yk = dl - dcomp;  // Kahan step
      const float tk = dsm + yk;
      dcomp = (tk - dsm) - yk;
      dsm = tk;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        lam[n] = fmaf(g, cv[n][j], lam[n]);
        lam[n] *= kPrecise ? expf(dl * al[n]) : ex2_mufu(dl * al[n]);
      }
    }
  }
  float* o = summ + (slot * nch + ch) * kNS + 8 * q;
#pragma unroll
  for (int n = 0; n < 8; ++n) o[n] = lam[n];
  if (q == 0) dsum[slot * nch + ch] = dsm;
}

template <typename IO, int W>
cudaError_t launch_hist_io(const BwdArgs& a, cudaStream_t s) {
  const dim3 grid((unsigned)(a.batch * a.ngroups), (unsigned)(a.nsplit > 1 ? a.nsplit : 1)),
      block(32 * W);
  const size_t smem = (size_t)W * HGeo<IO>::kWarpBytes;
  auto k = bwd_hist_kernel<IO, W, 4>;
  if constexpr (!std::is_same<IO, float>::value) {
    if (a.kmufu == 3) k = bwd_hist_kernel<IO, W, 3>;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, block, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_hist(const BwdArgs& a, int io, cudaStream_t s) {
  if (a.wpb == 2) return io == 1 ? launch_hist_io<uint16_t, 2>(a, s) : launch_hist_io<float, 2>(a, s);
  return io == 1 ? launch_hist_io<uint16_t, 4>(a, s) : launch_hist_io<float, 4>(a, s);
}

// Warps per CTA for this shape: 4 (fewer dB/dC partials) when all CTAs are resident at once,
// else 2 when that makes them all resident, else 4.
template <typename IO>
int pick_wpb_io(int batch, int dim) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int wpr = (dim + kCW - 1) / kCW;
  int occ4 = 0, occ2 = 0;
  auto k4 = bwd_hist_kernel<IO, 4, 4>;
  auto k2 = bwd_hist_kernel<IO, 2, 4>;
  const size_t s4 = 4 * (size_t)HGeo<IO>::kWarpBytes, s2 = 2 * (size_t)HGeo<IO>::kWarpBytes;
  if (cudaFuncSetAttribute(k4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s4) != cudaSuccess ||
      cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ4, k4, 128, s4) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, k2, 64, s2) != cudaSuccess) {
    cudaGetLastError();
    return 4;
  }
  const long long ctas4 = (long long)batch * ((wpr + 3) / 4), ctas2 = (long long)batch * ((wpr + 1) / 2);
  if (ctas4 <= (long long)occ4 * sms) return 4;
  if (ctas2 <= (long long)occ2 * sms) return 2;
  return 4;
}

int bwd_hist_pick_wpb(int io, int batch, int dim) {
  return io == 1 ? pick_wpb_io<uint16_t>(batch, dim) : pick_wpb_io<float>(batch, dim);
}

namespace {
template <typename IO>
int ctas_per_sm_io(int wpb) {
  int occ = 0;
  const size_t smem = (size_t)wpb * HGeo<IO>::kWarpBytes;
  auto k = wpb == 2 ? bwd_hist_kernel<IO, 2, 4> : bwd_hist_kernel<IO, 4, 4>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, 32 * wpb, smem) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  return occ < 1 ? 1 : occ;
}
}  // namespace

int bwd_hist_ctas_per_sm(int io, int wpb) {
  return io == 1 ? ctas_per_sm_io<uint16_t>(wpb) : ctas_per_sm_io<float>(wpb);
}

cudaError_t launch_bwd_summary(const BwdArgs& a, int io, float* summ, float* dsum, cudaStream_t s) {
  if (a.nsplit <= 1) return cudaSuccess;
  const long long threads = 2LL * a.batch * a.dim;
  const dim3 grid((unsigned)((threads + 127) / 128), (unsigned)(a.nsplit - 1)), block(128);
  if (io == 1) bwd_summary_kernel<uint16_t><<<grid, block, 0, s>>>(a, summ, dsum);
  else bwd_summary_kernel<float><<<grid, block, 0, s>>>(a, summ, dsum);
  return cudaGetLastError();
}

}  // namespace ssm
