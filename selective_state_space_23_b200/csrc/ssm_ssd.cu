// Scalar-decay selective scan (N = 16, 32, 64, 128) in its chunked matrix form,
// on the tensor cores, sm_100a, bf16 io.
//
// With one decay rate A_d per channel (the Mamba-2 restriction noted on the "2024 Reading List:
// Neural Network" page, section on state-space models, where the scalar transition is what lets
// the state grow to N = 64..128), the scan h_t = e^{Δ_t A_d} h_{t-1} + Δ_t x_t B_t,
// y_t = C_t . h_t + D_d x_t, out_t = y_t silu(z_t) has, over a chunk of T = 16 steps with
// cumulative steps S_t = Σ_{r <= t} Δ_r (from the chunk start) and state h_in entering it,
//   y_t   = Σ_{s <= t} (C_t . B_s) e^{A (S_t - S_s)} Δ_s x_s  +  e^{A S_t} (C_t . h_in)  +  D x_t
//   h_out = e^{A S_{T-1}} h_in + Σ_s e^{A (S_{T-1} - S_s)} Δ_s x_s B_s,
// the masked-matrix ("state-space duality") form of the scan, whose products over states and
// steps are dense contractions.  Because A is a scalar per channel, the decay factor is rank one
// in (t, s) for each channel: e^{A (S_t - S_s)} = P_t Q_s with P_t = e^{A (S_t - S_m)} and
// Q_s = 1 / P_s about the chunk's middle step m.  With B, C shared by the channels of a batch
// row, a warp's 16 channels take per chunk four tensor-core products (bf16 in, f32 accumulate):
//   G   = C B^T                     [16 t x 16 s]   K = N    (masked to s <= t)
//   Y1' = X1' mask(G)^T              [16 d x 16 t]   K = 16,  X1'[d][s] = Q_s Δ_s x_s
//   Y2' = H' C^T                     [16 d x 16 t]   K = N,   H' = h_in transposed [d][n]
//                                    (H' as a bf16 pair plus its remainder: two products)
//   U'  = X2' B                      [16 d x N]      K = 16,  X2'[d][s] = e^{A (S_end - S_s)} Δ_s x_s
// and y = P Y1 + e^{A S_t} Y2 + D x,  H' <- e^{A S_end} H' + U'.
//
// B200 mapping (one warp = 16 channels, a CTA = W warps of one batch row and B/C group):
//   * the transposed state H' [16 d][N] lives in the warp's MMA accumulator registers (f32) for
//     the whole sequence: the U' product accumulates straight into it, and its accumulator
//     layout is also the A-operand layout of Y2' (packed to bf16), so the state never touches
//     shared memory;
//   * G's accumulators are, after the mask, the B operand of Y1' (no shared-memory round trip);
//   * the chunk's B, C tiles ([N][16 steps], as stored in HBM) stream into a 4-stage
//     shared-memory ring by cp.async and are read with ldmatrix (.trans where the product needs
//     them transposed): rows padded to 48 bytes, conflict-free; one CTA barrier per chunk;
//   * each lane's elementwise work covers exactly the (channel, step) pairs it holds in the
//     accumulators: channels g, g+8 and steps 2tg, 2tg+1, 2tg+8, 2tg+9 of the chunk
//     (g = lane / 4, tg = lane % 4); the cumulative steps S_t are a scan over the 4 lanes of a
//     quad (warp shuffles); u, delta, z are prefetched one chunk ahead into registers;
//   * P_t and Q_s grow as e^{|A| S} inside a chunk: a channel whose chunk would leave the safe
//     range (|A| |S_t - S_m| > 60 or |A| |S_t| > 80, or a non-finite step) takes no part in that
//     chunk's products (its inputs are zeroed, its state kept) and is computed for that chunk by
//     an exact sequential pass over its states held by the quad instead.
// The products are small (K = 16 or N per 16-step chunk) and carry the sequence's dependency from
// chunk to chunk, so they run as warp-level mma.sync.m16n8k16 rather than tcgen05 tiles.
//
// Time split (few channels, long sequences): segments of whole chunks run side by side.  A
// summary launch (MODE kSsdSummary) runs every segment but the last from a zero state, keeping
// only the state update (no G, Y1, Y2, gate or outputs), and writes its end state and ΣΔ; the
// host chains those segment maps (h -> e^{A ΣΔ} h + h_end) into each segment's entering state;
// the output launch then runs every segment from its entering state.
#include <stdint.h>
#include <stdlib.h>

#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"
#include "ssm_mma.cuh"

namespace ssm {
namespace {

using namespace ssd;

// u, delta, z of the lane's two channels and four steps of one chunk, as bf16 pairs:
// w[c][0] = steps 2tg, 2tg+1 and w[c][1] = steps 2tg+8, 2tg+9 of channel c.
struct ChunkIn {
  uint32_t u[2][2], dl[2][2], z[2][2];
};

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* p, long long t, int L, bool vec) {
  if (vec) return __ldg(reinterpret_cast<const uint32_t*>(p + t));
  const uint32_t lo = t < L ? (uint32_t)__ldg(p + t) : 0u;
  const uint32_t hi = t + 1 < L ? (uint32_t)__ldg(p + t + 1) : 0u;
  return lo | (hi << 16);
}

// The state entering chunk `slot` of the warp's 16 channels (transposed accumulator layout: 2
// channels x N/4 states per lane) into the checkpoint array, f32 [batch][dim][ceil(L / 16)][N]:
// the layout of the per-state scan's checkpoints, which hold the same states (the state
// entering every 16-step block), so either forward's checkpoints serve either backward.
// kStageCkpt<N>: the lanes' pairs go through the warp's staging tile (rows of N + 8 floats:
// conflict-free 64-bit writes and 128-bit reads), so that each channel's row leaves as whole
// 16-byte pieces of consecutive lanes rather than 8-byte pieces of 16 rows per store (1 x 256 x
// 2^20, N = 64: the backward's checkpoint pass 2 ms faster).  At N = 128 the tile would cost the
// kernel a resident CTA per SM, and the pairs are stored directly.
template <int N>
constexpr bool kStageCkpt = N <= 64;

template <int N>
__device__ __forceinline__ void store_state(const FwdArgs& a, const float (&Ht)[N / 8][4],
                                            float* stage, int slot, int b, int dw, int lane) {
  constexpr int LD = N + 8;
  const int g = lane >> 2, tg = lane & 3;
  const long long nslots = (a.L + kT - 1) / kT;
  if constexpr (!kStageCkpt<N>) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      if (dw + g + 8 * c >= a.dim) continue;
      float* row = a.ckpt + (((long long)b * a.dim + dw + g + 8 * c) * nslots + slot) * N + 2 * tg;
#pragma unroll
      for (int nt = 0; nt < N / 8; ++nt)
        *reinterpret_cast<float2*>(row + 8 * nt) = make_float2(Ht[nt][2 * c], Ht[nt][2 * c + 1]);
    }
    return;
  }
  __syncwarp();  // the previous chunk's rows have left the tile
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int nt = 0; nt < N / 8; ++nt)
      *reinterpret_cast<float2*>(stage + (g + 8 * c) * LD + 8 * nt + 2 * tg) =
          make_float2(Ht[nt][2 * c], Ht[nt][2 * c + 1]);
  __syncwarp();
#pragma unroll
  for (int i = lane; i < 16 * (N / 4); i += 32) {
    const int r = i / (N / 4), q = i % (N / 4);
    if (dw + r < a.dim)
      *reinterpret_cast<float4*>(a.ckpt + (((long long)b * a.dim + dw + r) * nslots + slot) * N + 4 * q) =
          *reinterpret_cast<const float4*>(stage + r * LD + 4 * q);
  }
}

// MODE: kSsdOut (gated outputs), kSsdOutCkpt (and the state entering every chunk into a.ckpt),
// kSsdSummary (segment end state and ΣΔ from zero), kSsdCkpt (only the state entering every
// chunk into a.ckpt, for the backward).  ZOH: the zero-order-hold input coefficient.  Both are
// template parameters so that the plain output kernel carries no code of the others.
template <int N, int W, int MODE, bool ZOH>
__global__ void __launch_bounds__(32 * W) ssd_fwd_kernel(const __grid_constant__ FwdArgs a) {
  constexpr bool SUMMARY = MODE == kSsdSummary;
  constexpr bool NOOUT = MODE == kSsdSummary || MODE == kSsdCkpt;  // no gate, readout or outputs
  constexpr bool CKPT = MODE == kSsdCkpt || MODE == kSsdOutCkpt;    // checkpoints written
  // states that a backward or a chain reads take the state update's remainder term too
  constexpr bool EXACT = MODE != kSsdOut;
  constexpr int kNT = N / 8;  // n8 tiles of the state
  extern __shared__ float4 smem_ssd[];
  SsdStage<N>* ring = reinterpret_cast<SsdStage<N>*>(smem_ssd);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // checkpoint modes: the warp's staging tile of 16 rows after the ring
  float* stage = reinterpret_cast<float*>(ring + kStages) +
                 ((CKPT && kStageCkpt<N>) ? warp * 16 * (N + 8) : 0);
  const int g = lane >> 2, tg = lane & 3;
  const int tiles_d = (a.dim + 16 * W - 1) / (16 * W);
  const int b = blockIdx.x / tiles_d;
  const int d0 = (blockIdx.x % tiles_d) * 16 * W;
  const int L = a.L;
  // this CTA's time segment: chunks [kc0, kc0 + nchunk) (the whole sequence without a split)
  const int seg = blockIdx.y;
  const int kc0 = seg * (a.chunk_len / kT);
  const int nchunk = (min(L, (seg + 1) * a.chunk_len) - kc0 * kT + kT - 1) / kT;
  const long long nch = (long long)a.batch * a.dim;
  const int gbc = d0 / (a.dim / a.bc_groups);
  const uint16_t* Bg = reinterpret_cast<const uint16_t*>(a.B) + ((long long)b * a.bc_groups + gbc) * N * (long long)L;
  const uint16_t* Cg = reinterpret_cast<const uint16_t*>(a.C) + ((long long)b * a.bc_groups + gbc) * N * (long long)L;

  // the lane's two channels (rows g and g + 8 of the warp's 16); idle ones shadow the last
  int dch[2];
  bool act[2];
  long long row[2];
  float al[2], bias[2], Dd[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int d = d0 + 16 * warp + g + 8 * c;
    act[c] = d < a.dim;
    dch[c] = act[c] ? d : a.dim - 1;
    row[c] = ((long long)b * a.dim + dch[c]) * L;
    al[c] = a.A[dch[c]] * kLog2e;
    bias[c] = a.dt_bias ? a.dt_bias[dch[c]] : 0.f;
    Dd[c] = a.D ? a.D[dch[c]] : 0.f;
  }
  const uint16_t* up = reinterpret_cast<const uint16_t*>(a.u);
  const uint16_t* dp = reinterpret_cast<const uint16_t*>(a.delta);
  const uint16_t* zp = reinterpret_cast<const uint16_t*>(a.z);
  uint16_t* op = reinterpret_cast<uint16_t*>(a.out);

  // the transposed state H'[d][n] in accumulator layout: Ht[nt][0..1] = channel g, states
  // 8 nt + 2 tg + {0, 1}; Ht[nt][2..3] = channel g + 8, same states
  // entering state: zero for a summary; the chained state of the segment with a split; else h0
  const float* hsrc = SUMMARY ? nullptr : (a.hin ? a.hin + (long long)seg * nch * N : a.h0);
  float Ht[kNT][4];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = e >> 1, n = 8 * nt + 2 * tg + (e & 1);
      Ht[nt][e] = hsrc ? hsrc[((long long)b * a.dim + dch[c]) * N + n] : 0.f;
    }
  }
  float dacc[2] = {0.f, 0.f}, dcmp[2] = {0.f, 0.f};  // ΣΔ of the segment (summary, Kahan)

  // B/C tiles of chunk k into ring slot k % kStages: 16-byte cp.async pieces when rows allow
  // them, else element loads (ragged tail, unaligned rows) with zeros past L
  const auto issue = [&](int k) {
    if (k < nchunk) {
      SsdStage<N>& st = ring[k % kStages];
      const int t0 = (kc0 + k) * kT;
      if (a.rows16 && t0 + kT <= L) {
        for (int p = tid; p < 4 * N; p += 32 * W) {
          const int which = p / (2 * N), rem = p % (2 * N), n = rem >> 1, h = rem & 1;
          const uint16_t* src = (which ? Cg : Bg) + (long long)n * L + t0 + 8 * h;
          uint16_t* dst = (which ? st.Cs : st.Bs) + n * kLdS + 8 * h;
          cp16(dst, src);
        }
      } else {
        for (int p = tid; p < 2 * N * kT; p += 32 * W) {
          const int which = p / (N * kT), rem = p % (N * kT), n = rem / kT, t = rem % kT;
          const uint16_t* src = (which ? Cg : Bg) + (long long)n * L + t0 + t;
          (which ? st.Cs : st.Bs)[n * kLdS + t] = t0 + t < L ? *src : (uint16_t)0;
        }
      }
    }
    cp_commit();
  };
  const bool vec_rows = a.rows16 != 0;
  const auto load_in = [&](int k, ChunkIn& in) {
    const int t0 = (kc0 + k) * kT;
    const bool vec = vec_rows && t0 + kT <= L;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const long long t = t0 + 2 * tg + 8 * hh;
        in.u[c][hh] = ld_pair(up + row[c], t, L, vec);
        in.dl[c][hh] = ld_pair(dp + row[c], t, L, vec);
        in.z[c][hh] = zp ? ld_pair(zp + row[c], t, L, vec) : 0u;
      }
    }
  };

#pragma unroll
  for (int k = 0; k < kStages - 1; ++k) issue(k);
  ChunkIn nxt;
  load_in(0, nxt);

  for (int k = 0; k < nchunk; ++k) {
    cp_wait<kStages - 2>();  // chunk k's B/C tiles have landed (this thread's copies)
    __syncthreads();         // ... every thread's; and every warp is done with chunk k - 1's slot
    issue(k + kStages - 1);  // into the slot chunk k - 1 used
    const ChunkIn cur = nxt;
    if (k + 1 < nchunk) load_in(k + 1, nxt);
    const SsdStage<N>& st = ring[k % kStages];
    const int t0 = (kc0 + k) * kT;
    if (CKPT) store_state<N>(a, Ht, stage, kc0 + k, b, d0 + 16 * warp, lane);

    // ---- per (channel, step): Δ, Δx, gate; index j: steps 2tg, 2tg+1, 2tg+8, 2tg+9
    float dl[2][4], xv[2][4], gt[2][4], uv[2][4];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t wu = cur.u[c][j >> 1], wd = cur.dl[c][j >> 1], wz = cur.z[c][j >> 1];
        const float u = (j & 1) ? bf16_hi(wu) : bf16_lo(wu);
        const float v = ((j & 1) ? bf16_hi(wd) : bf16_lo(wd)) + bias[c];
        const int t = t0 + 2 * tg + (j & 1) + 8 * (j >> 1);
        const bool live = t < L;
        const float D = a.softplus ? softplus_fast(v) : v;
        dl[c][j] = live ? D : 0.f;
        uv[c][j] = live ? u : 0.f;
        if constexpr (ZOH) xv[c][j] = zoh_c(dl[c][j], al[c] * kLn2) * uv[c][j];
        else xv[c][j] = dl[c][j] * uv[c][j];
        if (zp && !NOOUT) {
          const float z = (j & 1) ? bf16_hi(wz) : bf16_lo(wz);
          gt[c][j] = z * sigmoid_fast(z);
        } else {
          gt[c][j] = 1.f;
        }
      }
    }
    // ---- cumulative steps over the chunk: scans over the quad's lanes (lane tg holds the
    // pairs (2tg, 2tg+1) of the low and of the high 8 steps)
    float S[2][4], Sm[2], Se[2];
    bool fb[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float p = dl[c][0] + dl[c][1], q = dl[c][2] + dl[c][3];
      float ip = p, iq = q;
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        const float np = __shfl_up_sync(0xffffffffu, ip, off, 4);
        const float nq = __shfl_up_sync(0xffffffffu, iq, off, 4);
        if (tg >= off) {
          ip += np;
          iq += nq;
        }
      }
      const float lo_total = __shfl_sync(0xffffffffu, ip, 3, 4);
      const float hi_total = __shfl_sync(0xffffffffu, iq, 3, 4);
      S[c][0] = ip - p + dl[c][0];
      S[c][1] = ip;
      S[c][2] = lo_total + iq - q + dl[c][2];
      S[c][3] = lo_total + iq;
      Sm[c] = lo_total;  // S at step 7, the chunk's middle
      Se[c] = lo_total + hi_total;
      if (SUMMARY) {  // Kahan-compensated ΣΔ over the segment's chunks
        const float yk = Se[c] - dcmp[c];
        const float tk = dacc[c] + yk;
        dcmp[c] = (tk - dacc[c]) - yk;
        dacc[c] = tk;
      }
      float mrel = 0.f, mabs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mrel = fmaxf(mrel, fabsf(S[c][j] - Sm[c]));
        mabs = fmaxf(mabs, fabsf(S[c][j]));
      }
      // NaN-safe: a non-finite step fails the comparisons
      int ok = (fabsf(al[c]) * kLn2 * mrel <= 60.f && fabsf(al[c]) * kLn2 * mabs <= 80.f) ? 1 : 0;
      ok &= __shfl_xor_sync(0xffffffffu, ok, 1, 4);
      ok &= __shfl_xor_sync(0xffffffffu, ok, 2, 4);
      fb[c] = ok == 0;
    }
    // ---- decay factors and the scaled inputs (A operands of Y1' and U')
    float P[2][4], E[2][4], scale[2];
    uint32_t x1[4], x2[4];  // A fragments: {row g k lo, row g+8 k lo, row g k hi, row g+8 k hi}
    uint32_t x2l[4];        // the remainders of x2 (summary and checkpoint passes)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float eAm = ex2_mufu(Sm[c] * al[c]);
      const float eEm = ex2_mufu((Se[c] - Sm[c]) * al[c]);
      scale[c] = fb[c] ? 1.f : ex2_mufu(Se[c] * al[c]);
      float q1[4], q2[4];
#pragma unroll
      for (int j = 0; j < 4; j += 2) {  // packed f32x2 over step pairs
        const float2 r = mul2(add2(make_float2(S[c][j], S[c][j + 1]), f2(-Sm[c])), f2(al[c]));
        P[c][j] = ex2_mufu(r.x);
        P[c][j + 1] = ex2_mufu(r.y);
        const float2 e = mul2(f2(eAm), make_float2(P[c][j], P[c][j + 1]));
        E[c][j] = e.x;
        E[c][j + 1] = e.y;
        const float2 q = mul2(make_float2(ex2_mufu(-r.x), ex2_mufu(-r.y)),
                              make_float2(xv[c][j], xv[c][j + 1]));
        const float2 qq = mul2(f2(eEm), q);
        q1[j] = fb[c] ? 0.f : q.x;
        q1[j + 1] = fb[c] ? 0.f : q.y;
        q2[j] = fb[c] ? 0.f : qq.x;
        q2[j + 1] = fb[c] ? 0.f : qq.y;
      }
      x1[c] = pack_bf16x2(q1[0], q1[1]);
      x1[2 + c] = pack_bf16x2(q1[2], q1[3]);
      split_bf16x2(q2[0], q2[1], x2[c], x2l[c]);
      split_bf16x2(q2[2], q2[3], x2[2 + c], x2l[2 + c]);
    }

    // ---- G = C B^T and Y2' = H' C^T, sharing the C fragments of each 16-state k-step
    float G[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // s tiles 0..7, 8..15
    float Y2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // t tiles 0..7, 8..15
#pragma unroll
    for (int kk = 0; kk < (NOOUT ? 0 : N / 16); ++kk) {
      uint32_t cf[4], bf[4];
      ldsm_x4_t(cf, blk(st.Cs, 16 * kk, lane));  // {t0-7|n lo, t8-15|n lo, t0-7|n hi, t8-15|n hi}
      ldsm_x4_t(bf, blk(st.Bs, 16 * kk, lane));  // {s0-7|n lo, s8-15|n lo, s0-7|n hi, s8-15|n hi}
      mma16816(G[0], cf[0], cf[1], cf[2], cf[3], bf[0], bf[2]);
      mma16816(G[1], cf[0], cf[1], cf[2], cf[3], bf[1], bf[3]);
      // the f32 state as a bf16 pair plus its bf16 remainder: one bf16 operand would round h to
      // 8 bits, an error of 2^-9 |h| per state summed over N states in C . h_in
      uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
      split_bf16x2(Ht[2 * kk][0], Ht[2 * kk][1], h0, l0);
      split_bf16x2(Ht[2 * kk][2], Ht[2 * kk][3], h1, l1);
      split_bf16x2(Ht[2 * kk + 1][0], Ht[2 * kk + 1][1], h2, l2);
      split_bf16x2(Ht[2 * kk + 1][2], Ht[2 * kk + 1][3], h3, l3);
      mma16816(Y2[0], h0, h1, h2, h3, cf[0], cf[2]);
      mma16816(Y2[1], h0, h1, h2, h3, cf[1], cf[3]);
      mma16816(Y2[0], l0, l1, l2, l3, cf[0], cf[2]);
      mma16816(Y2[1], l0, l1, l2, l3, cf[1], cf[3]);
    }
    // ---- H' <- e^{A S_end} H' + X2' B   (fb channels: scale 1, zero inputs: unchanged)
#pragma unroll
    for (int nt = 0; nt < kNT; nt += 2) {
      uint32_t bn[4];
      ldsm_x4(bn, blk(st.Bs, 8 * nt, lane));  // {n tile nt: s lo, s hi; n tile nt+1: s lo, s hi}
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // packed f32x2: the two states of a channel share its scale
        const float2 sc = make_float2(scale[c], scale[c]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float2 h = mul2(make_float2(Ht[nt + u][2 * c], Ht[nt + u][2 * c + 1]), sc);
          Ht[nt + u][2 * c] = h.x;
          Ht[nt + u][2 * c + 1] = h.y;
        }
      }
      mma16816(Ht[nt], x2[0], x2[1], x2[2], x2[3], bn[0], bn[1]);
      mma16816(Ht[nt + 1], x2[0], x2[1], x2[2], x2[3], bn[2], bn[3]);
      if constexpr (EXACT) {  // states that a backward or a chain reads: the remainder term too
        mma16816(Ht[nt], x2l[0], x2l[1], x2l[2], x2l[3], bn[0], bn[1]);
        mma16816(Ht[nt + 1], x2l[0], x2l[1], x2l[2], x2l[3], bn[2], bn[3]);
      }
    }
    // ---- Y1' = X1' mask(G)^T: G's accumulators (rows t, cols s) are the B fragments
    // (k = s, n = t) once masked to s <= t
    float Y1[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (!NOOUT) {
      const int s0 = 2 * tg, r0 = g;
      const auto m = [](float v, int s, int t) { return s <= t ? v : 0.f; };
      // t tile 0: rows t = g; t tile 1: rows t = g + 8
      const uint32_t b00 = pack_bf16x2(m(G[0][0], s0, r0), m(G[0][1], s0 + 1, r0));
      const uint32_t b01 = pack_bf16x2(m(G[1][0], s0 + 8, r0), m(G[1][1], s0 + 9, r0));
      const uint32_t b10 = pack_bf16x2(m(G[0][2], s0, r0 + 8), m(G[0][3], s0 + 1, r0 + 8));
      const uint32_t b11 = pack_bf16x2(m(G[1][2], s0 + 8, r0 + 8), m(G[1][3], s0 + 9, r0 + 8));
      mma16816(Y1[0], x1[0], x1[1], x1[2], x1[3], b00, b01);
      mma16816(Y1[1], x1[0], x1[1], x1[2], x1[3], b10, b11);
    }
    // ---- outputs: y = P Y1 + e^{A S_t} Y2 + D x, gated.  Accumulator (tile T, e): channel
    // e / 2, step index j = 2 T + e % 2
    float yo[2][4];
#pragma unroll
    for (int T = 0; T < 2; ++T) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // packed f32x2 over the steps j = 2T, 2T + 1
        const int j = 2 * T;
        const float2 du = mul2(make_float2(Dd[c], Dd[c]), make_float2(uv[c][j], uv[c][j + 1]));
        const float2 y2 = fma2(make_float2(E[c][j], E[c][j + 1]),
                               make_float2(Y2[T][2 * c], Y2[T][2 * c + 1]), du);
        const float2 y = fma2(make_float2(P[c][j], P[c][j + 1]),
                              make_float2(Y1[T][2 * c], Y1[T][2 * c + 1]), y2);
        const float2 o = mul2(y, make_float2(gt[c][j], gt[c][j + 1]));
        yo[c][j] = o.x;
        yo[c][j + 1] = o.y;
      }
    }
    // ---- channels outside the factorisation's range this chunk: exact sequential pass over
    // the states the quad holds (rare; warp-uniform branch, per-channel predicates)
    if (__any_sync(0xffffffffu, fb[0] || fb[1])) {
      const int qb = lane & ~3;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int to = (t & 7) >> 1, jo = (t & 1) + 2 * (t >> 3);  // owner lane, its index
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float dt = __shfl_sync(0xffffffffu, dl[c][jo], qb | to);
          const float xt = __shfl_sync(0xffffffffu, xv[c][jo], qb | to);
          const float ab = ex2_mufu(dt * al[c]);
          float yp = 0.f;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int n = 8 * nt + 2 * tg + e;
              const float bv = bf16_to_f32(st.Bs[n * kLdS + t]);
              const float cv = bf16_to_f32(st.Cs[n * kLdS + t]);
              float& h = Ht[nt][2 * c + e];
              if (fb[c]) h = fmaf(ab, h, xt * bv);
              yp = fmaf(cv, h, yp);
            }
          }
          if (NOOUT) continue;
          yp += __shfl_xor_sync(0xffffffffu, yp, 1);
          yp += __shfl_xor_sync(0xffffffffu, yp, 2);
          if (fb[c] && tg == to) yo[c][jo] = fmaf(Dd[c], uv[c][jo], yp) * gt[c][jo];
        }
      }
    }
    // ---- store the chunk's outputs (bf16 pairs of steps)
#pragma unroll
    for (int c = 0; c < (NOOUT ? 0 : 2); ++c) {
      if (!act[c]) continue;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const long long t = t0 + 2 * tg + 8 * hh;
        const uint32_t w = pack_bf16x2(yo[c][2 * hh], yo[c][2 * hh + 1]);
        if (vec_rows && t0 + kT <= L) {
          *reinterpret_cast<uint32_t*>(op + row[c] + t) = w;
        } else {
          if (t < L) op[row[c] + t] = (uint16_t)(w & 0xffffu);
          if (t + 1 < L) op[row[c] + t + 1] = (uint16_t)(w >> 16);
        }
      }
    }
  }
  cp_wait<0>();
  if (MODE == kSsdCkpt) return;
  if (SUMMARY) {
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = e >> 1, n = 8 * nt + 2 * tg + (e & 1);
        if (act[c]) a.summ[((long long)seg * nch + (long long)b * a.dim + dch[c]) * N + n] = Ht[nt][e];
      }
    }
#pragma unroll
    for (int c = 0; c < 2; ++c)
      if (act[c] && tg == 0) a.dsum[(long long)seg * nch + (long long)b * a.dim + dch[c]] = dacc[c];
    return;
  }
  if (a.hL && (seg + 1) * a.chunk_len >= L) {
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = e >> 1, n = 8 * nt + 2 * tg + (e & 1);
        if (act[c]) a.hL[((long long)b * a.dim + dch[c]) * N + n] = Ht[nt][e];
      }
    }
  }
}

template <int N, int W>
cudaError_t launch_n(const FwdArgs& a, int mode, cudaStream_t s) {
  const int segs = mode == kSsdSummary ? a.nchunk - 1 : a.nchunk;  // the last summary is unused
  if (segs <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((long long)a.batch * ((a.dim + 16 * W - 1) / (16 * W))), (unsigned)segs);
  if (mode == kSsdOut && a.ckpt) mode = kSsdOutCkpt;
  const size_t smem =
      kStages * sizeof(SsdStage<N>) +
      ((kStageCkpt<N> && (mode == kSsdCkpt || mode == kSsdOutCkpt)) ? (size_t)W * 16 * (N + 8) * 4 : 0);
  const auto pick = [&](auto zoh) {
    constexpr bool Z = decltype(zoh)::value;
    return mode == kSsdSummary ? ssd_fwd_kernel<N, W, kSsdSummary, Z>
         : mode == kSsdCkpt    ? ssd_fwd_kernel<N, W, kSsdCkpt, Z>
         : mode == kSsdOutCkpt ? ssd_fwd_kernel<N, W, kSsdOutCkpt, Z>
                               : ssd_fwd_kernel<N, W, kSsdOut, Z>;
  };
  auto k = a.zoh ? pick(std::true_type()) : pick(std::false_type());
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, 32 * W, smem, s>>>(a);
  return cudaGetLastError();
}

template <int N>
cudaError_t launch_w(const FwdArgs& a, int mode, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 2 warps per CTA (32 channels) when 64-channel CTAs would leave fewer than 2 per SM
  // (SSM_SSD_WPB=2 or 4 forces the choice)
  const long long ctas4 = (long long)a.batch * ((a.dim + 63) / 64);
  bool two = ctas4 < 2LL * sms;
  const char* env = getenv("SSM_SSD_WPB");
  if (env && (atoi(env) == 2 || atoi(env) == 4)) two = atoi(env) == 2;
  return two ? launch_n<N, 2>(a, mode, s) : launch_n<N, 4>(a, mode, s);
}

}  // namespace

cudaError_t launch_ssd_fwd(const FwdArgs& a, int mode, cudaStream_t s) {
  switch (a.N) {
    case 16: return launch_w<16>(a, mode, s);
    case 32: return launch_w<32>(a, mode, s);
    case 64: return launch_w<64>(a, mode, s);
    case 128: return launch_w<128>(a, mode, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ssm
