// One-token recurrent (decode) step of the selective SSM, sm_100a.
//
// Generation runs the model as a recurrence that keeps only a fixed D x N state per layer and
// costs O(1) per token ("Mamba: ..." summary page, "Sorular": no KV cache during generation;
// mamba-minimal news page: recurrent mode for one-step-at-a-time inference).  Per channel
// c = (b, d):
//   Δ = softplus(dt + dt_bias_d);  h_n <- exp(Δ A_dn) h_n + Δ B_n x   (in place)
//   out = (Σ_n C_n h_n + D_d x) * silu(z)
//
// Variants (the same recurrence as the scan's): one decay rate A_d per channel (A is [dim]); the
// zero-order-hold input coefficient c = (e^{ΔA} - 1)/A (library expm1f: the step is memory-bound,
// so the accurate form costs nothing); B, C per group of channels ([batch][groups][N]).
//
// The step is bound by HBM traffic on the f32 state (read + write of batch*D*N*4 bytes).  For
// N = 16 two lanes share a channel, each holding 8 consecutive states as two 128-bit accesses
// (a warp streams 1 KB of contiguous state per access pair); the two partial readouts are
// combined with one shuffle.  Other N use four lanes of 4 states with per-element guards.
#include <stdlib.h>

#include <type_traits>

#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace {

template <typename IO> __device__ __forceinline__ float ld_io(const void* p, long long i);
template <> __device__ __forceinline__ float ld_io<float>(const void* p, long long i) {
  return reinterpret_cast<const float*>(p)[i];
}
template <> __device__ __forceinline__ float ld_io<uint16_t>(const void* p, long long i) {
  return bf16_to_f32(reinterpret_cast<const uint16_t*>(p)[i]);
}
template <typename IO> __device__ __forceinline__ void st_io(void* p, long long i, float v);
template <> __device__ __forceinline__ void st_io<float>(void* p, long long i, float v) {
  reinterpret_cast<float*>(p)[i] = v;
}
template <> __device__ __forceinline__ void st_io<uint16_t>(void* p, long long i, float v) {
  reinterpret_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
}

// SSM_DECODE_STREAM=0 selects the per-thread form of the N = 16 decode step instead of the
// streamed one (for measurements; both compute the same arithmetic).
// float4 state vectors per lane of the one-rate decode with more than 16 states (1, 2 or 4;
// SSM_DECODE_VECTORS overrides the default)
int decode_scalar_vectors() {
  const char* v = getenv("SSM_DECODE_VECTORS");
  const int n = v ? atoi(v) : 2;
  return (n == 1 || n == 2 || n == 4) ? n : 2;
}

bool getenv_stream_enabled() {
  const char* v = getenv("SSM_DECODE_STREAM");
  return !(v && v[0] == '0');
}

// Input coefficient of B x: Δ, or with the ZOH term (e^{ΔA} - 1)/A (Δ as A -> 0).
__device__ __forceinline__ float decode_coef(float dt, float An, bool zoh) {
  if (!zoh) return dt;
  return fabsf(An) < 1e-20f ? dt : expm1f(dt * An) / An;
}

// VEC: N == 16 and the state is 16-byte aligned (one float4 per lane).
template <typename IO, bool VEC>
__global__ void __launch_bounds__(256) decode_kernel(const DecodeArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  const long long nch = (long long)a.batch * a.dim;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool act = (gid >> 2) < nch;
  const long long ch = act ? (gid >> 2) : nch - 1;  // idle lanes shadow a valid channel
  const int q = (int)(gid & 3);
  const int b = (int)(ch / a.dim), d = (int)(ch % a.dim);
  const int N = a.N;

  const float xv = ld_io<IO>(a.x, ch);
  float v = ld_io<IO>(a.dt, ch) + (a.dt_bias ? a.dt_bias[d] : 0.f);
  const float dt = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
  const float dx = dt * xv;

  float h[4], An[4], Bn[4], Cn[4];
  float* sp = a.state + ch * N + 4 * q;
  const long long bc = ((long long)b * a.bc_groups + d / (a.dim / a.bc_groups)) * N;
  if (VEC) {
    const float4 h4 = *reinterpret_cast<const float4*>(sp);
    h[0] = h4.x; h[1] = h4.y; h[2] = h4.z; h[3] = h4.w;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = 4 * q + i;
    const bool live = n < N;
    if (!VEC) h[i] = live ? sp[i] : 0.f;
    // A times log2 e for the MUFU exponential (every decode form rounds the same product)
    An[i] = live ? a.A[a.scalar_a ? (long long)d : (long long)d * N + n] * ((kPrecise || a.zoh) ? 1.f : kLog2e)
                 : 0.f;
    Bn[i] = live ? ld_io<IO>(a.B, bc + n) : 0.f;
    Cn[i] = live ? ld_io<IO>(a.C, bc + n) : 0.f;
  }
  float y = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float abar = (kPrecise || a.zoh) ? expf(dt * An[i]) : ex2_mufu(dt * An[i]);
    const float bx = a.zoh ? decode_coef(dt, An[i], true) * xv : dx;
    h[i] = fmaf(abar, h[i], bx * Bn[i]);
    y = fmaf(Cn[i], h[i], y);
  }
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  y += __shfl_xor_sync(0xffffffffu, y, 2);
  if (!act) return;
  if (VEC) {
    *reinterpret_cast<float4*>(sp) = make_float4(h[0], h[1], h[2], h[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (4 * q + i < N) sp[i] = h[i];
  }
  if (q == 0) {
    y += (a.D ? a.D[d] : 0.f) * xv;
    if (a.z) {
      const float zv = ld_io<IO>(a.z, ch);
      y *= zv * (kPrecise ? sigmoid_precise(zv) : sigmoid_fast(zv));
    }
    st_io<IO>(a.out, ch, y);
  }
}

// One decay rate per channel with N = 32, 64 or 128 states (the state sizes of the scan's
// chunked matrix form): LPC lanes per channel, V x 4 states each (N = 4 V LPC), the state V
// 128-bit loads and stores per lane, all issued before the first is used.  With one rate per
// channel the decay and the input coefficient are formed once per lane (rounded as in the other
// decode forms); the readout is a shuffle reduction over the channel's lanes.
template <typename IO, int LPC, int V>
__global__ void __launch_bounds__(256) decode_scalar_kernel(const DecodeArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  constexpr int N = 4 * V * LPC;
  const long long nch = (long long)a.batch * a.dim;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool act = gid / LPC < nch;
  const long long ch = act ? gid / LPC : nch - 1;  // idle lanes shadow a valid channel
  const int q = (int)(gid % LPC);                    // states [4Vq, 4Vq + 4V)
  const int b = (int)(ch / a.dim), d = (int)(ch % a.dim);

  const float xv = ld_io<IO>(a.x, ch);
  const float v = ld_io<IO>(a.dt, ch) + (a.dt_bias ? a.dt_bias[d] : 0.f);
  const float dt = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
  const float An = a.A[d] * ((kPrecise || a.zoh) ? 1.f : kLog2e);
  const float abar = (kPrecise || a.zoh) ? expf(dt * An) : ex2_mufu(dt * An);
  const float bx = (a.zoh ? decode_coef(dt, An, true) : dt) * xv;

  float4* sp = reinterpret_cast<float4*>(a.state + ch * N) + V * q;
  float4 h[V];
#pragma unroll
  for (int k = 0; k < V; ++k) h[k] = sp[k];
  const long long bc = ((long long)b * a.bc_groups + d / (a.dim / a.bc_groups)) * N + 4 * V * q;
  float y = 0.f;
#pragma unroll
  for (int k = 0; k < V; ++k) {
    float* hk = reinterpret_cast<float*>(&h[k]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hk[i] = fmaf(abar, hk[i], bx * ld_io<IO>(a.B, bc + 4 * k + i));
      y = fmaf(ld_io<IO>(a.C, bc + 4 * k + i), hk[i], y);
    }
  }
#pragma unroll
  for (int m = 1; m < LPC; m <<= 1) y += __shfl_xor_sync(0xffffffffu, y, m);
  if (!act) return;
#pragma unroll
  for (int k = 0; k < V; ++k) sp[k] = h[k];
  if (q == 0) {
    y += (a.D ? a.D[d] : 0.f) * xv;
    if (a.z) {
      const float zv = ld_io<IO>(a.z, ch);
      y *= zv * (kPrecise ? sigmoid_precise(zv) : sigmoid_fast(zv));
    }
    st_io<IO>(a.out, ch, y);
  }
}

// N == 16 with 16-byte aligned tensors: two lanes per channel, 8 states each, every access a
// 128-bit load or store (state 2 x 16 B, A 2 x 16 B, B and C 16 B of bf16 or 2 x 16 B of f32).
template <typename IO>
__global__ void __launch_bounds__(256) decode16_kernel(const DecodeArgs a) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  const long long nch = (long long)a.batch * a.dim;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool act = (gid >> 1) < nch;
  const long long ch = act ? (gid >> 1) : nch - 1;  // idle lanes shadow a valid channel
  const int q = (int)(gid & 1);                      // states [8q, 8q + 8)
  const int b = (int)(ch / a.dim), d = (int)(ch % a.dim);

  const float xv = ld_io<IO>(a.x, ch);
  const float v = ld_io<IO>(a.dt, ch) + (a.dt_bias ? a.dt_bias[d] : 0.f);
  const float dt = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
  const float dx = dt * xv;

  float* sp = a.state + ch * kNS + 8 * q;
  const float4 h0 = reinterpret_cast<const float4*>(sp)[0];  // default caching: the state is
  const float4 h1 = reinterpret_cast<const float4*>(sp)[1];  // reused by the next step
  float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  // A times log2 e for the MUFU exponential (every decode form rounds the same product)
  const float ascale = (kPrecise || a.zoh) ? 1.f : kLog2e;
  float An[8];
  if (a.scalar_a) {
    const float ad = __ldg(a.A + d) * ascale;
#pragma unroll
    for (int i = 0; i < 8; ++i) An[i] = ad;
  } else {
    const float4* ap = reinterpret_cast<const float4*>(a.A + (long long)d * kNS + 8 * q);
    const float4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
    const float at[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) An[i] = at[i] * ascale;
  }
  const long long bc = ((long long)b * a.bc_groups + d / (a.dim / a.bc_groups)) * kNS + 8 * q;
  float Bn[8], Cn[8];
  if (sizeof(IO) == 2) {
    const uint4 bw = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.B) + bc));
    const uint4 cw = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.C) + bc));
    const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w}, cc[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      Bn[2 * i] = bf16_lo(bb[i]); Bn[2 * i + 1] = bf16_hi(bb[i]);
      Cn[2 * i] = bf16_lo(cc[i]); Cn[2 * i + 1] = bf16_hi(cc[i]);
    }
  } else {
    const float4* bp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.B) + bc);
    const float4* cp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.C) + bc);
    const float4 b0 = __ldg(bp), b1 = __ldg(bp + 1), c0 = __ldg(cp), c1 = __ldg(cp + 1);
    const float bt[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    const float ct[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) { Bn[i] = bt[i]; Cn[i] = ct[i]; }
  }
  float y = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float abar = (kPrecise || a.zoh) ? expf(dt * An[i]) : ex2_mufu(dt * An[i]);
    const float bx = a.zoh ? decode_coef(dt, An[i], true) * xv : dx;
    h[i] = fmaf(abar, h[i], bx * Bn[i]);
    y = fmaf(Cn[i], h[i], y);
  }
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  if (!act) return;
  reinterpret_cast<float4*>(sp)[0] = make_float4(h[0], h[1], h[2], h[3]);
  reinterpret_cast<float4*>(sp)[1] = make_float4(h[4], h[5], h[6], h[7]);
  if (q == 0) {
    y += (a.D ? a.D[d] : 0.f) * xv;
    if (a.z) {
      const float zv = ld_io<IO>(a.z, ch);
      y *= zv * (kPrecise ? sigmoid_precise(zv) : sigmoid_fast(zv));
    }
    st_io<IO>(a.out, ch, y);
  }
}

// ---------------------------------------------------------------- streamed form
// The state is the step's only large operand (batch x dim x 16 f32, read and written once).  A
// thread that loads its channel's 64 bytes and waits for them keeps few bytes in flight per
// SM.  Here persistent CTAs stream tiles of kTile consecutive channels through a kStages-deep
// shared-memory ring with bulk asynchronous copies (one cp.async.bulk per operand and tile,
// completing on the stage's mbarrier), so kStages tiles per CTA are in flight with no register
// cost.  A CTA keeps one block of kTile channels d and walks down the batch rows, so its rows of
// A (and D, dt_bias) are loaded once.  Every wait on an mbarrier is bounded: after kSpinLimit
// polls the kernel counts a timeout in g_wait_timeouts (read by ssm_wait_timeouts()), waits
// (bounded again) for the copies it issued, and returns.
constexpr int kTile = 128;                 // channels per tile (2 threads each)
constexpr int kStages = 4;
constexpr int kStreamThreads = 2 * kTile;
constexpr long long kSpinLimit = 1LL << 22;

__device__ unsigned int g_wait_timeouts = 0;

template <typename IO>
struct StreamStage {
  float state[kTile * kNS];
  IO x[kTile], dt[kTile], z[kTile];
  IO B[kNS], C[kNS];
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
// true when the phase with this parity has completed; false after kSpinLimit polls
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (long long i = 0; i < kSpinLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// bytes (a multiple of 16) from global src to shared dst (both 16-byte aligned), counted on bar
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

template <typename IO>
__global__ void __launch_bounds__(kStreamThreads) decode_stream_kernel(const __grid_constant__ DecodeArgs a,
                                                                       int rows_per_cta) {
  constexpr bool kPrecise = std::is_same<IO, float>::value;
  extern __shared__ float4 smem_dec[];
  StreamStage<IO>* st = reinterpret_cast<StreamStage<IO>*>(smem_dec);
  __shared__ __align__(8) uint64_t bars[kStages];
  const int tid = threadIdx.x;
  const int nblk_d = a.dim / kTile;
  const int dblk = blockIdx.x % nblk_d;
  const int b0 = (blockIdx.x / nblk_d) * rows_per_cta;
  const int nrows = min(rows_per_cta, a.batch - b0);
  if (nrows <= 0) return;
  const int d0 = dblk * kTile;
  const int gbc = d0 / (a.dim / a.bc_groups);  // the tile's channels share one B/C group
  const int cl = tid >> 1, q = tid & 1;        // channel in the tile, half of its states
  const int d = d0 + cl;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s]);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  const size_t es = sizeof(IO);
  const auto issue = [&](int r, int stage) {  // batch row b0 + r into stage
    StreamStage<IO>& sg = st[stage];
    const long long c0 = (long long)(b0 + r) * a.dim + d0;
    const uint32_t bytes = (uint32_t)(kTile * kNS * 4 + (a.z ? 3 : 2) * kTile * es + 2 * kNS * es);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    mbar_expect(&bars[stage], bytes);
    bulk_load(sg.state, a.state + c0 * kNS, kTile * kNS * 4, &bars[stage]);
    bulk_load(sg.x, reinterpret_cast<const IO*>(a.x) + c0, kTile * es, &bars[stage]);
    bulk_load(sg.dt, reinterpret_cast<const IO*>(a.dt) + c0, kTile * es, &bars[stage]);
    if (a.z) bulk_load(sg.z, reinterpret_cast<const IO*>(a.z) + c0, kTile * es, &bars[stage]);
    const long long bc = ((long long)(b0 + r) * a.bc_groups + gbc) * kNS;
    bulk_load(sg.B, reinterpret_cast<const IO*>(a.B) + bc, kNS * es, &bars[stage]);
    bulk_load(sg.C, reinterpret_cast<const IO*>(a.C) + bc, kNS * es, &bars[stage]);
  };
  if (tid == 0)
    for (int r = 0; r < kStages && r < nrows; ++r) issue(r, r);

  // per-channel parameters, once for every batch row of the CTA (A times log2 e for the MUFU
  // exponential of the bf16 path)
  const float ascale = (kPrecise || a.zoh) ? 1.f : kLog2e;
  float An[8];
  if (a.scalar_a) {
    const float ad = __ldg(a.A + d) * ascale;
#pragma unroll
    for (int i = 0; i < 8; ++i) An[i] = ad;
  } else {
    const float4* ap = reinterpret_cast<const float4*>(a.A + (long long)d * kNS + 8 * q);
    const float4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
    An[0] = a0.x * ascale; An[1] = a0.y * ascale; An[2] = a0.z * ascale; An[3] = a0.w * ascale;
    An[4] = a1.x * ascale; An[5] = a1.y * ascale; An[6] = a1.z * ascale; An[7] = a1.w * ascale;
  }
  const float bias = a.dt_bias ? a.dt_bias[d] : 0.f;
  const float Dd = a.D ? a.D[d] : 0.f;

  // one barrier per row: it carries every thread's "row r + 1 has landed" and marks the end of
  // every thread's reads of row r, after which row r's stage is refilled
  bool ok = __syncthreads_and(mbar_wait(&bars[0], 0u));
  int r = 0;
  for (; ok && r < nrows; ++r) {
    const int stage = r % kStages;
    const StreamStage<IO>& sg = st[stage];
    const float xv = ld_io<IO>(sg.x, cl);
    const float v = ld_io<IO>(sg.dt, cl) + bias;
    const float dt = !a.softplus ? v : (kPrecise ? softplus_precise(v) : softplus_fast(v));
    const float dx = dt * xv;
    // each thread's 8 states are 32 bytes, so threads 4 apart would read the same banks: those
    // with bit 2 set read their two halves in the other order
    const int sw = (tid >> 2) & 1;
    const float4* hp = reinterpret_cast<const float4*>(sg.state + cl * kNS + 8 * q);
    const float4 ha = hp[sw], hb = hp[sw ^ 1];
    const float4 h0 = sw ? hb : ha, h1 = sw ? ha : hb;
    float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    float Bn[8], Cn[8];
    if constexpr (sizeof(IO) == 2) {
      const uint4 bw = *reinterpret_cast<const uint4*>(sg.B + 8 * q);
      const uint4 cw = *reinterpret_cast<const uint4*>(sg.C + 8 * q);
      const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w}, cc[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        Bn[2 * i] = bf16_lo(bb[i]); Bn[2 * i + 1] = bf16_hi(bb[i]);
        Cn[2 * i] = bf16_lo(cc[i]); Cn[2 * i + 1] = bf16_hi(cc[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        Bn[i] = ld_io<IO>(sg.B, 8 * q + i);
        Cn[i] = ld_io<IO>(sg.C, 8 * q + i);
      }
    }
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float abar = (kPrecise || a.zoh) ? expf(dt * An[i]) : ex2_mufu(dt * An[i]);
      const float bx = a.zoh ? decode_coef(dt, An[i], true) * xv : dx;
      h[i] = fmaf(abar, h[i], bx * Bn[i]);
      y = fmaf(Cn[i], h[i], y);
    }
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    const float zv = a.z ? ld_io<IO>(sg.z, cl) : 0.f;
    const bool landed = r + 1 >= nrows || mbar_wait(&bars[(r + 1) % kStages], (uint32_t)(((r + 1) / kStages) & 1));
    ok = __syncthreads_and(landed);
    if (ok && tid == 0 && r + kStages < nrows) issue(r + kStages, stage);
    const long long ch = (long long)(b0 + r) * a.dim + d;
    float4* sp = reinterpret_cast<float4*>(a.state + ch * kNS + 8 * q);
    sp[0] = make_float4(h[0], h[1], h[2], h[3]);
    sp[1] = make_float4(h[4], h[5], h[6], h[7]);
    if (q == 0) {
      y += Dd * xv;
      if (a.z) y *= zv * (kPrecise ? sigmoid_precise(zv) : sigmoid_fast(zv));
      st_io<IO>(a.out, ch, y);
    }
  }
  if (!ok) {
    // a copy never completed: record it, wait (bounded) for the copies still in flight so none
    // lands after the CTA's shared memory is released, and stop.  Rows before the failed one
    // are complete; the failed row and the ones after it are not written.
    if (tid == 0) atomicAdd(&g_wait_timeouts, 1u);
    for (int rr = r; rr < nrows && rr < r + kStages; ++rr)  // r: the row that did not land
      mbar_wait(&bars[rr % kStages], (uint32_t)((rr / kStages) & 1));
  }
}

template <typename IO>
cudaError_t launch_stream(const DecodeArgs& a, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nblk_d = a.dim / kTile;
  // 2 to 4 resident CTAs per SM, each walking a run of batch rows; the run length is chosen so
  // that the CTAs spread evenly over the SMs
  int rows = a.batch, grid = nblk_d;
  double best = -1.0;
  for (int k = 2; k <= 4; ++k) {
    const int g = max(1, min(a.batch, (int)((double)k * sms / nblk_d + 0.5)));
    const int rw = (a.batch + g - 1) / g;
    const int ng = (a.batch + rw - 1) / rw;
    const int gr = nblk_d * ng;
    const double eff = (double)gr / ((double)sms * ((gr + sms - 1) / sms)) *
                       ((double)a.batch / ((double)ng * rw));
    if (eff > best) {
      best = eff;
      rows = rw;
      grid = gr;
    }
  }
  const size_t smem = kStages * sizeof(StreamStage<IO>);
  auto k = decode_stream_kernel<IO>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k<<<grid, kStreamThreads, smem, s>>>(a, rows);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const DecodeArgs& a, cudaStream_t s) {
  const int tpb = 256;
  const auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  // the streamed form: 16 states, whole tiles of channels inside one batch row and one B/C
  // group, every bulk copy 16-byte aligned and a multiple of 16 bytes
  const bool stream_ok = a.N == kNS && a.dim % kTile == 0 &&
                         (a.bc_groups == 1 || (a.dim / a.bc_groups) % kTile == 0) &&
                         al16(a.state) && (a.scalar_a || al16(a.A)) && al16(a.B) && al16(a.C) &&
                         al16(a.x) && al16(a.dt) && (a.z == nullptr || al16(a.z)) &&
                         kNS * sizeof(IO) % 16 == 0 && getenv_stream_enabled();
  if (stream_ok) return launch_stream<IO>(a, s);
  if (a.N > kNS) {  // one rate per channel, N = 32, 64 or 128, 16-byte aligned state (host-checked)
    const int V = decode_scalar_vectors();
    const long long threads = (long long)a.batch * a.dim * (a.N / (4 * V));
    const unsigned grid = (unsigned)((threads + tpb - 1) / tpb);
    if (V == 1) {
      switch (a.N) {
        case 32: decode_scalar_kernel<IO, 8, 1><<<grid, tpb, 0, s>>>(a); break;
        case 64: decode_scalar_kernel<IO, 16, 1><<<grid, tpb, 0, s>>>(a); break;
        case 128: decode_scalar_kernel<IO, 32, 1><<<grid, tpb, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
      }
    } else if (V == 2) {
      switch (a.N) {
        case 32: decode_scalar_kernel<IO, 4, 2><<<grid, tpb, 0, s>>>(a); break;
        case 64: decode_scalar_kernel<IO, 8, 2><<<grid, tpb, 0, s>>>(a); break;
        case 128: decode_scalar_kernel<IO, 16, 2><<<grid, tpb, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
      }
    } else {
      switch (a.N) {
        case 32: decode_scalar_kernel<IO, 2, 4><<<grid, tpb, 0, s>>>(a); break;
        case 64: decode_scalar_kernel<IO, 4, 4><<<grid, tpb, 0, s>>>(a); break;
        case 128: decode_scalar_kernel<IO, 8, 4><<<grid, tpb, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
      }
    }
    return cudaGetLastError();
  }
  if (a.N == kNS && al16(a.state) && (a.scalar_a || al16(a.A)) && al16(a.B) && al16(a.C)) {
    const long long threads = (long long)a.batch * a.dim * 2;
    decode16_kernel<IO><<<(unsigned)((threads + tpb - 1) / tpb), tpb, 0, s>>>(a);
  } else {
    const long long threads = (long long)a.batch * a.dim * 4;
    const unsigned grid = (unsigned)((threads + tpb - 1) / tpb);
    const bool vec = a.N == kNS && al16(a.state);
    if (vec) decode_kernel<IO, true><<<grid, tpb, 0, s>>>(a);
    else decode_kernel<IO, false><<<grid, tpb, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int io, cudaStream_t s) {
  return io == 1 ? launch_io<uint16_t>(a, s) : launch_io<float>(a, s);
}

int decode_wait_timeouts(unsigned int* out) {
  return cudaMemcpyFromSymbol(out, g_wait_timeouts, sizeof(unsigned int)) == cudaSuccess ? 0 : -1;
}

}  // namespace ssm
