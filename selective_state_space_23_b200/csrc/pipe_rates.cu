// Throughput of the arithmetic pipes the scan kernels use, per SM and clock (sm_100a): FP32 FMA
// (scalar and packed f32x2) and the MUFU exponential.  These rates are the unit counts behind
// the forward kernel's arithmetic roofline.  Each thread runs 8 independent dependency chains of
// one instruction kind for `iters` rounds (enough resident warps to cover the latency); thread 0
// of each CTA records its SM, the SM clock (clock64) and the global nanosecond timer at start and
// end, and the rate of an SM is (instructions x lanes of the CTAs it ran) / (last end - first
// start on that SM), per clock and per nanosecond; their ratio is the clock the SM ran at.  Not
// part of the scan library: built as its own small shared library for this measurement.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kChains = 8;

__device__ __forceinline__ long long global_ns() {
  unsigned long long v;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(v));
  return (long long)v;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// kind 0: scalar FFMA, 1: packed FFMA2 (counts 2 FP32 ops per lane), 2: MUFU ex2
template <int KIND>
__global__ void pipe_kernel(float* sink, int iters, long long* t) {
  const long long g0 = global_ns();
  const long long t0 = clock64();
  float a[kChains];
  float2 p[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) {
    a[i] = 1e-3f * (threadIdx.x + i);
    p[i] = make_float2(a[i], -a[i]);
  }
  const float m = 0.999f, c = 1e-4f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) {
        if (KIND == 0) a[i] = fmaf(a[i], m, c);
        else if (KIND == 1) p[i] = __ffma2_rn(p[i], make_float2(m, m), make_float2(c, c));
        else a[i] = ex2_approx(-a[i]);
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += a[i] + p[i].x + p[i].y;
  if (s == 12345.f) sink[threadIdx.x] = s;  // keeps the chains alive
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    const long long t1 = clock64();
    t[5 * blockIdx.x] = t0;
    t[5 * blockIdx.x + 1] = t1;
    t[5 * blockIdx.x + 2] = smid;
    t[5 * blockIdx.x + 3] = g0;
    t[5 * blockIdx.x + 4] = global_ns();
  }
}

}  // namespace

// Runs one pipe kind with `ctas_per_sm` CTAs of `threads` threads per SM; writes the mean over
// SMs of ops per SM per SM-clock cycle (FP32 operations, FFMA2 counting 2 per lane, or
// exponentials) to rate_out[0], the same per nanosecond to rate_out[1] and the mean SM clock in
// MHz (clock64 ticks per microsecond) to rate_out[2]; returns 0, or a nonzero error code.
extern "C" __attribute__((visibility("default"))) int ssm_pipe_probe(int kind, int iters,
                                                                      int ctas_per_sm, int threads,
                                                                      double* rate_out) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
  const int ctas = sms * ctas_per_sm;
  float* sink = nullptr;
  long long* t = nullptr;
  if (cudaMalloc(&sink, threads * sizeof(float)) != cudaSuccess) return 2;
  if (cudaMalloc(&t, 5 * (size_t)ctas * sizeof(long long)) != cudaSuccess) return 2;
  for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
    if (kind == 0) pipe_kernel<0><<<ctas, threads>>>(sink, iters, t);
    else if (kind == 1) pipe_kernel<1><<<ctas, threads>>>(sink, iters, t);
    else pipe_kernel<2><<<ctas, threads>>>(sink, iters, t);
  }
  cudaError_t e = cudaDeviceSynchronize();
  long long* h = new long long[5 * (size_t)ctas];
  if (e == cudaSuccess) e = cudaMemcpy(h, t, 5 * (size_t)ctas * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaFree(sink);
  cudaFree(t);
  if (e != cudaSuccess) {
    delete[] h;
    return (int)e;
  }
  const double ops_per_cta = (double)iters * 16 * kChains * threads * (kind == 1 ? 2 : 1);
  const int kMaxSm = 1024;
  static long long first[kMaxSm], last[kMaxSm], gfirst[kMaxSm], glast[kMaxSm];
  static int count[kMaxSm];
  for (int i = 0; i < kMaxSm; ++i) {
    first[i] = gfirst[i] = 0x7fffffffffffffffLL;
    last[i] = glast[i] = 0;
    count[i] = 0;
  }
  for (int i = 0; i < ctas; ++i) {
    const long long* r = h + 5 * (size_t)i;
    const int sm = (int)r[2];
    if (sm < 0 || sm >= kMaxSm) continue;
    first[sm] = r[0] < first[sm] ? r[0] : first[sm];
    last[sm] = r[1] > last[sm] ? r[1] : last[sm];
    gfirst[sm] = r[3] < gfirst[sm] ? r[3] : gfirst[sm];
    glast[sm] = r[4] > glast[sm] ? r[4] : glast[sm];
    ++count[sm];
  }
  delete[] h;
  double per_clk = 0.0, per_ns = 0.0, mhz = 0.0;
  int n = 0;
  for (int i = 0; i < kMaxSm; ++i)
    if (count[i] > 0 && last[i] > first[i] && glast[i] > gfirst[i]) {
      per_clk += count[i] * ops_per_cta / (double)(last[i] - first[i]);
      per_ns += count[i] * ops_per_cta / (double)(glast[i] - gfirst[i]);
      mhz += 1e3 * (double)(last[i] - first[i]) / (double)(glast[i] - gfirst[i]);
      ++n;
    }
  if (n == 0) return 3;
  rate_out[0] = per_clk / n;
  rate_out[1] = per_ns / n;
  rate_out[2] = mhz / n;
  return 0;
}
