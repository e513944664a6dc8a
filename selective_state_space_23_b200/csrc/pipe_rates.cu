// Throughput of the arithmetic pipes the scan kernels use, per SM and clock (sm_100a): FP32 FMA
// (scalar and packed f32x2) and the MUFU exponential.  These rates are the unit counts behind
// the forward kernel's arithmetic roofline.  Each thread runs 8 independent dependency chains of
// one instruction kind for `iters` rounds (enough resident warps to cover the latency); thread 0
// of each CTA records its SM and the SM clock (clock64) at start and end, and the rate of an SM
// is (instructions x lanes of the CTAs it ran) / (last end - first start on that SM).  Not part
// of the scan library: built as its own small shared library for this measurement.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kChains = 8;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// kind 0: scalar FFMA, 1: packed FFMA2 (counts 2 FP32 ops per lane), 2: MUFU ex2
template <int KIND>
__global__ void pipe_kernel(float* sink, int iters, long long* t) {
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
    t[3 * blockIdx.x] = t0;
    t[3 * blockIdx.x + 1] = clock64();
    t[3 * blockIdx.x + 2] = smid;
  }
}

}  // namespace

// Runs one pipe kind with `ctas_per_sm` CTAs of `threads` threads per SM; writes the mean over
// SMs of ops per SM per cycle (FP32 operations, FFMA2 counting 2 per lane, or exponentials) and
// returns 0, or a nonzero error code.
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
  if (cudaMalloc(&t, 3 * (size_t)ctas * sizeof(long long)) != cudaSuccess) return 2;
  for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
    if (kind == 0) pipe_kernel<0><<<ctas, threads>>>(sink, iters, t);
    else if (kind == 1) pipe_kernel<1><<<ctas, threads>>>(sink, iters, t);
    else pipe_kernel<2><<<ctas, threads>>>(sink, iters, t);
  }
  cudaError_t e = cudaDeviceSynchronize();
  long long* h = new long long[3 * (size_t)ctas];
  if (e == cudaSuccess) e = cudaMemcpy(h, t, 3 * (size_t)ctas * sizeof(long long), cudaMemcpyDeviceToHost);
  cudaFree(sink);
  cudaFree(t);
  if (e != cudaSuccess) {
    delete[] h;
    return (int)e;
  }
  const double ops_per_cta = (double)iters * 16 * kChains * threads * (kind == 1 ? 2 : 1);
  const int kMaxSm = 1024;
  long long first[kMaxSm], last[kMaxSm];
  int count[kMaxSm];
  for (int i = 0; i < kMaxSm; ++i) {
    first[i] = 0x7fffffffffffffffLL;
    last[i] = 0;
    count[i] = 0;
  }
  for (int i = 0; i < ctas; ++i) {
    const int sm = (int)h[3 * i + 2];
    if (sm < 0 || sm >= kMaxSm) continue;
    first[sm] = h[3 * i] < first[sm] ? h[3 * i] : first[sm];
    last[sm] = h[3 * i + 1] > last[sm] ? h[3 * i + 1] : last[sm];
    ++count[sm];
  }
  delete[] h;
  double sum = 0.0;
  int n = 0;
  for (int i = 0; i < kMaxSm; ++i)
    if (count[i] > 0 && last[i] > first[i]) {
      sum += count[i] * ops_per_cta / (double)(last[i] - first[i]);
      ++n;
    }
  if (n == 0) return 3;
  *rate_out = sum / n;
  return 0;
}
