// Forward selective scan (S6), sm_100a: dispatch over io type and direction, and the carry pass
// of the time split.  The kernels and their design notes are in ssm_fwd_impl.cuh.
#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {

cudaError_t launch_fwd_bf16(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu, cudaStream_t s);
cudaError_t launch_fwd_f32(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu, cudaStream_t s);
cudaError_t launch_fwd_rev_bf16(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu,
                                cudaStream_t s);
cudaError_t launch_fwd_rev_f32(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu,
                               cudaStream_t s);
cudaError_t launch_fwd_lane_bf16(const FwdArgs& a, int mode, int kmufu, cudaStream_t s);
cudaError_t launch_fwd_lane_f32(const FwdArgs& a, int mode, cudaStream_t s);

namespace {

// Chain the chunk summaries: h_in(0) = h0, h_in(j+1) = exp(A ΣΔ_j) h_in(j) + h_end(j).
// Each chunk j is the affine map h -> a_j h + b_j with a_j = exp(A ΣΔ_j), b_j = h_end(j) (its
// end state from zero); composing maps is associative, (a, b) after (a', b') =
// (a a', a b' + b) -- the parallel associative scan of the linear recurrence ("Temel Fikirler"
// and "Donanım Duyarlı Durum Genişletme" on the Mamba summary page).  One warp per
// (channel, state): the chunks are taken 32 at a time, one per lane, composed with a
// Kogge-Stone inclusive scan over warp shuffles, and applied to the state entering the group.
__global__ void fwd_carry_kernel(const FwdArgs a, const float* __restrict__ summ,
                                 const float* __restrict__ dsum, float* __restrict__ hin) {
  const long long nch = (long long)a.batch * a.dim;
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= nch * kNS) return;  // whole warps leave together
  const long long ch = wid / kNS;
  const int n = (int)(wid % kNS);
  const int d = (int)(ch % a.dim);
  const float An = n >= a.N ? 0.f : (a.scalar_a ? a.A[d] : a.A[(long long)d * a.N + n]);
  float carry = (a.h0 && n < a.N) ? a.h0[ch * a.N + n] : 0.f;  // h_in of the group's first chunk
  if (lane == 0) hin[ch * kNS + n] = carry;
  for (int g = 0; g < a.nchunk - 1; g += 32) {
    const int j = g + lane;  // chunk whose map this lane holds
    float ma = 1.f, mb = 0.f;  // identity past the last summarised chunk
    if (j < a.nchunk - 1) {
      ma = expf(An * dsum[(long long)j * nch + ch]);
      mb = summ[((long long)j * nch + ch) * kNS + n];
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float pa = __shfl_up_sync(0xffffffffu, ma, off);
      const float pb = __shfl_up_sync(0xffffffffu, mb, off);
      if (lane >= off) {  // this lane's maps after the earlier lanes' maps
        mb = fmaf(ma, pb, mb);
        ma = ma * pa;
      }
    }
    const float hj = fmaf(ma, carry, mb);  // state entering chunk j + 1
    if (j < a.nchunk - 1) hin[((long long)(j + 1) * nch + ch) * kNS + n] = hj;
    carry = __shfl_sync(0xffffffffu, hj, 31);
  }
}

}  // namespace

cudaError_t launch_fwd(const FwdArgs& a, int io, bool vec, int mode, int wpb, int kmufu,
                       cudaStream_t s) {
  // fp32: library expf for every state (the MUFU split does not apply)
  if (a.reverse)
    return io == 1 ? launch_fwd_rev_bf16(a, vec, mode, wpb, kmufu, s)
                   : launch_fwd_rev_f32(a, vec, mode, wpb, 16, s);
  return io == 1 ? launch_fwd_bf16(a, vec, mode, wpb, kmufu, s)
                 : launch_fwd_f32(a, vec, mode, wpb, 16, s);
}

cudaError_t launch_fwd_lane(const FwdArgs& a, int io, int mode, int kmufu, cudaStream_t s) {
  return io == 1 ? launch_fwd_lane_bf16(a, mode, kmufu, s) : launch_fwd_lane_f32(a, mode, s);
}

cudaError_t launch_fwd_carry(const FwdArgs& a, const float* summ, const float* dsum, float* hin,
                             cudaStream_t s) {
  const long long threads = (long long)a.batch * a.dim * kNS * 32;  // one warp per (channel, state)
  const int tpb = 256;
  fwd_carry_kernel<<<(unsigned)((threads + tpb - 1) / tpb), tpb, 0, s>>>(a, summ, dsum, hin);
  return cudaGetLastError();
}

}  // namespace ssm
