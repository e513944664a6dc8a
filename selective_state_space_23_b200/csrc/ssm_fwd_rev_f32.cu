// Forward-scan kernels: fp32 io, reverse scan (the kernels themselves are in ssm_fwd_impl.cuh; each io type
// and direction is its own translation unit so that they compile in parallel).
#include "ssm_fwd_impl.cuh"

namespace ssm {

cudaError_t launch_fwd_rev_f32(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu, cudaStream_t s) {
  return vec ? launch_io<float, true, true>(a, mode, wpb, kmufu, s)
             : launch_io<float, false, true>(a, mode, wpb, kmufu, s);
}

}  // namespace ssm
