// Forward-scan kernels: bf16 io, forward direction (the kernels themselves are in ssm_fwd_impl.cuh; each io type
// and direction is its own translation unit so that they compile in parallel).
#include "ssm_fwd_impl.cuh"

namespace ssm {

cudaError_t launch_fwd_bf16(const FwdArgs& a, bool vec, int mode, int wpb, int kmufu, cudaStream_t s) {
  return vec ? launch_io<uint16_t, true, false>(a, mode, wpb, kmufu, s)
             : launch_io<uint16_t, false, false>(a, mode, wpb, kmufu, s);
}

}  // namespace ssm
