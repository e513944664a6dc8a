// One-lane-per-channel forward kernels, fp32 io (library expf for every state, so there is no
// exponential split).  The kernel is in ssm_fwd_lane.cuh.
#include "ssm_fwd_lane.cuh"

namespace ssm {

cudaError_t launch_fwd_lane_f32(const FwdArgs& a, int mode, cudaStream_t s) {
  switch (mode) {
    case kFwdOut: lane::launch_lane_one<float, kFwdOut, 8, 8>(a, s); break;
    case kFwdSummary: lane::launch_lane_one<float, kFwdSummary, 8, 8>(a, s); break;
    default: lane::launch_lane_one<float, kFwdCkpt, 8, 8>(a, s); break;
  }
  return cudaGetLastError();
}

}  // namespace ssm
