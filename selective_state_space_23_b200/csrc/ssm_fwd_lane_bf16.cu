// One-lane-per-channel forward kernels, bf16 io (the kernel is in ssm_fwd_lane.cuh; each io type
// is its own translation unit so that they compile in parallel).
#include "ssm_fwd_lane.cuh"

namespace ssm {

// kmufu: exponentials on the MUFU unit of every 16 (per pair of steps: KE + KO of the 16 state
// pairs), the rest on the FMA-pipe polynomial.
template <int MODE>
static void launch_bf16_mode(const FwdArgs& a, int kmufu, cudaStream_t s) {
  using IO = uint16_t;
  switch (kmufu) {
    case 16: lane::launch_lane_one<IO, MODE, 8, 8>(a, s); break;
    case 15: lane::launch_lane_one<IO, MODE, 8, 7>(a, s); break;
    case 13: lane::launch_lane_one<IO, MODE, 7, 6>(a, s); break;
    case 12: lane::launch_lane_one<IO, MODE, 6, 6>(a, s); break;
    case 11: lane::launch_lane_one<IO, MODE, 6, 5>(a, s); break;
    case 10: lane::launch_lane_one<IO, MODE, 5, 5>(a, s); break;
    default: lane::launch_lane_one<IO, MODE, 7, 7>(a, s); break;
  }
}

cudaError_t launch_fwd_lane_bf16(const FwdArgs& a, int mode, int kmufu, cudaStream_t s) {
  switch (mode) {
    case kFwdOut: launch_bf16_mode<kFwdOut>(a, kmufu, s); break;
    case kFwdSummary: launch_bf16_mode<kFwdSummary>(a, kmufu, s); break;
    default: launch_bf16_mode<kFwdCkpt>(a, kmufu, s); break;
  }
  return cudaGetLastError();
}

}  // namespace ssm
