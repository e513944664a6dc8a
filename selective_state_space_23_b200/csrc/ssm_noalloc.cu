// Forward scan for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a serving process that reserved
// all device memory for its own pool when it started and forbids any further cudaMalloc, a
// plugin that runs inside a host application which owns every allocation, or code that must
// not call cudaMalloc/cudaFree on its hot path because those calls can synchronise the whole
// device and stall work on other streams.  For them, ssm_scan_fwd_noalloc runs the same
// forward kernels as ssm_scan_fwd, taking the time-split scratch (per-chunk end states, step
// sums and entering states) from one statically sized array in device memory that is part of
// the library image instead of from a caller workspace.
//
// The array is a file-scope __device__ variable: every GPU on which the library is loaded holds
// SSM_NOALLOC_SCRATCH_BYTES of it until the process exits, and every call on that GPU shares
// it.  Its contents survive from one call to the next; each call writes every scratch word it
// later reads before reading it, so nothing needs clearing.  Two calls whose work overlaps on
// the GPU (different streams, or different host threads) race on the array.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_fwd_scratch[SSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};
void* g_scratch_ctx[kMaxDevices] = {nullptr};

// cuCtxGetCurrent, reached through the runtime so that the library does not link libcuda.
typedef int (*PFN_ctxGetCurrent)(void**);
PFN_ctxGetCurrent ctx_get_current_fn() {
  static PFN_ctxGetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_ctxGetCurrent>(p);
    cudaGetLastError();
  });
  return fn;
}

void* current_context() {
  void* ctx = nullptr;
  PFN_ctxGetCurrent fn = ctx_get_current_fn();
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device.  In host code the symbol name is
// only a host-side handle, so the address is looked up with that device current.  It is cached
// per device together with the context it belongs to: if the context changes (after
// cudaDeviceReset, for instance, the module is loaded again and the array may move), or if the
// context cannot be identified, the address is looked up again.
int scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "ssm_scan_fwd_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
    ssm::set_last_error(msg);
    return SSM_ECUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    ssm::set_last_error("ssm_scan_fwd_noalloc: device index out of range");
    return SSM_EUNSUPPORTED;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  void* ctx = current_context();
  if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess || !p) {
      char msg[256];
      snprintf(msg, sizeof(msg), "ssm_scan_fwd_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      ssm::set_last_error(msg);
      g_scratch_addr[dev] = nullptr;
      return SSM_ECUDA;
    }
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context();  // the lookup made the device's context current
  }
  *out = g_scratch_addr[dev];
  return SSM_OK;
}

}  // namespace

extern "C" SSM_API int ssm_scan_fwd_noalloc(const void* u, const void* delta, const float* A,
                                            const void* B, const void* C, const float* D,
                                            const void* z, const float* dt_bias,
                                            int delta_softplus, const float* h0, float* hL,
                                            void* out, float* ckpt, int batch, int dim,
                                            int seqlen, int dstate, int io_dtype, void* stream) {
  const size_t need = ssm_scan_fwd_workspace_size(batch, dim, seqlen, dstate, io_dtype);
  if (need > (size_t)SSM_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "ssm_scan_fwd_noalloc: this shape needs %zu bytes of scratch, the static array holds "
             "%zu; use ssm_scan_fwd with a workspace",
             need, (size_t)SSM_NOALLOC_SCRATCH_BYTES);
    ssm::set_last_error(msg);
    return SSM_EUNSUPPORTED;
  }
  void* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != SSM_OK) return rc;
  return ssm_scan_fwd(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, hL, out, ckpt, scratch,
                      (size_t)SSM_NOALLOC_SCRATCH_BYTES, batch, dim, seqlen, dstate, io_dtype,
                      stream);
}
