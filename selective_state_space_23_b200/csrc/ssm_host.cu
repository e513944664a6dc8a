// Forward scan from and to host memory, pipelined over batch rows.
//
// A caller whose sequences live in host memory needs three things per call: copy the inputs to
// the GPU, scan, copy the output back.  Issued on one stream these run one after another and the
// GPU idles during both copies.  Here the batch is cut into chunks of rows that flow through
// three streams -- host-to-device copies, the scan, device-to-host copies -- with two device
// buffers per chunk stage, so the copy of chunk k+1 in, the scan of chunk k and the copy of
// chunk k-1 out run at the same time (the two copy directions use separate copy engines).  The
// streams and events are created once per device on first use and kept until the process exits;
// device buffers come from the caller's workspace.
#include <cuda_runtime.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_kernels.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSlots = 2;    // chunk buffers per stage in flight
constexpr int kChunks = 8;   // target number of chunks of the batch

struct Pipe {
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t ev_in[kSlots], ev_comp[kSlots], ev_out[kSlots];
  cudaEvent_t ev_start, ev_end;
  bool ready = false;
};

std::mutex g_mu;  // one pipeline per device; a call holds it while it enqueues its work
Pipe g_pipe[kMaxDevices];

int cuda_error(cudaError_t e, const char* what) {
  char msg[256];
  snprintf(msg, sizeof(msg), "ssm_scan_fwd_host: %s: %s", what, cudaGetErrorString(e));
  ssm::set_last_error(msg);
  return SSM_ECUDA;
}

int arg_error(int code, const char* what) {
  char msg[256];
  snprintf(msg, sizeof(msg), "ssm_scan_fwd_host: %s", what);
  ssm::set_last_error(msg);
  return code;
}

// The current device's pipeline, created on first use (caller holds g_mu).
int pipe_on_current_device(Pipe** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return arg_error(SSM_EUNSUPPORTED, "device index out of range");
  Pipe& p = g_pipe[dev];
  if (!p.ready) {
    cudaStream_t* ss[3] = {&p.in, &p.comp, &p.out};
    for (cudaStream_t* s : ss)
      if ((e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking)) != cudaSuccess)
        return cuda_error(e, "cudaStreamCreateWithFlags");
    for (int j = 0; j < kSlots; ++j) {
      cudaEvent_t* es[3] = {&p.ev_in[j], &p.ev_comp[j], &p.ev_out[j]};
      for (cudaEvent_t* ev : es)
        if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
          return cuda_error(e, "cudaEventCreateWithFlags");
    }
    if ((e = cudaEventCreateWithFlags(&p.ev_start, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&p.ev_end, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_error(e, "cudaEventCreateWithFlags");
    p.ready = true;
  }
  *out = &p;
  return SSM_OK;
}

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Device buffers of one chunk slot: u, delta, z, out; B, C; h0, hL; the scan's own workspace.
struct HostPlan {
  int rows;
  size_t x, bc, st, ws, slot, total;
};

HostPlan plan_host(int batch, int dim, int seqlen, int dstate, int io) {
  HostPlan p;
  const size_t es = io == SSM_BF16 ? 2 : 4;
  p.rows = std::max(1, (batch + kChunks - 1) / kChunks);
  p.x = align_up((size_t)p.rows * dim * seqlen * es);
  p.bc = align_up((size_t)p.rows * dstate * seqlen * es);
  p.st = align_up((size_t)p.rows * dim * dstate * 4);
  p.ws = align_up(ssm_scan_fwd_workspace_size(p.rows, dim, seqlen, dstate, io));
  p.slot = 4 * p.x + 2 * p.bc + 2 * p.st + p.ws;
  p.total = kSlots * p.slot;
  return p;
}

cudaError_t h2d(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s);
}

cudaError_t d2h(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s);
}

}  // namespace

extern "C" {

size_t ssm_scan_fwd_host_workspace_size(int batch, int dim, int seqlen, int dstate, int io_dtype) {
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0 || dstate > SSM_MAX_DSTATE ||
      (io_dtype != SSM_F32 && io_dtype != SSM_BF16))
    return 0;
  return plan_host(batch, dim, seqlen, dstate, io_dtype).total;
}

int ssm_scan_fwd_host(const void* u, const void* delta, const float* A, const void* B,
                      const void* C, const float* D, const void* z, const float* dt_bias,
                      int delta_softplus, const float* h0, float* hL, void* out, void* workspace,
                      size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                      int io_dtype, void* stream) {
  const size_t need = ssm_scan_fwd_host_workspace_size(batch, dim, seqlen, dstate, io_dtype);
  if (need == 0) return arg_error(SSM_EINVAL, "invalid shape or io dtype");
  if (!u || !delta || !B || !C || !out) return arg_error(SSM_EINVAL, "NULL host input or output");
  if (!workspace || workspace_bytes < need) {
    char msg[160];
    snprintf(msg, sizeof(msg), "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    return arg_error(SSM_EWORKSPACE, msg);
  }
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return arg_error(SSM_EINVAL, "workspace is not 256-byte aligned");

  const HostPlan pl = plan_host(batch, dim, seqlen, dstate, io_dtype);
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  const size_t x_row = (size_t)dim * seqlen * es, bc_row = (size_t)dstate * seqlen * es;
  const size_t st_row = (size_t)dim * dstate * 4;
  const char* hu = static_cast<const char*>(u);
  const char* hd = static_cast<const char*>(delta);
  const char* hz = static_cast<const char*>(z);
  const char* hB = static_cast<const char*>(B);
  const char* hC = static_cast<const char*>(C);
  char* ho = static_cast<char*>(out);

  std::lock_guard<std::mutex> lk(g_mu);
  Pipe* p = nullptr;
  int rc = pipe_on_current_device(&p);
  if (rc != SSM_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  // everything queued on the caller's stream so far comes first
  if ((e = cudaEventRecord(p->ev_start, s)) != cudaSuccess) return cuda_error(e, "cudaEventRecord");
  cudaStreamWaitEvent(p->in, p->ev_start, 0);
  cudaStreamWaitEvent(p->comp, p->ev_start, 0);
  cudaStreamWaitEvent(p->out, p->ev_start, 0);

  const int nchunk = (batch + pl.rows - 1) / pl.rows;
  for (int k = 0; k < nchunk; ++k) {
    const int j = k % kSlots;
    const int b0 = k * pl.rows, nb = std::min(pl.rows, batch - b0);
    char* slot = static_cast<char*>(workspace) + (size_t)j * pl.slot;
    char* du = slot;
    char* dd = du + pl.x;
    char* dz = dd + pl.x;
    char* dout = dz + pl.x;
    char* dB = dout + pl.x;
    char* dC = dB + pl.bc;
    float* dh0 = reinterpret_cast<float*>(dC + pl.bc);
    float* dhL = reinterpret_cast<float*>(reinterpret_cast<char*>(dh0) + pl.st);
    char* dws = reinterpret_cast<char*>(dhL) + pl.st;

    // inputs in, once the scan of the chunk that used this slot before has read them
    cudaStreamWaitEvent(p->in, p->ev_comp[j], 0);
    const size_t xb = nb * x_row, bcb = nb * bc_row;
    if ((e = h2d(du, hu + b0 * x_row, xb, p->in)) != cudaSuccess ||
        (e = h2d(dd, hd + b0 * x_row, xb, p->in)) != cudaSuccess ||
        (hz && (e = h2d(dz, hz + b0 * x_row, xb, p->in)) != cudaSuccess) ||
        (e = h2d(dB, hB + b0 * bc_row, bcb, p->in)) != cudaSuccess ||
        (e = h2d(dC, hC + b0 * bc_row, bcb, p->in)) != cudaSuccess ||
        (h0 && (e = h2d(dh0, h0 + (size_t)b0 * dim * dstate, nb * st_row, p->in)) != cudaSuccess))
      return cuda_error(e, "host-to-device copy");
    cudaEventRecord(p->ev_in[j], p->in);

    // the scan, once the inputs are in and the slot's previous output has gone out
    cudaStreamWaitEvent(p->comp, p->ev_in[j], 0);
    cudaStreamWaitEvent(p->comp, p->ev_out[j], 0);
    rc = ssm_scan_fwd(du, dd, A, dB, dC, D, hz ? dz : nullptr, dt_bias, delta_softplus,
                      h0 ? dh0 : nullptr, hL ? dhL : nullptr, dout, nullptr,
                      pl.ws ? dws : nullptr, pl.ws, nb, dim, seqlen, dstate, io_dtype, p->comp);
    if (rc != SSM_OK) return rc;
    cudaEventRecord(p->ev_comp[j], p->comp);

    // output back
    cudaStreamWaitEvent(p->out, p->ev_comp[j], 0);
    if ((e = d2h(ho + b0 * x_row, dout, xb, p->out)) != cudaSuccess ||
        (hL && (e = d2h(hL + (size_t)b0 * dim * dstate, dhL, nb * st_row, p->out)) != cudaSuccess))
      return cuda_error(e, "device-to-host copy");
    cudaEventRecord(p->ev_out[j], p->out);
  }
  // the caller's stream continues after the last copy out
  if ((e = cudaEventRecord(p->ev_end, p->out)) != cudaSuccess) return cuda_error(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(s, p->ev_end, 0)) != cudaSuccess)
    return cuda_error(e, "cudaStreamWaitEvent");
  return SSM_OK;
}

}  // extern "C"
