// C-ABI layer: argument validation, launch planning and workspace carving for the selective
// scan kernels.  Declarations and the full contract are in include/ssm_scan.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/ssm_scan.h"
#include "ssm_kernels.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SSM_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------------ device properties
int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  static std::mutex mu;
  static int cached[64] = {0};
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

int env_int(const char* name, int dflt) {
  const char* v = getenv(name);
  if (!v || !*v) return dflt;
  return atoi(v);
}

// ------------------------------------------------------------------ pointer validation
typedef int (*PFN_getAddressRange)(unsigned long long*, size_t*, unsigned long long);

PFN_getAddressRange address_range_fn() {
  static PFN_getAddressRange fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_getAddressRange>(p);
    cudaGetLastError();
  });
  return fn;
}

// The pointer must be usable by kernels on the current device and hold `bytes` bytes.
int check_ptr(const void* p, size_t bytes, size_t align, const char* name) {
  if (!p) return fail(SSM_EINVAL, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % align)
    return fail(SSM_EINVAL, "%s is not %zu-byte aligned", name, align);
  cudaPointerAttributes at;
  cudaError_t e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(SSM_EINVAL, "%s: cannot query pointer (%s)", name, cudaGetErrorString(e));
  }
  int dev = -1;
  cudaGetDevice(&dev);
  switch (at.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged: {
      if (at.type == cudaMemoryTypeDevice && at.device != dev)
        return fail(SSM_EINVAL, "%s lives on device %d, current device is %d", name, at.device, dev);
      PFN_getAddressRange fn = address_range_fn();
      if (fn) {
        unsigned long long base = 0;
        size_t size = 0;
        if (fn(&base, &size, (unsigned long long)(uintptr_t)p) == 0) {
          const unsigned long long q = (unsigned long long)(uintptr_t)p;
          if (q < base || q - base + bytes > size)
            return fail(SSM_EINVAL, "%s: allocation holds %llu bytes from this pointer, %zu needed",
                        name, (unsigned long long)(base + size - q), bytes);
        }
      }
      return SSM_OK;
    }
    case cudaMemoryTypeHost:
      if (at.devicePointer != p)
        return fail(SSM_EINVAL, "%s is page-locked host memory not mapped at the same address", name);
      return SSM_OK;
    default:
      return fail(SSM_EINVAL, "%s is not device-accessible memory (pageable host pointer?)", name);
  }
}

int check_opt(const void* p, size_t bytes, size_t align, const char* name) {
  return p ? check_ptr(p, bytes, align, name) : SSM_OK;
}

#define TRY(x)                 \
  do {                         \
    int _rc = (x);             \
    if (_rc != SSM_OK) return _rc; \
  } while (0)

int check_dims(int batch, int dim, int seqlen, int dstate, int io, int max_dstate = SSM_MAX_DSTATE) {
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0)
    return fail(SSM_EINVAL, "sizes must be positive (batch=%d dim=%d seqlen=%d dstate=%d)", batch,
                dim, seqlen, dstate);
  if (io != SSM_F32 && io != SSM_BF16) return fail(SSM_EINVAL, "io_dtype %d is not SSM_F32/SSM_BF16", io);
  if (dstate > max_dstate)
    return fail(SSM_EUNSUPPORTED, "dstate %d > %d is not implemented", dstate, max_dstate);
  if ((long long)batch * ((dim + 31) / 32) > (1LL << 30))
    return fail(SSM_EUNSUPPORTED, "batch*dim too large for one launch");
  return SSM_OK;
}

size_t esize(int io) { return io == SSM_BF16 ? 2 : 4; }

// B/C groups: dim must split into groups of whole warps (16 channels each), or into single
// channels (bc_groups == dim: B/C per channel).
int check_groups(int dim, int bc_groups) {
  if (bc_groups < 1) return fail(SSM_EINVAL, "bc_groups must be >= 1, got %d", bc_groups);
  if (bc_groups == 1 || bc_groups == dim) return SSM_OK;
  if (dim % bc_groups != 0) return fail(SSM_EINVAL, "dim %d is not a multiple of bc_groups %d", dim, bc_groups);
  if ((dim / bc_groups) % 16 != 0)
    return fail(SSM_EUNSUPPORTED,
                "grouped B/C needs dim / bc_groups to be a multiple of 16, or bc_groups == dim "
                "(got %d channels per group)",
                dim / bc_groups);
  return SSM_OK;
}
size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ forward launch plan
struct FwdPlan {
  int nchunk;
  int chunk_len;
  size_t ws_bytes;
};

// Lanes per channel of the general forward kernel (8 states per lane).
int fwd_lpc() { return 2; }

// Kernel family of the forward scan.  The general two-lanes-per-channel kernel
// (ssm_fwd_impl.cuh) serves every variant and layout and is the default: measured on B200 it is
// faster than the one-lane-per-channel kernel (ssm_fwd_lane.cuh) on every workload here (8 x 2048
// x 2048: 263 against 314 us), whose single warp per scheduler leaves fixed-latency dependencies
// exposed.  SSM_FWD_KERNEL=lane selects the latter for the default variant when its rows allow
// 16-byte copies.
bool fwd_lane_allowed() {
  const char* v = getenv("SSM_FWD_KERNEL");
  return v && strcmp(v, "lane") == 0;
}

// Channels per warp of each kernel family.
int fwd_chw(bool lane) { return lane ? 32 : 32 / fwd_lpc(); }

FwdPlan plan_fwd(int batch, int dim, int seqlen, int chw) {
  const int smsp = 4 * sm_count();
  const long long warps = (long long)batch * ((dim + chw - 1) / chw);
  const int nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  int S = 1;
  const int forced = env_int("SSM_FWD_SPLIT", 0);
  if (forced > 0) {
    S = forced;
  } else if (warps * 2 < smsp) {
    // fewer than half a warp per scheduler: split time so every scheduler gets ~2 warps
    S = (int)((2LL * smsp + warps - 1) / warps);
  }
  S = S < 1 ? 1 : (S > nblk ? nblk : S);
  FwdPlan p;
  if (S <= 1) {
    p.nchunk = 1;
    p.chunk_len = nblk * ssm::kBlk;
    p.ws_bytes = 0;
    return p;
  }
  const int blk_per_chunk = (nblk + S - 1) / S;
  p.chunk_len = blk_per_chunk * ssm::kBlk;
  p.nchunk = (seqlen + p.chunk_len - 1) / p.chunk_len;
  if (p.nchunk <= 1) {
    p.nchunk = 1;
    p.ws_bytes = 0;
    return p;
  }
  const size_t nch = (size_t)batch * dim;
  p.ws_bytes = align_up(p.nchunk * nch * ssm::kNS * 4) * 2 + align_up(p.nchunk * nch * 4);
  return p;
}

// Time segments of the chunked matrix form (scalar decay, N > 16): as for the per-state scan,
// segments of whole 16-step chunks when the warps (16 channels each) fill fewer than half the
// schedulers (SSM_SSD_SPLIT overrides); scratch for the segments' end states, entering states
// and ΣΔ.
FwdPlan plan_ssd(int batch, int dim, int seqlen, int dstate) {
  const int smsp = 4 * sm_count();
  const long long warps = (long long)batch * ((dim + 15) / 16);
  const int nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  int S = env_int("SSM_SSD_SPLIT", 0);
  if (S <= 0) S = warps * 2 < smsp ? (int)((2LL * smsp + warps - 1) / warps) : 1;
  S = S < 1 ? 1 : (S > nblk ? nblk : S);
  FwdPlan p;
  const int blk_per = (nblk + S - 1) / S;
  p.chunk_len = blk_per * ssm::kBlk;
  p.nchunk = (seqlen + p.chunk_len - 1) / p.chunk_len;
  const size_t nch = (size_t)batch * dim;
  p.ws_bytes = p.nchunk > 1 ? 2 * align_up((size_t)p.nchunk * nch * dstate * 4) +
                                  align_up((size_t)p.nchunk * nch * 4)
                            : 0;
  return p;
}

__global__ void chain_kernel(const float* __restrict__ hend, const float* __restrict__ dsum,
                             const float* __restrict__ A, int scalar_a,
                             const float* __restrict__ h0, float* __restrict__ hin, int nseg,
                             long long nch, int dim, int N);

// The reverse scan in the chunked matrix form runs the forward-direction kernels on inputs
// mirrored along time into the workspace: `rows_x` bf16 rows of u-like tensors (u, delta, z;
// and dout in the backward) and B, C.  Bytes of those copies.
size_t mirror_bytes(int batch, int dim, int seqlen, int dstate, int bc_groups, int rows_x) {
  const size_t nx = (size_t)batch * dim * seqlen * 2;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * 2;
  return (size_t)rows_x * align_up(nx) + 2 * align_up(nbc);
}

// Workspace that covers the plan of either kernel family (the family is chosen per call, from
// the pointers' alignment too).
size_t fwd_ws_bytes(int batch, int dim, int seqlen) {
  const size_t a = plan_fwd(batch, dim, seqlen, fwd_chw(false)).ws_bytes;
  const size_t b = plan_fwd(batch, dim, seqlen, fwd_chw(true)).ws_bytes;
  return a > b ? a : b;
}

// Launch tuning of the forward kernel (measured on B200; the environment variables override it
// for experiments): one warp per CTA; 14 of every 16 exponentials per lane and step pair on the
// MUFU unit, the rest on the FMA-pipe polynomial (best on 8 x 2048 and 4 x 5120 channels and on
// the time-split 1 x 256 x 2^20 sequence).
int fwd_wpb() {
  const int w = env_int("SSM_FWD_WPB", 1);
  return (w == 1 || w == 2 || w == 4) ? w : 1;
}
int fwd_kmufu(long long warps) {
  (void)warps;
  return env_int("SSM_FWD_KMUFU", 14);
}

// The output kernel's 255-register form pays off below 8 warps per SM (SSM_FWD_WIDE=0/1 forces it).
int fwd_wide(long long warps) { return env_int("SSM_FWD_WIDE", warps < 8LL * sm_count() ? 1 : 0); }

struct BwdLayout {
  size_t ckpt, part_bc, part_adt, split, fwd_ws, total;
  int wpb, ngroups;
  int nsplit;  // the most time chunks the history backward may take for this shape
};

// Time split of the register-history backward: when its CTAs (batch rows x channel groups) fill
// less than one wave, time is cut into chunks of whole 16-step blocks (SSM_BWD_SPLIT
// overrides).  Returns the number of chunks (1: none); *bpc = blocks per chunk.
//
// Measured on B200 (backward of 4 x 5120, 8 x 2048, 2 x 2048, 1 x 2048 and 1 x 256 channels):
// a grid just over one wave (e.g. 640 CTAs on 444 slots) is the worst case, since its second
// wave runs nearly a whole chunk for a few CTAs; a grid that fills one wave exactly does well
// when its chunks stay long (>= 32 blocks); otherwise about four waves of chunks of >= 16 blocks
// balance the SMs best (4 x 5120 x 2048: 1.52 -> 1.35 ms, 2 x 2048 x 8192: 1.43 -> 1.13 ms),
// and where chunks of 16 blocks cannot make two waves, one wave.
int plan_bwd_split(int batch, int dim, int seqlen, int wpb, int ctas_per_sm, int* bpc) {
  const int nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  const long long ctas = (long long)batch * (((dim + 15) / 16 + wpb - 1) / wpb);
  const long long slots = (long long)sm_count() * ctas_per_sm;
  long long S = env_int("SSM_BWD_SPLIT", 0);
  if (S <= 0) {
    if (ctas >= slots) {
      S = 1;
    } else {
      const long long s1 = slots / ctas;  // the most chunks that still fit one wave
      if (s1 >= 2 && 20 * s1 * ctas >= 19 * slots && nblk >= 32 * s1) {
        S = s1;
      } else {
        const long long by_len = nblk / 16 > 1 ? nblk / 16 : 1;
        S = (4 * slots + ctas - 1) / ctas;
        S = S < by_len ? S : by_len;
        // too short a sequence for several waves: rather one wave than just over one
        if (S * ctas < 2 * slots) S = s1 < by_len ? s1 : by_len;
      }
    }
  }
  S = S < 1 ? 1 : (S > nblk ? nblk : S);
  *bpc = (int)((nblk + S - 1) / S);
  return (nblk + *bpc - 1) / *bpc;
}

// Whether the history backward (and so its time split) can serve this request, judged from the
// shape and flags alone (the pointers' alignment is checked at the call).
bool bwd_hist_shape(int dim, int seqlen, int dstate, int bc_groups, int flags) {
  return !(flags & (SSM_REVERSE | SSM_ZOH | SSM_CHANNELS_LAST)) && dstate == ssm::kNS &&
         seqlen % 8 == 0 && !(bc_groups == dim && bc_groups > 1);
}

BwdLayout layout_bwd(int batch, int dim, int seqlen, int dstate, bool have_ckpt, int bc_groups,
                     int io_dtype, int flags) {
  BwdLayout l;
  // one warp per CTA: CTAs of several warps synchronise once per block for the dB/dC partials,
  // which measured slower on B200 than writing one partial per warp (and with grouped B/C every
  // CTA must lie inside one group)
  l.wpb = bc_groups > 1 ? 1 : env_int("SSM_BWD_WPB", 1);
  if (l.wpb < 1 || l.wpb > 4) l.wpb = 1;
  const int warps_per_b = (dim + 15) / 16;  // 16 channels per warp
  l.ngroups = (warps_per_b + l.wpb - 1) / l.wpb;
  const size_t nch = (size_t)batch * dim;
  const size_t nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  l.ckpt = have_ckpt ? 0 : align_up(nch * nblk * dstate * 4);
  l.part_bc = align_up((size_t)l.ngroups * batch * 2 * ssm::kNS * seqlen * 4);
  // 4 warps per CTA give the fewest CTAs, hence the most chunks
  int bpc = 0;
  l.nsplit = bwd_hist_shape(dim, seqlen, dstate, bc_groups, flags)
                 ? plan_bwd_split(batch, dim, seqlen, 4, ssm::bwd_hist_ctas_per_sm(io_dtype, 4), &bpc)
                 : 1;
  l.part_adt = align_up((size_t)l.nsplit * nch * (ssm::kNS + 2) * 4);
  // chunk summaries and entering adjoints [nsplit][nch][16], chunk ΣΔ [nsplit][nch]
  l.split = l.nsplit > 1 ? 2 * align_up((size_t)l.nsplit * nch * ssm::kNS * 4) +
                               align_up((size_t)l.nsplit * nch * 4)
                         : 0;
  // the replay pass without checkpoints takes the forward's own time split
  l.fwd_ws = have_ckpt ? 0 : fwd_ws_bytes(batch, dim, seqlen);
  l.total = l.ckpt + l.part_bc + l.part_adt + l.split + l.fwd_ws;
  return l;
}

}  // namespace

namespace ssm {
// Records a message for ssm_last_error() on the calling thread (used by entry points that live
// in other translation units).
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
// The pointer validation of the entry points, for entry points in other translation units: the
// pointer is usable by kernels on the current device and its allocation holds `bytes` bytes.
int check_device_ptr(const void* p, size_t bytes, size_t align, const char* name) {
  return check_ptr(p, bytes, align, name);
}
}  // namespace ssm

extern "C" {

const char* ssm_status_string(int status) {
  switch (status) {
    case SSM_OK: return "ok";
    case SSM_EINVAL: return "invalid argument";
    case SSM_EUNSUPPORTED: return "unsupported";
    case SSM_ECUDA: return "CUDA error";
    case SSM_EWORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

const char* ssm_last_error(void) { return g_err; }

const char* ssm_version(void) { return "ssm_b200 0.1 (sm_100a)"; }

size_t ssm_scan_fwd_workspace_size(int batch, int dim, int seqlen, int dstate, int io_dtype) {
  if (check_dims(batch, dim, seqlen, dstate, io_dtype) != SSM_OK) return 0;
  return fwd_ws_bytes(batch, dim, seqlen);
}

}  // extern "C"

namespace {

// Forward scan.  flags: SSM_SCALAR_A (A is [dim], one decay rate per channel, instead of
// [dim][dstate]) and SSM_REVERSE (scan from t = L-1 down to 0).
int scan_fwd_impl(const void* u, const void* delta, const float* A, const void* B, const void* C,
                  const float* D, const void* z, const float* dt_bias, int delta_softplus,
                  const float* h0, float* hL, void* out, float* ckpt, void* workspace,
                  size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                  int io_dtype, void* stream, int flags, int bc_groups) {
  g_err[0] = 0;
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH | SSM_CHANNELS_LAST))
    return fail(SSM_EINVAL, "unknown flags 0x%x", flags);
  const bool scalar_a = (flags & SSM_SCALAR_A) != 0;
  // scalar decay takes N up to 128 (the chunked matrix form, ssm_ssd.cu); per-state decay 16
  TRY(check_dims(batch, dim, seqlen, dstate, io_dtype, scalar_a ? SSM_MAX_DSTATE_SCALAR : SSM_MAX_DSTATE));
  TRY(check_groups(dim, bc_groups));
  const size_t es = esize(io_dtype);
  const size_t nx = (size_t)batch * dim * seqlen * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * es;
  const size_t nst = (size_t)batch * dim * dstate * 4;
  const size_t nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  TRY(check_ptr(u, nx, es, "u"));
  TRY(check_ptr(delta, nx, es, "delta"));
  TRY(check_ptr(A, (size_t)dim * (scalar_a ? 1 : dstate) * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_ptr(out, nx, es, "out"));
  TRY(check_opt(D, (size_t)dim * 4, 4, "D"));
  TRY(check_opt(z, nx, es, "z"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  TRY(check_opt(h0, nst, 4, "h0"));
  TRY(check_opt(hL, nst, 4, "hL"));
  TRY(check_opt(ckpt, (size_t)batch * dim * nblk * dstate * 4, 4, "ckpt"));
  if (out == u || out == delta || out == z) return fail(SSM_EINVAL, "out aliases an input");

  const bool zoh = (flags & SSM_ZOH) != 0, reverse = (flags & SSM_REVERSE) != 0;
  const bool channels_last = (flags & SSM_CHANNELS_LAST) != 0;
  // 128-bit row accesses need rows along L; the channels-last layout takes element accesses
  const bool vec = !channels_last && (seqlen * es) % 16 == 0 && aligned16(u) &&
                   aligned16(delta) && aligned16(z) && aligned16(out) && aligned16(B) &&
                   aligned16(C);
  // scalar decay with N > 16: the chunked matrix form on the tensor cores (bf16, N = 32, 64 or
  // 128, forward direction, [batch][dim][L] rows, B/C shared by each 64-channel tile).  With
  // N = 16 the same form serves the requests it takes; SSM_SCALAR_FORM=state keeps those on the
  // per-state kernel.  Both write the same checkpoints (the state entering every 16-step block).
  const char* sform = getenv("SSM_SCALAR_FORM");
  const bool chunked16 = scalar_a && dstate == ssm::kNS && io_dtype == SSM_BF16 &&
                         !(flags & (SSM_ZOH | SSM_REVERSE | SSM_CHANNELS_LAST)) &&
                         (bc_groups == 1 || (dim % bc_groups == 0 && (dim / bc_groups) % 64 == 0)) &&
                         !(sform && strcmp(sform, "state") == 0);
  // f32 io with N > 16: the sum of 16-state f32 forwards over the state slices (ssm_slices.cu)
  if (dstate > SSM_MAX_DSTATE && io_dtype == SSM_F32)
    return ssm::scan_fwd_slices(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, hL, out,
                                ckpt, workspace, workspace_bytes, batch, dim, seqlen, dstate,
                                bc_groups, io_dtype, flags, stream);
  if (dstate > SSM_MAX_DSTATE || chunked16) {
    if (io_dtype != SSM_BF16 || (dstate != 16 && dstate != 32 && dstate != 64 && dstate != 128) ||
        channels_last ||
        !(bc_groups == 1 || (dim % bc_groups == 0 && (dim / bc_groups) % 64 == 0)))
      return fail(SSM_EUNSUPPORTED,
                  "scalar decay with dstate %d > %d needs bf16 or f32 io, dstate 32, 64 or 128, the "
                  "default layout and B/C groups of whole 64-channel tiles", dstate,
                  SSM_MAX_DSTATE);
    if (!aligned16(ckpt))
      return fail(SSM_EINVAL, "ckpt must be 16-byte aligned (chunked matrix form)");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    // reverse: the kernels scan inputs mirrored along time (copies at the workspace's start);
    // the output is mirrored back in place at the end
    const size_t mb = reverse ? mirror_bytes(batch, dim, seqlen, dstate, bc_groups, 3) : 0;
    const void *ku = u, *kd = delta, *kz = z, *kB = B, *kC = C;
    if (reverse) {
      if (!workspace || workspace_bytes < mb)
        return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed (reverse scan)",
                    workspace_bytes, mb);
      if (reinterpret_cast<uintptr_t>(workspace) & 255)
        return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
      TRY(check_ptr(workspace, mb, 256, "workspace"));
      char* m = reinterpret_cast<char*>(workspace);
      const long long rx = (long long)batch * dim, rbc = (long long)batch * bc_groups * dstate;
      void* mu = m;
      void* md = m + align_up(nx);
      void* mz = z ? m + 2 * align_up(nx) : nullptr;
      void* mB = m + 3 * align_up(nx);
      void* mC = m + 3 * align_up(nx) + align_up(nbc);
      if ((e = ssm::mirror_rows(u, mu, rx, seqlen, s)) != cudaSuccess ||
          (e = ssm::mirror_rows(delta, md, rx, seqlen, s)) != cudaSuccess ||
          (z && (e = ssm::mirror_rows(z, mz, rx, seqlen, s)) != cudaSuccess) ||
          (e = ssm::mirror_rows(B, mB, rbc, seqlen, s)) != cudaSuccess ||
          (e = ssm::mirror_rows(C, mC, rbc, seqlen, s)) != cudaSuccess)
        return cuda_fail(e, "reverse scan: mirrored inputs");
      ku = mu; kd = md; kz = mz; kB = mB; kC = mC;
      workspace = m + mb;
      workspace_bytes -= mb;
    }
    ssm::FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.u = ku; a.delta = kd; a.z = kz; a.B = kB; a.C = kC;
    a.A = A; a.D = D; a.dt_bias = dt_bias; a.h0 = h0; a.out = out; a.hL = hL; a.ckpt = ckpt;
    a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
    a.softplus = delta_softplus ? 1 : 0;
    a.scalar_a = 1;
    a.zoh = zoh ? 1 : 0;
    a.bc_groups = bc_groups;
    a.rows16 = vec ? 1 : 0;
    FwdPlan plan = plan_ssd(batch, dim, seqlen, dstate);
    if (plan.nchunk > 1 && (!workspace || workspace_bytes < plan.ws_bytes ||
                            (reinterpret_cast<uintptr_t>(workspace) & 255))) {
      plan.nchunk = 1;  // not enough scratch: same result without the time split
      plan.chunk_len = (int)nblk * ssm::kBlk;
    }
    a.chunk_len = plan.chunk_len;
    a.nchunk = plan.nchunk;
    if (plan.nchunk > 1) {
      TRY(check_ptr(workspace, plan.ws_bytes, 256, "workspace"));
      const size_t nch = (size_t)batch * dim;
      const size_t seg = align_up((size_t)plan.nchunk * nch * dstate * 4);
      char* w = reinterpret_cast<char*>(workspace);
      a.summ = reinterpret_cast<float*>(w);
      float* hin = reinterpret_cast<float*>(w + seg);
      a.dsum = reinterpret_cast<float*>(w + 2 * seg);
      if ((e = ssm::launch_ssd_fwd(a, ssm::kSsdSummary, s)) != cudaSuccess)
        return cuda_fail(e, "summary pass (chunked matrix form)");
      const long long n = (long long)nch * dstate;
      chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.summ, a.dsum, A, 1, h0, hin,
                                                               plan.nchunk, (long long)nch, dim,
                                                               dstate);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "carry (chunked matrix form)");
      a.hin = hin;
    }
    e = ssm::launch_ssd_fwd(a, ssm::kSsdOut, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward pass (chunked matrix form)");
    if (reverse && (e = ssm::mirror_rows(out, out, (long long)batch * dim, seqlen, s)) != cudaSuccess)
      return cuda_fail(e, "reverse scan: mirrored output");
    return SSM_OK;
  }
  // B/C per channel (bc_groups == dim > 1): the per-state kernel of ssm_pcbc.cu, no time split
  const bool pcbc = bc_groups == dim && bc_groups > 1;
  if (pcbc && (scalar_a || zoh || reverse || channels_last))
    return fail(SSM_EUNSUPPORTED, "B/C per channel combines with no other variant flag");
  const bool lane = !pcbc && fwd_lane_allowed() && vec && !scalar_a && !zoh && !reverse &&
                    (bc_groups == 1 || (dim / bc_groups) % 32 == 0);
  FwdPlan plan = plan_fwd(batch, dim, seqlen, fwd_chw(lane));
  if (pcbc) plan.nchunk = 1;
  if (plan.nchunk > 1 && (!workspace || workspace_bytes < plan.ws_bytes ||
                          (reinterpret_cast<uintptr_t>(workspace) & 255))) {
    plan.nchunk = 1;  // not enough scratch: same result without the time split
    plan.chunk_len = (int)nblk * ssm::kBlk;
  }
  if (plan.nchunk > 1) TRY(check_ptr(workspace, plan.ws_bytes, 256, "workspace"));

  ssm::FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.A = A; a.D = D; a.dt_bias = dt_bias; a.h0 = h0;
  a.out = out; a.hL = hL; a.ckpt = ckpt;
  a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
  a.chunk_len = plan.chunk_len; a.nchunk = plan.nchunk;
  a.softplus = delta_softplus ? 1 : 0;
  a.scalar_a = scalar_a ? 1 : 0;
  a.reverse = (flags & SSM_REVERSE) ? 1 : 0;
  a.zoh = (flags & SSM_ZOH) ? 1 : 0;
  a.bc_groups = bc_groups;
  a.lpc = (scalar_a || a.zoh || bc_groups > 1) ? 2 : fwd_lpc();
  a.warps_per_b = (dim + 32 / a.lpc - 1) / (32 / a.lpc);
  a.channels_last = channels_last ? 1 : 0;
  if (lane) {
    a.lpc = 1;
    a.warps_per_b = (dim + 31) / 32;
  } else if (a.channels_last) {
    a.lpc = 2;
    a.warps_per_b = (dim + 15) / 16;
    // 16-byte tiles of 8 channels (or states) per lane: every warp full, rows 16-byte aligned
    a.cl_tile = dim % 16 == 0 && dstate == 16 && (dim * es) % 16 == 0 && aligned16(u) &&
                aligned16(delta) && aligned16(z) && aligned16(out) && aligned16(B) &&
                aligned16(C);
  }
  a.nwarps = (long long)batch * a.warps_per_b;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int wpb = fwd_wpb();
  const int km = fwd_kmufu(a.nwarps * (long long)plan.nchunk);
  a.wide = fwd_wide(a.nwarps * (long long)plan.nchunk);
  cudaError_t e;
  if (pcbc) {
    plan.chunk_len = (int)nblk * ssm::kBlk;
    a.chunk_len = plan.chunk_len; a.nchunk = 1;
    const bool pvec = (seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) &&
                      aligned16(z) && aligned16(out) && aligned16(B) && aligned16(C);
    if ((e = ssm::launch_fwd_pcbc(a, io_dtype, pvec, ssm::kFwdOut, s)) != cudaSuccess)
      return cuda_fail(e, "forward pass (B/C per channel)");
    return SSM_OK;
  }
  if (plan.nchunk > 1) {
    const size_t nch = (size_t)batch * dim;
    char* w = reinterpret_cast<char*>(workspace);
    float* summ = reinterpret_cast<float*>(w);
    float* hin = reinterpret_cast<float*>(w + align_up(plan.nchunk * nch * ssm::kNS * 4));
    float* dsum = reinterpret_cast<float*>(w + 2 * align_up(plan.nchunk * nch * ssm::kNS * 4));
    ssm::FwdArgs as = a;
    as.summ = summ; as.dsum = dsum;
    as.out = nullptr; as.hL = nullptr; as.ckpt = nullptr; as.h0 = nullptr;
    e = lane ? ssm::launch_fwd_lane(as, io_dtype, ssm::kFwdSummary, km, s)
             : ssm::launch_fwd(as, io_dtype, vec, ssm::kFwdSummary, wpb, km, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward summary pass");
    if ((e = ssm::launch_fwd_carry(a, summ, dsum, hin, s)) != cudaSuccess)
      return cuda_fail(e, "forward carry pass");
    a.hin = hin;
  }
  e = lane ? ssm::launch_fwd_lane(a, io_dtype, ssm::kFwdOut, km, s)
           : ssm::launch_fwd(a, io_dtype, vec, ssm::kFwdOut, wpb, km, s);
  if (e != cudaSuccess) return cuda_fail(e, "forward pass");
  return SSM_OK;
}

// Time chunks of a whole-sequence summary and its scratch: the forward's plan with one more
// chunk slot (summaries, entering states, ΣΔ).
// Sequence summary of a scalar-decay scan with N = 32, 64 or 128 in bf16: the chunked matrix
// form's summary pass over every one of the planner's S segments (each from a zero state), the
// chain of the S segment maps from zero (its (S+1)-th entering state is the sequence's end
// state), and the finishing kernel.  Workspace: per-segment end states [S][batch*dim][N],
// entering states [S+1][batch*dim][N], per-segment ΣΔ [S][batch*dim].
struct SummaryChunkedLayout {
  FwdPlan plan;
  size_t summ, hin, ds, total;
};

SummaryChunkedLayout summary_chunked_layout(int batch, int dim, int seqlen, int dstate) {
  SummaryChunkedLayout l;
  l.plan = plan_ssd(batch, dim, seqlen, dstate);
  const size_t nch = (size_t)batch * dim, S = (size_t)l.plan.nchunk;
  l.summ = 0;
  l.hin = align_up(S * nch * dstate * 4);
  l.ds = l.hin + align_up((S + 1) * nch * dstate * 4);
  l.total = l.ds + align_up(S * nch * 4);
  return l;
}

__global__ void summary_finish_kernel(const float* __restrict__ hin_end, int hs,
                                      const float* __restrict__ dsum, int S, long long nch, int N,
                                      float* __restrict__ hend, float* __restrict__ dsum_out);

int summary_chunked(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* dt_bias, int delta_softplus, float* hend,
                    float* dsum, void* workspace, size_t workspace_bytes, int batch, int dim,
                    int seqlen, int dstate, int bc_groups, int flags, void* stream) {
  if (dstate != 32 && dstate != 64 && dstate != 128)
    return fail(SSM_EUNSUPPORTED, "a bf16 sequence summary with dstate %d > %d takes 32, 64 or 128",
                dstate, SSM_MAX_DSTATE);
  if (!(bc_groups == 1 || (dim % bc_groups == 0 && (dim / bc_groups) % 64 == 0)))
    return fail(SSM_EUNSUPPORTED, "a bf16 sequence summary with dstate > %d takes B/C shared or in "
                "groups of whole 64-channel tiles", SSM_MAX_DSTATE);
  const size_t es = 2;
  const size_t nx = (size_t)batch * dim * seqlen * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * es;
  const size_t nch = (size_t)batch * dim;
  TRY(check_ptr(u, nx, es, "u"));
  TRY(check_ptr(delta, nx, es, "delta"));
  TRY(check_ptr(A, (size_t)dim * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  TRY(check_ptr(hend, nch * dstate * 4, 4, "hend"));
  TRY(check_opt(dsum, nch * 4, 4, "dsum"));
  const SummaryChunkedLayout l = summary_chunked_layout(batch, dim, seqlen, dstate);
  if (!workspace || workspace_bytes < l.total)
    return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, l.total);
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  TRY(check_ptr(workspace, l.total, 256, "workspace"));
  char* w = reinterpret_cast<char*>(workspace);
  const int S = l.plan.nchunk;
  ssm::FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.u = u; a.delta = delta; a.B = B; a.C = C; a.A = A; a.dt_bias = dt_bias;
  a.summ = reinterpret_cast<float*>(w + l.summ);
  a.dsum = reinterpret_cast<float*>(w + l.ds);
  a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
  a.softplus = delta_softplus ? 1 : 0;
  a.scalar_a = 1;
  a.zoh = (flags & SSM_ZOH) ? 1 : 0;
  a.bc_groups = bc_groups;
  a.rows16 = ((size_t)seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) &&
             aligned16(B) && aligned16(C);
  a.chunk_len = l.plan.chunk_len;
  a.nchunk = S + 1;  // the summary pass covers segments 0 .. S-1, every one of the sequence
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ssm::launch_ssd_fwd(a, ssm::kSsdSummary, s);
  if (e != cudaSuccess) return cuda_fail(e, "sequence summary (chunked matrix form)");
  float* hin = reinterpret_cast<float*>(w + l.hin);
  const long long n = (long long)nch * dstate;
  chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.summ, a.dsum, A, 1, nullptr, hin,
                                                           S + 1, (long long)nch, dim, dstate);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "sequence summary chain");
  summary_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      hin + (size_t)S * nch * dstate, dstate, a.dsum, S, (long long)nch, dstate, hend, dsum);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "sequence summary finish");
  return SSM_OK;
}

FwdPlan plan_summary(int batch, int dim, int seqlen) {
  FwdPlan p = plan_fwd(batch, dim, seqlen, fwd_chw(false));
  const size_t nch = (size_t)batch * dim;
  const size_t slots = (size_t)p.nchunk + 1;
  p.ws_bytes = 2 * align_up(slots * nch * ssm::kNS * 4) + align_up(slots * nch * 4);
  return p;
}

// The end state from zero of a whole sequence, out of the carry's entering states (rows of hs
// floats per channel) into [batch][dim][N], and each channel's ΣΔ summed (Kahan) over the S
// chunk summaries.
__global__ void summary_finish_kernel(const float* __restrict__ hin_end, int hs,
                                      const float* __restrict__ dsum, int S, long long nch, int N,
                                      float* __restrict__ hend, float* __restrict__ dsum_out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nch * N) return;
  const long long ch = i / N;
  const int n = (int)(i % N);
  hend[i] = hin_end[ch * hs + n];
  if (n == 0 && dsum_out) {
    float acc = 0.f, comp = 0.f;
    for (int j = 0; j < S; ++j) {
      const float y = dsum[(long long)j * nch + ch] - comp;
      const float t = acc + y;
      comp = (t - acc) - y;
      acc = t;
    }
    dsum_out[ch] = acc;
  }
}

// The state entering each of nseg consecutive segments: hin[0] = h0 (zero without one) and
// hin[r + 1] = exp(A ΣΔ_r) hin[r] + hend[r], the composition of the segments' affine maps in
// order (one thread per (channel, state), the segments in sequence).
__global__ void chain_kernel(const float* __restrict__ hend, const float* __restrict__ dsum,
                             const float* __restrict__ A, int scalar_a,
                             const float* __restrict__ h0, float* __restrict__ hin, int nseg,
                             long long nch, int dim, int N) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nch * N) return;
  const long long ch = i / N;
  const int n = (int)(i % N), d = (int)(ch % dim);
  const float An = scalar_a ? A[d] : A[(long long)d * N + n];
  const long long stride = nch * N;
  float h = h0 ? h0[i] : 0.f;
  for (int r = 0; r < nseg; ++r) {
    hin[(long long)r * stride + i] = h;
    if (r + 1 < nseg)  // the last segment's map is not needed (nor, for a split, written)
      h = fmaf(expf(An * dsum[(long long)r * nch + ch]), h, hend[(long long)r * stride + i]);
  }
}

// A[d] copied to every state: Af[d][n] = A[d].
__global__ void broadcast_a_kernel(const float* __restrict__ A, float* __restrict__ Af, int dim,
                                   int N) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < (long long)dim * N) Af[i] = A[i / N];
}

// dA[d] = sum over n of dAf[d][n], in the order n = 0 .. N-1.
__global__ void reduce_da_kernel(const float* __restrict__ dAf, float* __restrict__ dA, int dim,
                                 int N) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= dim) return;
  float acc = 0.f;
  for (int n = 0; n < N; ++n) acc += dAf[(long long)d * N + n];
  dA[d] = acc;
}

}  // namespace

extern "C" {

int ssm_scan_fwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                 const float* D, const void* z, const float* dt_bias, int delta_softplus,
                 const float* h0, float* hL, void* out, float* ckpt, void* workspace,
                 size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                 int io_dtype, void* stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, hL, out, ckpt,
                       workspace, workspace_bytes, batch, dim, seqlen, dstate, io_dtype, stream, 0, 1);
}

size_t ssm_scan_fwd_ex_workspace_size(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                      int io_dtype, int flags) {
  if (bc_groups < 1) return 0;
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE && io_dtype == SSM_F32)  // 16-state slices
    return ssm::scan_fwd_slices_workspace(batch, dim, seqlen, dstate, bc_groups, io_dtype, flags);
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE) {  // the chunked matrix form's segments
    if (check_dims(batch, dim, seqlen, dstate, io_dtype, SSM_MAX_DSTATE_SCALAR) != SSM_OK) return 0;
    return plan_ssd(batch, dim, seqlen, dstate).ws_bytes +
           ((flags & SSM_REVERSE) ? mirror_bytes(batch, dim, seqlen, dstate, bc_groups, 3) : 0);
  }
  return ssm_scan_fwd_workspace_size(batch, dim, seqlen, dstate, io_dtype);
}

int ssm_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                    void* workspace, size_t workspace_bytes, int batch, int dim, int seqlen,
                    int dstate, int bc_groups, int io_dtype, int flags, void* stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, hL, out, ckpt,
                       workspace, workspace_bytes, batch, dim, seqlen, dstate, io_dtype, stream,
                       flags, bc_groups);
}

size_t ssm_scan_fwd_scalar_a_workspace_size(int batch, int dim, int seqlen, int dstate,
                                            int io_dtype) {
  return ssm_scan_fwd_ex_workspace_size(batch, dim, seqlen, dstate, 1, io_dtype, SSM_SCALAR_A);
}

int ssm_scan_fwd_scalar_a(const void* u, const void* delta, const float* A, const void* B,
                          const void* C, const float* D, const void* z, const float* dt_bias,
                          int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                          void* workspace, size_t workspace_bytes, int batch, int dim, int seqlen,
                          int dstate, int io_dtype, void* stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, hL, out, ckpt,
                       workspace, workspace_bytes, batch, dim, seqlen, dstate, io_dtype, stream,
                       SSM_SCALAR_A, 1);
}

size_t ssm_scan_bwd_workspace_size(int batch, int dim, int seqlen, int dstate, int io_dtype,
                                   int have_ckpt) {
  if (check_dims(batch, dim, seqlen, dstate, io_dtype) != SSM_OK) return 0;
  return layout_bwd(batch, dim, seqlen, dstate, have_ckpt != 0, 1, io_dtype, 0).total;
}

}  // extern "C"

namespace {

// Backward of the per-state-decay scan (A is [dim][dstate]); reverse: of the reverse scan.
int scan_bwd_core(const void* u, const void* delta, const float* A, const void* B, const void* C,
                  const float* D, const void* z, const float* dt_bias, int delta_softplus,
                  const float* h0, const void* dout, const float* dhL, const float* ckpt,
                  void* du, void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                  float* ddt_bias, float* dh0, void* workspace, size_t workspace_bytes,
                  int batch, int dim, int seqlen, int dstate, int io_dtype, void* stream,
                  bool reverse, bool zoh, int bc_groups, bool channels_last = false) {
  TRY(check_dims(batch, dim, seqlen, dstate, io_dtype));
  TRY(check_groups(dim, bc_groups));
  const size_t es = esize(io_dtype);
  const size_t nx = (size_t)batch * dim * seqlen * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * es;
  const size_t nst = (size_t)batch * dim * dstate * 4;
  const size_t nblk = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  TRY(check_ptr(u, nx, es, "u"));
  TRY(check_ptr(delta, nx, es, "delta"));
  TRY(check_ptr(A, (size_t)dim * dstate * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_ptr(dout, nx, es, "dout"));
  TRY(check_opt(D, (size_t)dim * 4, 4, "D"));
  TRY(check_opt(z, nx, es, "z"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  TRY(check_opt(h0, nst, 4, "h0"));
  TRY(check_opt(dhL, nst, 4, "dhL"));
  TRY(check_opt(ckpt, (size_t)batch * dim * nblk * dstate * 4, 4, "ckpt"));
  TRY(check_opt(du, nx, es, "du"));
  TRY(check_opt(ddelta, nx, es, "ddelta"));
  TRY(check_opt(dz, nx, es, "dz"));
  TRY(check_opt(dB, nbc, es, "dB"));
  TRY(check_opt(dC, nbc, es, "dC"));
  TRY(check_opt(dA, (size_t)dim * dstate * 4, 4, "dA"));
  TRY(check_opt(dD, (size_t)dim * 4, 4, "dD"));
  TRY(check_opt(ddt_bias, (size_t)dim * 4, 4, "ddt_bias"));
  TRY(check_opt(dh0, nst, 4, "dh0"));
  if (!du && !ddelta && !dA && !dB && !dC && !dD && !dz && !ddt_bias && !dh0)
    return fail(SSM_EINVAL, "no gradient output requested");
  if (dz && !z) return fail(SSM_EINVAL, "dz requested but z is NULL");

  const int lflags = (reverse ? SSM_REVERSE : 0) | (zoh ? SSM_ZOH : 0) |
                     (channels_last ? SSM_CHANNELS_LAST : 0);
  const BwdLayout l = layout_bwd(batch, dim, seqlen, dstate, ckpt != nullptr, bc_groups,
                                 io_dtype, lflags);
  if (!workspace || workspace_bytes < l.total)
    return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, l.total);
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  TRY(check_ptr(workspace, l.total, 256, "workspace"));

  char* w = reinterpret_cast<char*>(workspace);
  float* ck_ws = reinterpret_cast<float*>(w);
  float* part_bc = reinterpret_cast<float*>(w + l.ckpt);
  float* part_adt = reinterpret_cast<float*>(w + l.ckpt + l.part_bc);
  char* split_ws = w + l.ckpt + l.part_bc + l.part_adt;
  char* fwd_ws = split_ws + l.split;
  const size_t nch = (size_t)batch * dim;
  const bool vec = !channels_last && (seqlen * es) % 16 == 0 && aligned16(u) &&
                   aligned16(delta) && aligned16(z) && aligned16(dout) && aligned16(du) &&
                   aligned16(ddelta) && aligned16(dz) && aligned16(B) && aligned16(C);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;

  const bool pcbc = bc_groups == dim && bc_groups > 1;
  if (pcbc && (reverse || zoh || channels_last))
    return fail(SSM_EUNSUPPORTED, "B/C per channel combines with no other variant flag");
  const bool pvec = (seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) &&
                    aligned16(z) && aligned16(dout) && aligned16(du) && aligned16(ddelta) &&
                    aligned16(dz) && aligned16(B) && aligned16(C) && aligned16(dB) && aligned16(dC);
  const float* ck = ckpt;
  if (!ck && pcbc) {
    ssm::FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.A = A; a.dt_bias = dt_bias; a.h0 = h0;
    a.ckpt = ck_ws;
    a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
    a.chunk_len = (int)nblk * ssm::kBlk; a.nchunk = 1;
    a.softplus = delta_softplus ? 1 : 0;
    a.bc_groups = bc_groups;
    if ((e = ssm::launch_fwd_pcbc(a, io_dtype, pvec, ssm::kFwdCkpt, s)) != cudaSuccess)
      return cuda_fail(e, "backward state replay pass (B/C per channel)");
    ck = ck_ws;
  }
  if (!ck) {
    ssm::FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.A = A; a.dt_bias = dt_bias; a.h0 = h0;
    a.ckpt = ck_ws;
    a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
    a.chunk_len = (int)nblk * ssm::kBlk; a.nchunk = 1;
    a.softplus = delta_softplus ? 1 : 0;
    a.reverse = reverse ? 1 : 0;
    a.zoh = zoh ? 1 : 0;
    a.bc_groups = bc_groups;
    a.channels_last = channels_last ? 1 : 0;
    const bool lane = fwd_lane_allowed() && vec && !reverse && !zoh &&
                      (bc_groups == 1 || (dim / bc_groups) % 32 == 0);
    a.lpc = lane ? 1 : ((zoh || bc_groups > 1) ? 2 : fwd_lpc());
    a.warps_per_b = (dim + fwd_chw(lane) - 1) / fwd_chw(lane);
    if (!lane) a.warps_per_b = (dim + 32 / a.lpc - 1) / (32 / a.lpc);
    a.nwarps = (long long)batch * a.warps_per_b;
    // with few channels the replay takes the forward's time split (summary, carry, replay)
    FwdPlan plan = plan_fwd(batch, dim, seqlen, fwd_chw(lane));
    if (plan.nchunk > 1 && plan.ws_bytes > l.fwd_ws) {
      plan.nchunk = 1;
      plan.chunk_len = (int)nblk * ssm::kBlk;
    }
    a.chunk_len = plan.chunk_len;
    a.nchunk = plan.nchunk;
    const int km = fwd_kmufu(a.nwarps * (long long)plan.nchunk);
    if (plan.nchunk > 1) {
      float* summ = reinterpret_cast<float*>(fwd_ws);
      float* hin = reinterpret_cast<float*>(fwd_ws + align_up(plan.nchunk * nch * ssm::kNS * 4));
      float* dsum = reinterpret_cast<float*>(fwd_ws + 2 * align_up(plan.nchunk * nch * ssm::kNS * 4));
      ssm::FwdArgs as = a;
      as.summ = summ; as.dsum = dsum;
      as.ckpt = nullptr; as.h0 = nullptr;
      e = lane ? ssm::launch_fwd_lane(as, io_dtype, ssm::kFwdSummary, km, s)
               : ssm::launch_fwd(as, io_dtype, vec, ssm::kFwdSummary, fwd_wpb(), km, s);
      if (e != cudaSuccess) return cuda_fail(e, "backward replay summary pass");
      if ((e = ssm::launch_fwd_carry(a, summ, dsum, hin, s)) != cudaSuccess)
        return cuda_fail(e, "backward replay carry pass");
      a.hin = hin;
    }
    e = lane ? ssm::launch_fwd_lane(a, io_dtype, ssm::kFwdCkpt, km, s)
             : ssm::launch_fwd(a, io_dtype, vec, ssm::kFwdCkpt, fwd_wpb(), km, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward state replay pass");
    ck = ck_ws;
  }
  ssm::BwdArgs b;
  memset(&b, 0, sizeof(b));
  b.u = u; b.delta = delta; b.z = z; b.B = B; b.C = C; b.A = A; b.D = D; b.dt_bias = dt_bias;
  b.dout = dout; b.dhL = dhL; b.ckpt = ck;
  b.du = du; b.ddelta = ddelta; b.dz = dz; b.dh0 = dh0;
  b.part_bc = part_bc; b.part_adt = part_adt;
  b.batch = batch; b.dim = dim; b.L = seqlen; b.N = dstate;
  b.softplus = delta_softplus ? 1 : 0;
  b.reverse = reverse ? 1 : 0;
  b.zoh = zoh ? 1 : 0;
  b.bc_groups = bc_groups;
  b.channels_last = channels_last ? 1 : 0;
  b.warps_per_b = (dim + 15) / 16;
  b.nwarps = (long long)batch * b.warps_per_b;
  b.wpb = l.wpb;
  b.ngroups = l.ngroups;
  b.kmufu = env_int("SSM_BWD_KMUFU", 4);  // all exponentials on MUFU measured fastest
  if (pcbc) {
    if ((e = ssm::launch_bwd_pcbc(b, io_dtype, pvec, dB, dC, s)) != cudaSuccess)
      return cuda_fail(e, "backward pass (B/C per channel)");
    if ((e = ssm::launch_bwd_finish_adt(b, dA, dD, ddt_bias, s)) != cudaSuccess)
      return cuda_fail(e, "backward reduction");
    return SSM_OK;
  }
  // the default variant with N = 16 and rows of whole 8-step pieces: the state history in
  // registers (ssm_bwd_hist.cu); SSM_BWD_KERNEL=pair forces the general kernel
  const char* bk = getenv("SSM_BWD_KERNEL");
  bool hist = !(bk && strcmp(bk, "pair") == 0) && vec && !reverse && !zoh && !channels_last &&
              dstate == ssm::kNS && seqlen % 8 == 0 && aligned16(ck) && aligned16(dhL) &&
              aligned16(dh0);
  if (hist) {
    int w = env_int("SSM_BWD_WPB", 0);
    if (w != 2 && w != 4) w = ssm::bwd_hist_pick_wpb(io_dtype, batch, dim);
    if (bc_groups > 1 && (dim / bc_groups) % (16 * w) != 0) w = 2;
    if (bc_groups > 1 && (dim / bc_groups) % (16 * w) != 0) hist = false;
    if (hist) {
      b.wpb = w;
      b.ngroups = (b.warps_per_b + w - 1) / w;
      // time split when the CTAs fill less than a wave: adjoint summaries of chunks 1 .. S-1,
      // chained from dhL by the carry pass, give each chunk the adjoint entering it
      int bpc = 0;
      int S = plan_bwd_split(batch, dim, seqlen, w, ssm::bwd_hist_ctas_per_sm(io_dtype, w), &bpc);
      if (S > l.nsplit) {
        bpc = (int)((nblk + l.nsplit - 1) / l.nsplit);
        S = (int)((nblk + bpc - 1) / bpc);
      }
      if (S > 1) {
        b.nsplit = S;
        b.blk_per_chunk = bpc;
        const size_t sz = align_up((size_t)l.nsplit * nch * ssm::kNS * 4);
        float* summ = reinterpret_cast<float*>(split_ws);
        float* lam_in = reinterpret_cast<float*>(split_ws + sz);
        float* dsum = reinterpret_cast<float*>(split_ws + 2 * sz);
        if ((e = ssm::launch_bwd_summary(b, io_dtype, summ, dsum, s)) != cudaSuccess)
          return cuda_fail(e, "backward summary pass");
        ssm::FwdArgs c;
        memset(&c, 0, sizeof(c));
        c.A = A; c.h0 = dhL;
        c.batch = batch; c.dim = dim; c.N = dstate;
        c.nchunk = S;
        if ((e = ssm::launch_fwd_carry(c, summ, dsum, lam_in, s)) != cudaSuccess)
          return cuda_fail(e, "backward carry pass");
        b.lam_in = lam_in;
      }
    }
  }
  e = hist ? ssm::launch_bwd_hist(b, io_dtype, s) : ssm::launch_bwd(b, io_dtype, vec, s);
  if (e != cudaSuccess) return cuda_fail(e, "backward pass");
  if ((e = ssm::launch_bwd_finish(b, io_dtype, dB, dC, dA, dD, ddt_bias, s)) != cudaSuccess)
    return cuda_fail(e, "backward reduction");
  return SSM_OK;
}

}  // namespace

namespace {

// The chunked-form backward of scalar decay (bf16, N = 16..128, forward direction, default
// layout, B/C shared by whole 64-channel tiles, no checkpoints given): the forward's checkpoint
// pass (with its own time split), the backward kernel, and the finishing sums.
bool chunked_bwd_ok(int dim, int dstate, int bc_groups, int io_dtype, int flags) {
  const char* v = getenv("SSM_SCALAR_BWD");  // "slices" / "state": the per-state kernels
  if (v && (strcmp(v, "slices") == 0 || strcmp(v, "state") == 0)) return false;
  return io_dtype == SSM_BF16 && (flags & ~(SSM_REVERSE | SSM_ZOH)) == SSM_SCALAR_A &&
         (dstate == 16 || dstate == 32 || dstate == 64 || dstate == 128) &&
         (bc_groups == 1 || (bc_groups < dim && dim % bc_groups == 0 && (dim / bc_groups) % 64 == 0));
}

// Time split of the chunked backward: when its CTAs (batch rows x 64-channel tiles) fill at most
// half of the resident slots (two per SM; one at N = 128, whose CTA takes most of an SM's shared
// memory), the chunks are cut into as many segments as still fit in one wave, each of at least 16
// chunks, and walked side by side from their chained adjoints (SSM_SSD_BWD_SPLIT overrides the
// segment count).  A grid that already fills most of a wave is not split: a second wave and the
// summary launch would cost more than the idle slots.
struct BwdSegPlan {
  int nseg, cps;  // segments, chunks per segment
};
BwdSegPlan plan_ssd_bwd(int batch, int dim, int seqlen, int dstate) {
  const int nck = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  const long long ctas = (long long)batch * ssm::ssd_bwd_ctas_per_row(dim);
  const long long target = (long long)sm_count() * (dstate >= 128 ? 1 : 2);
  const int forced = env_int("SSM_SSD_BWD_SPLIT", 0);
  int S = forced;
  if (S <= 0) {
    S = (int)(target / ctas);  // whole segments per channel tile within one wave
    S = S < nck / 16 ? S : (nck / 16 > 1 ? nck / 16 : 1);
  }
  S = S < 1 ? 1 : (S > nck ? nck : S);
  BwdSegPlan p;
  p.cps = (nck + S - 1) / S;
  p.nseg = (nck + p.cps - 1) / p.cps;
  return p;
}

struct ChunkedBwdLayout {
  size_t mir, ck, pbc, padt, musum, dsum, muin, fwd, total;
  BwdSegPlan seg;
};

// have_ckpt: the caller passes the forward's checkpoints (no checkpoint pass, no room for them);
// reverse: room for the inputs mirrored along time at the start
ChunkedBwdLayout chunked_bwd_layout(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                    bool have_ckpt, bool reverse) {
  ChunkedBwdLayout l;
  l.seg = plan_ssd_bwd(batch, dim, seqlen, dstate);
  l.mir = reverse ? mirror_bytes(batch, dim, seqlen, dstate, bc_groups, 4) : 0;
  const size_t nch = (size_t)batch * dim, S = (size_t)l.seg.nseg;
  const size_t nck = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  l.ck = have_ckpt ? 0 : align_up(nch * nck * dstate * 4);
  l.pbc = align_up((size_t)ssm::ssd_bwd_ctas_per_row(dim) * batch * 2 * dstate * seqlen * 4);
  l.padt = align_up(S * nch * 3 * 4);
  l.musum = S > 1 ? align_up(S * nch * dstate * 4) : 0;
  l.dsum = S > 1 ? align_up(S * nch * 4) : 0;
  l.muin = l.musum;
  l.fwd = have_ckpt ? 0 : plan_ssd(batch, dim, seqlen, dstate).ws_bytes;
  l.total = l.mir + l.ck + l.pbc + l.padt + l.musum + l.dsum + l.muin + l.fwd;
  return l;
}

int scan_bwd_chunked(const void* u, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* dt_bias,
                     int delta_softplus, const float* h0, const void* dout, const float* dhL,
                     const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                     float* ddt_bias, float* dh0, void* workspace, size_t workspace_bytes,
                     int batch, int dim, int seqlen, int dstate, int bc_groups, bool reverse,
                     bool zoh, void* stream) {
  const size_t es = 2;
  const size_t nx = (size_t)batch * dim * seqlen * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * es;
  const size_t nst = (size_t)batch * dim * dstate * 4;
  TRY(check_ptr(u, nx, es, "u"));
  TRY(check_ptr(delta, nx, es, "delta"));
  TRY(check_ptr(A, (size_t)dim * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_ptr(dout, nx, es, "dout"));
  TRY(check_opt(D, (size_t)dim * 4, 4, "D"));
  TRY(check_opt(z, nx, es, "z"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  TRY(check_opt(h0, nst, 4, "h0"));
  TRY(check_opt(dhL, nst, 4, "dhL"));
  TRY(check_opt(du, nx, es, "du"));
  TRY(check_opt(ddelta, nx, es, "ddelta"));
  TRY(check_opt(dz, nx, es, "dz"));
  TRY(check_opt(dB, nbc, es, "dB"));
  TRY(check_opt(dC, nbc, es, "dC"));
  TRY(check_opt(dA, (size_t)dim * 4, 4, "dA"));
  TRY(check_opt(dD, (size_t)dim * 4, 4, "dD"));
  TRY(check_opt(ddt_bias, (size_t)dim * 4, 4, "ddt_bias"));
  TRY(check_opt(dh0, nst, 4, "dh0"));
  const size_t nck = (seqlen + ssm::kBlk - 1) / ssm::kBlk;
  TRY(check_opt(ckpt, (size_t)batch * dim * nck * dstate * 4, 4, "ckpt"));
  if (!aligned16(ckpt))
    return fail(SSM_EINVAL, "ckpt must be 16-byte aligned (chunked matrix form)");
  if (!du && !ddelta && !dA && !dB && !dC && !dD && !dz && !ddt_bias && !dh0)
    return fail(SSM_EINVAL, "no gradient output requested");
  if (dz && !z) return fail(SSM_EINVAL, "dz requested but z is NULL");
  const ChunkedBwdLayout l =
      chunked_bwd_layout(batch, dim, seqlen, dstate, bc_groups, ckpt != nullptr, reverse);
  if (!workspace || workspace_bytes < l.total)
    return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, l.total);
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  TRY(check_ptr(workspace, l.total, 256, "workspace"));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  // reverse: the kernels scan the inputs mirrored along time; the gradients along time are
  // mirrored back in place at the end
  if (reverse) {
    char* m = reinterpret_cast<char*>(workspace);
    const long long rx = (long long)batch * dim, rbc = (long long)batch * bc_groups * dstate;
    void* mu = m;
    void* md = m + align_up(nx);
    void* mz = z ? m + 2 * align_up(nx) : nullptr;
    void* mo = m + 3 * align_up(nx);
    void* mB = m + 4 * align_up(nx);
    void* mC = m + 4 * align_up(nx) + align_up(nbc);
    if ((e = ssm::mirror_rows(u, mu, rx, seqlen, s)) != cudaSuccess ||
        (e = ssm::mirror_rows(delta, md, rx, seqlen, s)) != cudaSuccess ||
        (z && (e = ssm::mirror_rows(z, mz, rx, seqlen, s)) != cudaSuccess) ||
        (e = ssm::mirror_rows(dout, mo, rx, seqlen, s)) != cudaSuccess ||
        (e = ssm::mirror_rows(B, mB, rbc, seqlen, s)) != cudaSuccess ||
        (e = ssm::mirror_rows(C, mC, rbc, seqlen, s)) != cudaSuccess)
      return cuda_fail(e, "reverse scan backward: mirrored inputs");
    u = mu; delta = md; z = mz; dout = mo; B = mB; C = mC;
  }
  char* w = reinterpret_cast<char*>(workspace) + l.mir;
  float* ck = ckpt ? nullptr : reinterpret_cast<float*>(w);
  float* pbc = reinterpret_cast<float*>(w + l.ck);
  float* padt = reinterpret_cast<float*>(w + l.ck + l.pbc);
  float* musum = reinterpret_cast<float*>(w + l.ck + l.pbc + l.padt);
  float* dsum = reinterpret_cast<float*>(w + l.ck + l.pbc + l.padt + l.musum);
  float* muin = reinterpret_cast<float*>(w + l.ck + l.pbc + l.padt + l.musum + l.dsum);
  char* fws = w + l.ck + l.pbc + l.padt + l.musum + l.dsum + l.muin;
  const bool vec = (seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) && aligned16(z) &&
                   aligned16(B) && aligned16(C) && aligned16(dout);
  if (!ckpt) {
    // the state entering every chunk, from the forward in checkpoint mode
    ssm::FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
    a.A = A; a.dt_bias = dt_bias; a.h0 = h0;
    a.ckpt = ck;  // the state entering every chunk
    a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
    a.softplus = delta_softplus ? 1 : 0;
    a.scalar_a = 1;
    a.zoh = zoh ? 1 : 0;
    a.bc_groups = bc_groups;
    a.rows16 = vec ? 1 : 0;
    const FwdPlan plan = plan_ssd(batch, dim, seqlen, dstate);
    a.chunk_len = plan.chunk_len;
    a.nchunk = plan.nchunk;
    if (plan.nchunk > 1) {
      const size_t nch = (size_t)batch * dim;
      const size_t seg = align_up((size_t)plan.nchunk * nch * dstate * 4);
      a.summ = reinterpret_cast<float*>(fws);
      float* hin = reinterpret_cast<float*>(fws + seg);
      a.dsum = reinterpret_cast<float*>(fws + 2 * seg);
      if ((e = ssm::launch_ssd_fwd(a, ssm::kSsdSummary, s)) != cudaSuccess)
        return cuda_fail(e, "backward: summary pass (chunked matrix form)");
      const long long n = (long long)nch * dstate;
      chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.summ, a.dsum, A, 1, h0, hin,
                                                               plan.nchunk, (long long)nch, dim,
                                                               dstate);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward: carry");
      a.hin = hin;
    }
    if ((e = ssm::launch_ssd_fwd(a, ssm::kSsdCkpt, s)) != cudaSuccess)
      return cuda_fail(e, "backward: checkpoint pass (chunked matrix form)");
  }
  ssm::SsdBwdArgs b;
  memset(&b, 0, sizeof(b));
  b.u = reinterpret_cast<const uint16_t*>(u);
  b.delta = reinterpret_cast<const uint16_t*>(delta);
  b.z = reinterpret_cast<const uint16_t*>(z);
  b.B = reinterpret_cast<const uint16_t*>(B);
  b.C = reinterpret_cast<const uint16_t*>(C);
  b.dout = reinterpret_cast<const uint16_t*>(dout);
  b.A = A; b.D = D; b.dt_bias = dt_bias; b.dhL = dhL;
  b.ck = ckpt ? ckpt : ck;
  b.du = reinterpret_cast<uint16_t*>(du);
  b.ddelta = reinterpret_cast<uint16_t*>(ddelta);
  b.dz = reinterpret_cast<uint16_t*>(dz);
  b.dh0 = dh0;
  b.part_bc = pbc;
  b.part_adt = padt;
  b.batch = batch; b.dim = dim; b.L = seqlen; b.N = dstate; b.bc_groups = bc_groups;
  b.softplus = delta_softplus ? 1 : 0;
  b.rows16 = vec ? 1 : 0;
  b.need_bc = (dB || dC) ? 1 : 0;
  b.zoh = zoh ? 1 : 0;
  b.nseg = l.seg.nseg;
  b.cps = l.seg.cps;
  if (l.seg.nseg > 1) {
    // each segment's adjoint from zero at its end, then the chain of the segments in reverse
    b.mu_sum = musum;
    b.dsum = dsum;
    b.mu_in = muin;
    if ((e = ssm::launch_ssd_bwd(b, true, s)) != cudaSuccess)
      return cuda_fail(e, "backward: segment summaries (chunked matrix form)");
    const long long nch = (long long)batch * dim, n = nch * dstate;
    chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(musum, dsum, A, 1, dhL, muin,
                                                             l.seg.nseg, nch, dim, dstate);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward: adjoint chain");
  }
  if ((e = ssm::launch_ssd_bwd(b, false, s)) != cudaSuccess)
    return cuda_fail(e, "backward pass (chunked matrix form)");
  if ((e = ssm::launch_ssd_bwd_finish(b, dB, dC, dA, dD, ddt_bias, s)) != cudaSuccess)
    return cuda_fail(e, "backward reduction (chunked matrix form)");
  if (reverse) {
    const long long rx = (long long)batch * dim, rbc = (long long)batch * bc_groups * dstate;
    void* along[5] = {du, ddelta, dz, dB, dC};
    const long long rows[5] = {rx, rx, rx, rbc, rbc};
    for (int k = 0; k < 5; ++k)
      if (along[k] && (e = ssm::mirror_rows(along[k], along[k], rows[k], seqlen, s)) != cudaSuccess)
        return cuda_fail(e, "reverse scan backward: mirrored gradients");
  }
  return SSM_OK;
}

}  // namespace

extern "C" {

int ssm_scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                 const float* D, const void* z, const float* dt_bias, int delta_softplus,
                 const float* h0, const void* dout, const float* dhL, const float* ckpt,
                 void* du, void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                 float* ddt_bias, float* dh0, void* workspace, size_t workspace_bytes,
                 int batch, int dim, int seqlen, int dstate, int io_dtype, void* stream) {
  g_err[0] = 0;
  return scan_bwd_core(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL, ckpt, du,
                       ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace, workspace_bytes,
                       batch, dim, seqlen, dstate, io_dtype, stream, false, false, 1);
}

size_t ssm_scan_bwd_ex_workspace_size(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                      int io_dtype, int have_ckpt, int flags) {
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH | SSM_CHANNELS_LAST)) return 0;
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE) {  // chunked form, or slices
    if (chunked_bwd_ok(dim, dstate, bc_groups, io_dtype, flags))
      return chunked_bwd_layout(batch, dim, seqlen, dstate, bc_groups, have_ckpt != 0,
                                (flags & SSM_REVERSE) != 0).total;
    if (have_ckpt) return 0;
    return ssm::scan_bwd_slices_workspace(batch, dim, seqlen, dstate, bc_groups, io_dtype, flags);
  }
  if (dstate == 16 && chunked_bwd_ok(dim, dstate, bc_groups, io_dtype, flags)) {
    if (check_dims(batch, dim, seqlen, dstate, io_dtype) != SSM_OK) return 0;
    return chunked_bwd_layout(batch, dim, seqlen, dstate, bc_groups, have_ckpt != 0,
                              (flags & SSM_REVERSE) != 0).total;
  }
  if (check_dims(batch, dim, seqlen, dstate, io_dtype) != SSM_OK) return 0;
  if (check_groups(dim, bc_groups) != SSM_OK) return 0;
  const size_t base = layout_bwd(batch, dim, seqlen, dstate, have_ckpt != 0, bc_groups, io_dtype,
                                 flags & ~SSM_SCALAR_A).total;
  if (base == 0 || !(flags & SSM_SCALAR_A)) return base;
  return align_up((size_t)dim * dstate * 4) * 2 + base;
}

int ssm_scan_bwd_ex(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, const void* dout, const float* dhL,
                    const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC,
                    float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                    size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                    int bc_groups, int io_dtype, int flags, void* stream) {
  g_err[0] = 0;
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH | SSM_CHANNELS_LAST))
    return fail(SSM_EINVAL, "unknown flags 0x%x", flags);
  const bool reverse = (flags & SSM_REVERSE) != 0, zoh = (flags & SSM_ZOH) != 0;
  const bool cl = (flags & SSM_CHANNELS_LAST) != 0;
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE) {  // chunked form, or slices
    TRY(check_dims(batch, dim, seqlen, dstate, io_dtype, SSM_MAX_DSTATE_SCALAR));
    TRY(check_groups(dim, bc_groups));
    if (chunked_bwd_ok(dim, dstate, bc_groups, io_dtype, flags))
      return scan_bwd_chunked(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL,
                              ckpt, du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace,
                              workspace_bytes, batch, dim, seqlen, dstate, bc_groups, reverse,
                              zoh, stream);
    return ssm::scan_bwd_slices(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL,
                                ckpt, du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace,
                                workspace_bytes, batch, dim, seqlen, dstate, bc_groups, io_dtype,
                                flags, stream);
  }
  TRY(check_dims(batch, dim, seqlen, dstate, io_dtype));
  if (dstate == 16 && chunked_bwd_ok(dim, dstate, bc_groups, io_dtype, flags)) {
    TRY(check_groups(dim, bc_groups));
    return scan_bwd_chunked(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL, ckpt,
                            du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace,
                            workspace_bytes, batch, dim, seqlen, dstate, bc_groups, reverse,
                            zoh, stream);
  }
  if (!(flags & SSM_SCALAR_A))
    return scan_bwd_core(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL, ckpt,
                         du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace,
                         workspace_bytes, batch, dim, seqlen, dstate, io_dtype, stream, reverse,
                         zoh, bc_groups, cl);
  // scalar decay: broadcast A over the states, run the per-state backward, sum dA over n
  TRY(check_ptr(A, (size_t)dim * 4, 4, "A"));
  TRY(check_opt(dA, (size_t)dim * 4, 4, "dA"));
  const size_t head = align_up((size_t)dim * dstate * 4);
  const size_t need = ssm_scan_bwd_ex_workspace_size(batch, dim, seqlen, dstate, bc_groups,
                                                     io_dtype, ckpt != nullptr, flags);
  if (!workspace || workspace_bytes < need)
    return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  TRY(check_ptr(workspace, need, 256, "workspace"));
  char* w = reinterpret_cast<char*>(workspace);
  float* Af = reinterpret_cast<float*>(w);          // A broadcast to [dim][dstate]
  float* dAf = reinterpret_cast<float*>(w + head);  // dA per state, summed into dA[d] at the end
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long n = (long long)dim * dstate;
  broadcast_a_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(A, Af, dim, dstate);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decay broadcast");
  const int rc = scan_bwd_core(u, delta, Af, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL,
                               ckpt, du, ddelta, dA ? dAf : nullptr, dB, dC, dD, dz, ddt_bias,
                               dh0, w + 2 * head, workspace_bytes - 2 * head, batch, dim, seqlen,
                               dstate, io_dtype, stream, reverse, zoh, bc_groups, cl);
  if (rc != SSM_OK) return rc;
  if (dA) {
    reduce_da_kernel<<<(unsigned)((dim + 255) / 256), 256, 0, s>>>(dAf, dA, dim, dstate);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "decay gradient sum");
  }
  return SSM_OK;
}

size_t ssm_scan_bwd_scalar_a_workspace_size(int batch, int dim, int seqlen, int dstate,
                                            int io_dtype, int have_ckpt) {
  return ssm_scan_bwd_ex_workspace_size(batch, dim, seqlen, dstate, 1, io_dtype, have_ckpt,
                                        SSM_SCALAR_A);
}

int ssm_scan_bwd_scalar_a(const void* u, const void* delta, const float* A, const void* B,
                          const void* C, const float* D, const void* z, const float* dt_bias,
                          int delta_softplus, const float* h0, const void* dout, const float* dhL,
                          const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC,
                          float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                          size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                          int io_dtype, void* stream) {
  return ssm_scan_bwd_ex(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, dout, dhL, ckpt,
                         du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, workspace, workspace_bytes,
                         batch, dim, seqlen, dstate, 1, io_dtype, SSM_SCALAR_A, stream);
}

// Whole-sequence summary of the forward scan (the segment map of a sequence split across GPUs):
// the state after the sequence from a zero state and each channel's ΣΔ.  Runs the forward's
// summary pass over the planner's time chunks (one more chunk slot than chunks, so the carry
// pass's last entering state is the sequence's end state), the carry pass from zero, and a
// finishing kernel.
size_t ssm_scan_fwd_summary_workspace_size(int batch, int dim, int seqlen, int dstate,
                                           int bc_groups, int io_dtype, int flags) {
  if (flags & ~(SSM_SCALAR_A | SSM_ZOH)) return 0;
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE) {
    if (check_dims(batch, dim, seqlen, dstate, io_dtype, SSM_MAX_DSTATE_SCALAR) != SSM_OK ||
        check_groups(dim, bc_groups) != SSM_OK)
      return 0;
    if (io_dtype == SSM_F32)
      return ssm::scan_summary_slices_workspace(batch, dim, seqlen, dstate, bc_groups, flags);
    if (dstate != 32 && dstate != 64 && dstate != 128) return 0;
    return summary_chunked_layout(batch, dim, seqlen, dstate).total;
  }
  if (check_dims(batch, dim, seqlen, dstate, io_dtype) != SSM_OK) return 0;
  if (check_groups(dim, bc_groups) != SSM_OK) return 0;
  return plan_summary(batch, dim, seqlen).ws_bytes;
}

int ssm_scan_fwd_summary(const void* u, const void* delta, const float* A, const void* B,
                         const void* C, const float* dt_bias, int delta_softplus, float* hend,
                         float* dsum, void* workspace, size_t workspace_bytes, int batch,
                         int dim, int seqlen, int dstate, int bc_groups, int io_dtype, int flags,
                         void* stream) {
  g_err[0] = 0;
  if (flags & ~(SSM_SCALAR_A | SSM_ZOH))
    return fail(SSM_EINVAL, "unsupported flags 0x%x for a sequence summary", flags);
  if ((flags & SSM_SCALAR_A) && dstate > SSM_MAX_DSTATE) {
    TRY(check_dims(batch, dim, seqlen, dstate, io_dtype, SSM_MAX_DSTATE_SCALAR));
    TRY(check_groups(dim, bc_groups));
    if (io_dtype == SSM_F32)
      return ssm::scan_summary_slices(u, delta, A, B, C, dt_bias, delta_softplus, hend, dsum,
                                      workspace, workspace_bytes, batch, dim, seqlen, dstate,
                                      bc_groups, flags, stream);
    return summary_chunked(u, delta, A, B, C, dt_bias, delta_softplus, hend, dsum, workspace,
                           workspace_bytes, batch, dim, seqlen, dstate, bc_groups, flags, stream);
  }
  TRY(check_dims(batch, dim, seqlen, dstate, io_dtype));
  TRY(check_groups(dim, bc_groups));
  if (bc_groups == dim && bc_groups > 1)
    return fail(SSM_EUNSUPPORTED, "sequence summaries take shared or grouped B/C");
  const bool scalar_a = (flags & SSM_SCALAR_A) != 0;
  const size_t es = esize(io_dtype);
  const size_t nx = (size_t)batch * dim * seqlen * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * seqlen * es;
  const size_t nch = (size_t)batch * dim;
  TRY(check_ptr(u, nx, es, "u"));
  TRY(check_ptr(delta, nx, es, "delta"));
  TRY(check_ptr(A, (size_t)dim * (scalar_a ? 1 : dstate) * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  TRY(check_ptr(hend, nch * dstate * 4, 4, "hend"));
  TRY(check_opt(dsum, nch * 4, 4, "dsum"));
  const FwdPlan plan = plan_summary(batch, dim, seqlen);
  if (!workspace || workspace_bytes < plan.ws_bytes)
    return fail(SSM_EWORKSPACE, "workspace of %zu bytes given, %zu needed", workspace_bytes,
                plan.ws_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  TRY(check_ptr(workspace, plan.ws_bytes, 256, "workspace"));
  const int S = plan.nchunk;
  const size_t slots = (size_t)S + 1;
  char* w = reinterpret_cast<char*>(workspace);
  float* summ = reinterpret_cast<float*>(w);
  float* hin = reinterpret_cast<float*>(w + align_up(slots * nch * ssm::kNS * 4));
  float* ds = reinterpret_cast<float*>(w + 2 * align_up(slots * nch * ssm::kNS * 4));
  const bool vec = (seqlen * es) % 16 == 0 && aligned16(u) && aligned16(delta) && aligned16(B) &&
                   aligned16(C);
  ssm::FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.u = u; a.delta = delta; a.B = B; a.C = C; a.A = A; a.dt_bias = dt_bias;
  a.summ = summ; a.dsum = ds;
  a.batch = batch; a.dim = dim; a.L = seqlen; a.N = dstate;
  a.chunk_len = plan.chunk_len;
  a.nchunk = S + 1;  // the summary pass covers chunks 0 .. S-1, every one of the sequence
  a.softplus = delta_softplus ? 1 : 0;
  a.scalar_a = scalar_a ? 1 : 0;
  a.zoh = (flags & SSM_ZOH) ? 1 : 0;
  a.bc_groups = bc_groups;
  a.lpc = 2;
  a.warps_per_b = (dim + 15) / 16;
  a.nwarps = (long long)batch * a.warps_per_b;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ssm::launch_fwd(a, io_dtype, vec, ssm::kFwdSummary, fwd_wpb(),
                                  fwd_kmufu(a.nwarps * (long long)S), s);
  if (e != cudaSuccess) return cuda_fail(e, "sequence summary pass");
  if ((e = ssm::launch_fwd_carry(a, summ, ds, hin, s)) != cudaSuccess)
    return cuda_fail(e, "sequence summary carry");
  const long long n = (long long)nch * dstate;
  summary_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      hin + (size_t)S * nch * ssm::kNS, ssm::kNS, ds, S, (long long)nch, dstate, hend, dsum);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "sequence summary finish");
  return SSM_OK;
}

int ssm_scan_chain(const float* hend, const float* dsum, const float* A, const float* h0,
                   float* hin, int nseg, int batch, int dim, int dstate, int flags, void* stream) {
  g_err[0] = 0;
  if (flags & ~SSM_SCALAR_A) return fail(SSM_EINVAL, "unsupported flags 0x%x for a chain", flags);
  if (nseg <= 0) return fail(SSM_EINVAL, "nseg must be positive, got %d", nseg);
  const bool scalar_a = (flags & SSM_SCALAR_A) != 0;
  TRY(check_dims(batch, dim, 1, dstate, SSM_F32, scalar_a ? SSM_MAX_DSTATE_SCALAR : SSM_MAX_DSTATE));
  const size_t nch = (size_t)batch * dim;
  TRY(check_ptr(hend, (size_t)nseg * nch * dstate * 4, 4, "hend"));
  TRY(check_ptr(dsum, (size_t)nseg * nch * 4, 4, "dsum"));
  TRY(check_ptr(A, (size_t)dim * (scalar_a ? 1 : dstate) * 4, 4, "A"));
  TRY(check_opt(h0, nch * dstate * 4, 4, "h0"));
  TRY(check_ptr(hin, (size_t)nseg * nch * dstate * 4, 4, "hin"));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long n = (long long)nch * dstate;
  chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(hend, dsum, A, scalar_a ? 1 : 0, h0,
                                                           hin, nseg, (long long)nch, dim, dstate);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "segment chain");
  return SSM_OK;
}

int ssm_state_update_ex(float* state, const void* x, const void* dt, const float* A,
                        const void* B, const void* C, const float* D, const void* z,
                        const float* dt_bias, int delta_softplus, void* out, int batch, int dim,
                        int dstate, int bc_groups, int io_dtype, int flags, void* stream) {
  g_err[0] = 0;
  if (flags & ~(SSM_SCALAR_A | SSM_ZOH))
    return fail(SSM_EINVAL, "unsupported flags 0x%x for a decode step", flags);
  const bool scalar_a = (flags & SSM_SCALAR_A) != 0;
  // one rate per channel also takes N = 32, 64 or 128 (the chunked scan's state sizes)
  TRY(check_dims(batch, dim, 1, dstate, io_dtype, scalar_a ? SSM_MAX_DSTATE_SCALAR : SSM_MAX_DSTATE));
  TRY(check_groups(dim, bc_groups));
  if (dstate > SSM_MAX_DSTATE) {
    if (dstate != 32 && dstate != 64 && dstate != 128)
      return fail(SSM_EUNSUPPORTED, "a decode step with dstate %d > %d takes 32, 64 or 128",
                  dstate, SSM_MAX_DSTATE);
    if (!aligned16(state)) return fail(SSM_EINVAL, "state must be 16-byte aligned for dstate > 16");
  }
  const size_t es = esize(io_dtype);
  const size_t nx = (size_t)batch * dim * es;
  const size_t nbc = (size_t)batch * bc_groups * dstate * es;
  TRY(check_ptr(state, (size_t)batch * dim * dstate * 4, 4, "state"));
  TRY(check_ptr(x, nx, es, "x"));
  TRY(check_ptr(dt, nx, es, "dt"));
  TRY(check_ptr(A, (size_t)dim * (scalar_a ? 1 : dstate) * 4, 4, "A"));
  TRY(check_ptr(B, nbc, es, "B"));
  TRY(check_ptr(C, nbc, es, "C"));
  TRY(check_ptr(out, nx, es, "out"));
  TRY(check_opt(D, (size_t)dim * 4, 4, "D"));
  TRY(check_opt(z, nx, es, "z"));
  TRY(check_opt(dt_bias, (size_t)dim * 4, 4, "dt_bias"));
  ssm::DecodeArgs a;
  a.state = state; a.x = x; a.dt = dt; a.z = z; a.B = B; a.C = C; a.A = A; a.D = D;
  a.dt_bias = dt_bias; a.out = out;
  a.batch = batch; a.dim = dim; a.N = dstate; a.softplus = delta_softplus ? 1 : 0;
  a.scalar_a = scalar_a ? 1 : 0;
  a.zoh = (flags & SSM_ZOH) ? 1 : 0;
  a.bc_groups = bc_groups;
  cudaError_t e = ssm::launch_decode(a, io_dtype, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode step");
  return SSM_OK;
}

int ssm_wait_timeouts(unsigned int* count) {
  g_err[0] = 0;
  if (!count) return fail(SSM_EINVAL, "count is NULL");
  if (ssm::decode_wait_timeouts(count) != 0) {
    cudaError_t e = cudaGetLastError();
    return cuda_fail(e, "reading the wait-timeout counter");
  }
  return SSM_OK;
}

int ssm_state_update(float* state, const void* x, const void* dt, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* dt_bias,
                     int delta_softplus, void* out, int batch, int dim, int dstate,
                     int io_dtype, void* stream) {
  return ssm_state_update_ex(state, x, dt, A, B, C, D, z, dt_bias, delta_softplus, out, batch,
                             dim, dstate, 1, io_dtype, 0, stream);
}

}  // extern "C"
