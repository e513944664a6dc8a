// General element strides for the scan, its backward and the decode step (the *_strided entry
// points of include/ssm_scan.h).  The selective parameters are projections of the input
// ("Seçim Mekanizması (S6)" on the Mamba summary page), so callers hold u, delta, z, B and C as
// views of whatever layout their projections produce.  An io tensor whose strides are the dense
// ones is handed to the dense entry points in place; any other is gathered into a dense copy in
// the workspace (outputs: computed there and scattered back) by one copy kernel on the same
// stream, so results equal the dense calls' bitwise.  The copies cost one read and one write of
// each strided tensor: this is the compatibility path, the dense layouts are the fast one.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>

#include "../../include/ssm_scan.h"
#include "ssm_kernels.h"

namespace ssm {
namespace {

// A logical 4-index view: sizes n and element strides s (leading indices padded with n = 1).
struct View4 {
  long long n[4];
  long long s[4];
};

struct Copy4 {
  long long n[4];
  long long ss[4];  // source strides
  long long ds[4];  // destination strides
  int sub;          // rows of the innermost index per CTA (a power of two)
  int width;        // threads per row (blockDim.x / sub)
};

// dst[i0, i1, i2, i3] = src[i0, i1, i2, i3] under the two stride sets.  Each CTA copies `sub`
// rows of the innermost index at a time (several short rows share one CTA), row after row.
template <typename T>
__global__ void restride_kernel(const T* __restrict__ src, T* __restrict__ dst, const Copy4 c) {
  const long long rows = c.n[0] * c.n[1] * c.n[2];
  const int r_in = threadIdx.x / c.width, lane = threadIdx.x % c.width;
  for (long long row = (long long)blockIdx.x * c.sub + r_in; row < rows;
       row += (long long)gridDim.x * c.sub) {
    const long long i2 = row % c.n[2], r1 = row / c.n[2];
    const long long i1 = r1 % c.n[1], i0 = r1 / c.n[1];
    const T* sp = src + i0 * c.ss[0] + i1 * c.ss[1] + i2 * c.ss[2];
    T* dp = dst + i0 * c.ds[0] + i1 * c.ds[1] + i2 * c.ds[2];
    for (long long t = lane; t < c.n[3]; t += c.width) dp[t * c.ds[3]] = sp[t * c.ss[3]];
  }
}

View4 view(int rank, const long long* n, const long long* s) {
  View4 v;
  const int pad = 4 - rank;
  for (int k = 0; k < 4; ++k) {
    v.n[k] = k < pad ? 1 : n[k - pad];
    v.s[k] = k < pad ? 0 : s[k - pad];
  }
  return v;
}

View4 dense_of(const View4& v) {
  View4 d = v;
  long long e = 1;
  for (int k = 3; k >= 0; --k) {
    d.s[k] = e;
    e *= v.n[k];
  }
  return d;
}

bool is_dense(const View4& v) {
  long long e = 1;
  for (int k = 3; k >= 0; --k) {
    if (v.n[k] > 1 && v.s[k] != e) return false;
    e *= v.n[k];
  }
  return true;
}


// Elements from the first to the last one the view reaches (strides >= 0).
long long extent_of(const View4& v) {
  long long e = 1;
  for (int k = 0; k < 4; ++k) e += (v.n[k] - 1) * v.s[k];
  return e;
}

// No two elements share an address: sorted by stride, each stride exceeds the span of the
// smaller ones.
bool one_to_one(const View4& v) {
  int idx[4], m = 0;
  for (int k = 0; k < 4; ++k)
    if (v.n[k] > 1) idx[m++] = k;
  std::sort(idx, idx + m, [&](int a, int b) { return v.s[a] < v.s[b]; });
  long long span = 0;
  for (int j = 0; j < m; ++j) {
    if (v.s[idx[j]] <= span) return false;
    span += (v.n[idx[j]] - 1) * v.s[idx[j]];
  }
  return true;
}

int fail(int code, const char* fmt, const char* name) {
  char msg[256];
  snprintf(msg, sizeof(msg), fmt, name);
  set_last_error(msg);
  return code;
}

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Validates a strided tensor: strides >= 0, one-to-one for outputs, allocation covers the
// extent.
int check_view(const void* p, const View4& v, size_t es, const char* name, bool output) {
  for (int k = 0; k < 4; ++k)
    if (v.s[k] < 0) return fail(SSM_EINVAL, "%s: negative stride", name);
  if (output && !one_to_one(v))
    return fail(SSM_EINVAL, "%s: output strides map two elements to one address", name);
  return check_device_ptr(p, (size_t)extent_of(v) * es, es, name);
}

cudaError_t restride(const void* src, const View4& sv, void* dst, const View4& dv, size_t es,
                     cudaStream_t s) {
  Copy4 c;
  for (int k = 0; k < 4; ++k) {
    c.n[k] = sv.n[k];
    c.ss[k] = sv.s[k];
    c.ds[k] = dv.s[k];
  }
  int width = 32;
  while (width < 256 && width < c.n[3]) width <<= 1;
  c.width = width;
  c.sub = 256 / width;
  const long long rows = c.n[0] * c.n[1] * c.n[2];
  if (rows == 0 || c.n[3] == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (rows + c.sub - 1) / c.sub;
  const unsigned grid = (unsigned)std::min<long long>(want, 16LL * sms);
  if (es == 2)
    restride_kernel<uint16_t><<<grid, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(src),
                                                   reinterpret_cast<uint16_t*>(dst), c);
  else
    restride_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(src),
                                                reinterpret_cast<float*>(dst), c);
  return cudaGetLastError();
}

// One io tensor of a strided call: where the dense call reads or writes it.
struct Slot {
  const void* user;  // the caller's pointer (NULL: tensor absent)
  View4 v;           // the caller's view
  void* dense;       // what the dense call gets: user itself, or a workspace copy
  bool copy;
};

// Prepares an input: validates, and gathers it into `ws` unless it is dense.
int stage_input(Slot& t, const void* p, const View4& v, size_t es, char* ws, const char* name,
                cudaStream_t s) {
  t.user = p;
  t.v = v;
  t.dense = const_cast<void*>(p);
  t.copy = false;
  if (!p) return SSM_OK;
  int rc = check_view(p, v, es, name, false);
  if (rc != SSM_OK) return rc;
  if (is_dense(v)) return SSM_OK;
  t.dense = ws;
  t.copy = true;
  const cudaError_t e = restride(p, v, ws, dense_of(v), es, s);
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return SSM_ECUDA;
  }
  return SSM_OK;
}

// Prepares an output: validates; the dense call writes to `ws` unless the view is dense.
// `inout`: the tensor is also read (the decode state), so it is gathered first.
int stage_output(Slot& t, void* p, const View4& v, size_t es, char* ws, const char* name,
                 bool inout, cudaStream_t s) {
  t.user = p;
  t.v = v;
  t.dense = p;
  t.copy = false;
  if (!p) return SSM_OK;
  int rc = check_view(p, v, es, name, true);
  if (rc != SSM_OK) return rc;
  if (is_dense(v)) return SSM_OK;
  t.dense = ws;
  t.copy = true;
  if (inout) {
    const cudaError_t e = restride(p, v, ws, dense_of(v), es, s);
    if (e != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return SSM_ECUDA;
    }
  }
  return SSM_OK;
}

int scatter_output(const Slot& t, size_t es, cudaStream_t s) {
  if (!t.user || !t.copy) return SSM_OK;
  const cudaError_t e = restride(t.dense, dense_of(t.v), const_cast<void*>(t.user), t.v, es, s);
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return SSM_ECUDA;
  }
  return SSM_OK;
}

size_t esize(int io) { return io == SSM_BF16 ? 2 : 4; }

bool sizes_ok(long long a, long long b, long long c, long long d) {
  return a > 0 && b > 0 && c > 0 && d > 0;
}

#define TRY(x)                      \
  do {                              \
    const int _rc = (x);            \
    if (_rc != SSM_OK) return _rc;  \
  } while (0)

}  // namespace
}  // namespace ssm

using ssm::Slot;
using ssm::View4;

extern "C" {

size_t ssm_scan_fwd_strided_workspace_size(int batch, int dim, int seqlen, int dstate,
                                           int bc_groups, int io_dtype, int flags) {
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH)) return 0;
  if (!ssm::sizes_ok(batch, dim, seqlen, dstate) || bc_groups < 1) return 0;
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return 0;
  const size_t es = ssm::esize(io_dtype);
  const size_t x = ssm::align_up((size_t)batch * dim * seqlen * es);
  const size_t bc = ssm::align_up((size_t)batch * bc_groups * dstate * seqlen * es);
  const size_t inner = ssm::align_up(
      ssm_scan_fwd_ex_workspace_size(batch, dim, seqlen, dstate, bc_groups, io_dtype, flags));
  return 4 * x + 2 * bc + inner;
}

int ssm_scan_fwd_strided(const void* u, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* dt_bias,
                         int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                         void* workspace, size_t workspace_bytes, int batch, int dim, int seqlen,
                         int dstate, int bc_groups, int io_dtype, int flags,
                         const ssm_strides* st, void* stream) {
  ssm::set_last_error("");
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH))
    return ssm::fail(SSM_EINVAL, "%s", "unsupported flags for a strided call");
  if (!st) return ssm::fail(SSM_EINVAL, "%s", "strides is NULL");
  if (!ssm::sizes_ok(batch, dim, seqlen, dstate) || bc_groups < 1)
    return ssm::fail(SSM_EINVAL, "%s", "sizes must be positive");
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16)
    return ssm::fail(SSM_EINVAL, "%s", "io_dtype is not SSM_F32/SSM_BF16");
  const size_t need = ssm_scan_fwd_strided_workspace_size(batch, dim, seqlen, dstate, bc_groups,
                                                          io_dtype, flags);
  if (!workspace || workspace_bytes < need)
    return ssm::fail(SSM_EWORKSPACE, "%s", "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return ssm::fail(SSM_EINVAL, "%s", "workspace is not 256-byte aligned");
  TRY(ssm::check_device_ptr(workspace, need, 256, "workspace"));
  const size_t es = ssm::esize(io_dtype);
  const size_t x = ssm::align_up((size_t)batch * dim * seqlen * es);
  const size_t bc = ssm::align_up((size_t)batch * bc_groups * dstate * seqlen * es);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nx[3] = {batch, dim, seqlen};
  const long long nbc[4] = {batch, bc_groups, dstate, seqlen};
  if (!u || !delta || !B || !C || !out)
    return ssm::fail(SSM_EINVAL, "%s", "u, delta, B, C and out are required");
  Slot tu, td, tz, to, tB, tC;
  TRY(ssm::stage_input(tu, u, ssm::view(3, nx, st->u), es, w, "u", s));
  TRY(ssm::stage_input(td, delta, ssm::view(3, nx, st->delta), es, w + x, "delta", s));
  TRY(ssm::stage_input(tz, z, ssm::view(3, nx, st->z), es, w + 2 * x, "z", s));
  TRY(ssm::stage_output(to, out, ssm::view(3, nx, st->out), es, w + 3 * x, "out", false, s));
  TRY(ssm::stage_input(tB, B, ssm::view(4, nbc, st->B), es, w + 4 * x, "B", s));
  TRY(ssm::stage_input(tC, C, ssm::view(4, nbc, st->C), es, w + 4 * x + bc, "C", s));
  char* inner = w + 4 * x + 2 * bc;
  TRY(ssm_scan_fwd_ex(tu.dense, td.dense, A, tB.dense, tC.dense, D, tz.dense, dt_bias,
                      delta_softplus, h0, hL, to.dense, ckpt, inner, workspace_bytes - (inner - w),
                      batch, dim, seqlen, dstate, bc_groups, io_dtype, flags, stream));
  return ssm::scatter_output(to, es, s);
}

size_t ssm_scan_bwd_strided_workspace_size(int batch, int dim, int seqlen, int dstate,
                                           int bc_groups, int io_dtype, int have_ckpt,
                                           int flags) {
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH)) return 0;
  if (!ssm::sizes_ok(batch, dim, seqlen, dstate) || bc_groups < 1) return 0;
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return 0;
  const size_t es = ssm::esize(io_dtype);
  const size_t x = ssm::align_up((size_t)batch * dim * seqlen * es);
  const size_t bc = ssm::align_up((size_t)batch * bc_groups * dstate * seqlen * es);
  const size_t inner = ssm::align_up(ssm_scan_bwd_ex_workspace_size(
      batch, dim, seqlen, dstate, bc_groups, io_dtype, have_ckpt, flags));
  if (inner == 0) return 0;
  return 7 * x + 4 * bc + inner;
}

int ssm_scan_bwd_strided(const void* u, const void* delta, const float* A, const void* B,
                         const void* C, const float* D, const void* z, const float* dt_bias,
                         int delta_softplus, const float* h0, const void* dout, const float* dhL,
                         const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC,
                         float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                         size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                         int bc_groups, int io_dtype, int flags, const ssm_strides* st,
                         void* stream) {
  ssm::set_last_error("");
  if (flags & ~(SSM_SCALAR_A | SSM_REVERSE | SSM_ZOH))
    return ssm::fail(SSM_EINVAL, "%s", "unsupported flags for a strided call");
  if (!st) return ssm::fail(SSM_EINVAL, "%s", "strides is NULL");
  if (!ssm::sizes_ok(batch, dim, seqlen, dstate) || bc_groups < 1)
    return ssm::fail(SSM_EINVAL, "%s", "sizes must be positive");
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16)
    return ssm::fail(SSM_EINVAL, "%s", "io_dtype is not SSM_F32/SSM_BF16");
  const size_t need = ssm_scan_bwd_strided_workspace_size(batch, dim, seqlen, dstate, bc_groups,
                                                          io_dtype, ckpt != nullptr, flags);
  if (need == 0) return ssm::fail(SSM_EINVAL, "%s", "invalid sizes or groups");
  if (!workspace || workspace_bytes < need)
    return ssm::fail(SSM_EWORKSPACE, "%s", "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return ssm::fail(SSM_EINVAL, "%s", "workspace is not 256-byte aligned");
  TRY(ssm::check_device_ptr(workspace, need, 256, "workspace"));
  if (!u || !delta || !B || !C || !dout)
    return ssm::fail(SSM_EINVAL, "%s", "u, delta, B, C and dout are required");
  const size_t es = ssm::esize(io_dtype);
  const size_t x = ssm::align_up((size_t)batch * dim * seqlen * es);
  const size_t bc = ssm::align_up((size_t)batch * bc_groups * dstate * seqlen * es);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nx[3] = {batch, dim, seqlen};
  const long long nbc[4] = {batch, bc_groups, dstate, seqlen};
  Slot tu, td, tz, tg, tdu, tdd, tdz, tB, tC, tdB, tdC;
  TRY(ssm::stage_input(tu, u, ssm::view(3, nx, st->u), es, w, "u", s));
  TRY(ssm::stage_input(td, delta, ssm::view(3, nx, st->delta), es, w + x, "delta", s));
  TRY(ssm::stage_input(tz, z, ssm::view(3, nx, st->z), es, w + 2 * x, "z", s));
  TRY(ssm::stage_input(tg, dout, ssm::view(3, nx, st->dout), es, w + 3 * x, "dout", s));
  TRY(ssm::stage_output(tdu, du, ssm::view(3, nx, st->du), es, w + 4 * x, "du", false, s));
  TRY(ssm::stage_output(tdd, ddelta, ssm::view(3, nx, st->ddelta), es, w + 5 * x, "ddelta", false, s));
  TRY(ssm::stage_output(tdz, dz, ssm::view(3, nx, st->dz), es, w + 6 * x, "dz", false, s));
  char* wb = w + 7 * x;
  TRY(ssm::stage_input(tB, B, ssm::view(4, nbc, st->B), es, wb, "B", s));
  TRY(ssm::stage_input(tC, C, ssm::view(4, nbc, st->C), es, wb + bc, "C", s));
  TRY(ssm::stage_output(tdB, dB, ssm::view(4, nbc, st->dB), es, wb + 2 * bc, "dB", false, s));
  TRY(ssm::stage_output(tdC, dC, ssm::view(4, nbc, st->dC), es, wb + 3 * bc, "dC", false, s));
  char* inner = wb + 4 * bc;
  TRY(ssm_scan_bwd_ex(tu.dense, td.dense, A, tB.dense, tC.dense, D, tz.dense, dt_bias,
                      delta_softplus, h0, tg.dense, dhL, ckpt, tdu.dense, tdd.dense, dA,
                      tdB.dense, tdC.dense, dD, tdz.dense, ddt_bias, dh0, inner,
                      workspace_bytes - (inner - w), batch, dim, seqlen, dstate, bc_groups,
                      io_dtype, flags, stream));
  TRY(ssm::scatter_output(tdu, es, s));
  TRY(ssm::scatter_output(tdd, es, s));
  TRY(ssm::scatter_output(tdz, es, s));
  TRY(ssm::scatter_output(tdB, es, s));
  return ssm::scatter_output(tdC, es, s);
}

size_t ssm_state_update_strided_workspace_size(int batch, int dim, int dstate, int bc_groups,
                                               int io_dtype) {
  if (!ssm::sizes_ok(batch, dim, dstate, 1) || bc_groups < 1) return 0;
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return 0;
  const size_t es = ssm::esize(io_dtype);
  return ssm::align_up((size_t)batch * dim * dstate * 4) +
         4 * ssm::align_up((size_t)batch * dim * es) +
         2 * ssm::align_up((size_t)batch * bc_groups * dstate * es);
}

int ssm_state_update_strided(float* state, const void* x, const void* dt, const float* A,
                             const void* B, const void* C, const float* D, const void* z,
                             const float* dt_bias, int delta_softplus, void* out,
                             void* workspace, size_t workspace_bytes, int batch, int dim,
                             int dstate, int bc_groups, int io_dtype, int flags,
                             const ssm_decode_strides* st, void* stream) {
  ssm::set_last_error("");
  if (flags & ~(SSM_SCALAR_A | SSM_ZOH))
    return ssm::fail(SSM_EINVAL, "%s", "unsupported flags for a decode step");
  if (!st) return ssm::fail(SSM_EINVAL, "%s", "strides is NULL");
  const size_t need = ssm_state_update_strided_workspace_size(batch, dim, dstate, bc_groups, io_dtype);
  if (need == 0) return ssm::fail(SSM_EINVAL, "%s", "invalid sizes, groups or io_dtype");
  if (!workspace || workspace_bytes < need)
    return ssm::fail(SSM_EWORKSPACE, "%s", "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return ssm::fail(SSM_EINVAL, "%s", "workspace is not 256-byte aligned");
  TRY(ssm::check_device_ptr(workspace, need, 256, "workspace"));
  if (!state || !x || !dt || !B || !C || !out)
    return ssm::fail(SSM_EINVAL, "%s", "state, x, dt, B, C and out are required");
  const size_t es = ssm::esize(io_dtype);
  const size_t ss = ssm::align_up((size_t)batch * dim * dstate * 4);
  const size_t sx = ssm::align_up((size_t)batch * dim * es);
  const size_t sb = ssm::align_up((size_t)batch * bc_groups * dstate * es);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nst[3] = {batch, dim, dstate};
  const long long nx[2] = {batch, dim};
  const long long nbc[3] = {batch, bc_groups, dstate};
  Slot tst, tx, tdt, tz, to, tB, tC;
  TRY(ssm::stage_output(tst, state, ssm::view(3, nst, st->state), 4, w, "state", true, s));
  TRY(ssm::stage_input(tx, x, ssm::view(2, nx, st->x), es, w + ss, "x", s));
  TRY(ssm::stage_input(tdt, dt, ssm::view(2, nx, st->dt), es, w + ss + sx, "dt", s));
  TRY(ssm::stage_input(tz, z, ssm::view(2, nx, st->z), es, w + ss + 2 * sx, "z", s));
  TRY(ssm::stage_output(to, out, ssm::view(2, nx, st->out), es, w + ss + 3 * sx, "out", false, s));
  TRY(ssm::stage_input(tB, B, ssm::view(3, nbc, st->B), es, w + ss + 4 * sx, "B", s));
  TRY(ssm::stage_input(tC, C, ssm::view(3, nbc, st->C), es, w + ss + 4 * sx + sb, "C", s));
  TRY(ssm_state_update_ex(reinterpret_cast<float*>(tst.dense), tx.dense, tdt.dense, A, tB.dense,
                          tC.dense, D, tz.dense, dt_bias, delta_softplus, to.dense, batch, dim,
                          dstate, bc_groups, io_dtype, flags, stream));
  TRY(ssm::scatter_output(tst, 4, s));
  return ssm::scatter_output(to, es, s);
}

}  // extern "C"

namespace {
// Rows of L 16-bit elements mirrored along L: dst[r][t] = src[r][L - 1 - t].  In place
// (src == dst) each thread swaps one pair; otherwise each thread copies one element.
__global__ void mirror_rows_kernel(const uint16_t* __restrict__ src, uint16_t* dst,
                                   long long rows, int L, int in_place) {
  const long long per = in_place ? L / 2 : L;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * per) return;
  const long long r = i / per;
  const int t = (int)(i % per);
  const long long a = r * L + t, m = r * L + (L - 1 - t);
  if (in_place) {
    const uint16_t x = dst[a];
    dst[a] = dst[m];
    dst[m] = x;
  } else {
    dst[a] = src[m];
  }
}

// Eight 16-bit elements of a 16-byte word in reverse order.
__device__ __forceinline__ uint4 rev8(uint4 v) {
  const auto sw = [](uint32_t w) { return __byte_perm(w, 0, 0x1032); };  // swap the halves
  return make_uint4(sw(v.w), sw(v.z), sw(v.y), sw(v.x));
}

// The same with rows of L = 8 k elements and 16-byte aligned rows: one 16-byte piece per thread
// (copy), or, in place, a piece and its mirror image swapped (the middle piece of an odd count
// reversed by itself).
__global__ void mirror_rows8_kernel(const uint4* __restrict__ src, uint4* dst, long long rows,
                                    int L8, int in_place) {
  const long long per = in_place ? (L8 + 1) / 2 : L8;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * per) return;
  const long long r = i / per;
  const int p = (int)(i % per);
  const long long a = r * L8 + p, m = r * L8 + (L8 - 1 - p);
  if (in_place) {
    const uint4 x = dst[a], y = dst[m];
    dst[a] = rev8(y);
    if (m != a) dst[m] = rev8(x);
  } else {
    dst[a] = rev8(__ldcs(src + m));
  }
}
}  // namespace

namespace ssm {
// The reverse scan of the chunked matrix form runs its kernels on rows mirrored along time: rows
// [rows][L] of 16-bit elements from src into dst mirrored, or in place when src == dst.
cudaError_t mirror_rows(const void* src, void* dst, long long rows, int L, cudaStream_t s) {
  const int in_place = src == dst ? 1 : 0;
  const bool v8 = L % 8 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                  (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
  if (v8) {
    const int L8 = L / 8;
    const long long n = rows * (in_place ? (L8 + 1) / 2 : L8);
    if (n <= 0) return cudaSuccess;
    mirror_rows8_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), rows, L8, in_place);
    return cudaGetLastError();
  }
  const long long n = rows * (in_place ? L / 2 : L);
  if (n <= 0) return cudaSuccess;
  mirror_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      reinterpret_cast<const uint16_t*>(src), reinterpret_cast<uint16_t*>(dst), rows, L, in_place);
  return cudaGetLastError();
}

// The restride copy for other translation units: the 4-index view (sizes n, element strides ss)
// at src into the view with strides ds at dst (es = 2 or 4 bytes per element), on stream s.
cudaError_t copy_view(const void* src, const long long* n, const long long* ss, void* dst,
                      const long long* ds, size_t es, cudaStream_t s) {
  View4 sv, dv;
  for (int k = 0; k < 4; ++k) {
    sv.n[k] = dv.n[k] = n[k];
    sv.s[k] = ss[k];
    dv.s[k] = ds[k];
  }
  return restride(src, sv, dst, dv, es, s);
}
}  // namespace ssm
