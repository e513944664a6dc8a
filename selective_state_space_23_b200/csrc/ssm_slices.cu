// Backward of the scalar-decay scan for large state sizes (dstate = 16 k, k = 2, 4, 8), as a sum
// over 16-state slices.
//
// With one decay rate per channel (the Mamba-2 restriction noted on the "2024 Reading List:
// Neural Network" page), the states do not interact: state n follows
// h_t[n] = e^{Δ_t A} h_{t-1}[n] + Δ_t x_t B_t[n] on its own, and the output is
// y_t = Σ_n C_t[n] h_t[n] + D x_t.  Cut the states into slices of 16: y is the sum of the slices'
// outputs plus D x, and every gradient is linear in the slice outputs:
//   * du, ddelta, dz, dA, ddt_bias are sums over the slices of each slice's gradients (dz of a
//     slice is dout silu'(z) times that slice's output, so the sum is dout silu'(z) y);
//   * dB, dC, dh0 (and the slices of h0, dhL) are disjoint per slice;
//   * D enters one slice only (its du term g D and its dD).
// So the backward runs the library's 16-state backward once per slice (B, C, h0, dhL gathered
// into dense slices by the view copy kernel), accumulates du, ddelta, dz, dA, ddt_bias in f32,
// and scatters dB, dC, dh0 back.  It costs k times the 16-state backward: the compatibility path
// for training with N > 16 (bf16 runs the chunked matrix form, ssm_ssd.cu, ssm_ssd_bwd.cu).
//
// The forward in f32 io (which the chunked form, a bf16 tensor-core form, does not take) is the
// same sum: the gate multiplies the whole readout, so out = Σ_slices (y_slice + [first] D x)
// silu(z) is each slice's gated output summed in f32; hL and the checkpoints are disjoint per
// slice.  The first slice writes the output and each further one adds its own (f32).
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include "../../include/ssm_scan.h"
#include "ssm_device.cuh"
#include "ssm_kernels.h"

namespace ssm {
namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// acc[i] (+)= src[i] (first: =), src io-typed.
template <typename IO>
__global__ void accumulate_kernel(const IO* __restrict__ src, float* __restrict__ acc, long long n,
                                  int first) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    float v;
    if constexpr (sizeof(IO) == 2) v = bf16_to_f32(src[i]);
    else v = src[i];
    acc[i] = first ? v : acc[i] + v;
  }
}

// dst[i] = acc[i], rounded to the io type.
template <typename IO>
__global__ void store_kernel(const float* __restrict__ acc, IO* __restrict__ dst, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    if constexpr (sizeof(IO) == 2) dst[i] = f32_to_bf16(acc[i]);
    else dst[i] = acc[i];
  }
}

unsigned grid_for(long long n) {
  const long long g = (n + 255) / 256;
  return (unsigned)(g < 4096 ? (g > 0 ? g : 1) : 4096);
}

cudaError_t accumulate(const void* src, float* acc, long long n, bool first, size_t es,
                       cudaStream_t s) {
  if (es == 2)
    accumulate_kernel<uint16_t><<<grid_for(n), 256, 0, s>>>(reinterpret_cast<const uint16_t*>(src),
                                                           acc, n, first ? 1 : 0);
  else
    accumulate_kernel<float><<<grid_for(n), 256, 0, s>>>(reinterpret_cast<const float*>(src), acc,
                                                        n, first ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t store(const float* acc, void* dst, long long n, size_t es, cudaStream_t s) {
  if (es == 2)
    store_kernel<uint16_t><<<grid_for(n), 256, 0, s>>>(acc, reinterpret_cast<uint16_t*>(dst), n);
  else
    store_kernel<float><<<grid_for(n), 256, 0, s>>>(acc, reinterpret_cast<float*>(dst), n);
  return cudaGetLastError();
}

// Workspace layout of the slice backward (byte offsets).
struct SliceLayout {
  size_t bj, cj, dbj, dcj, duj, ddj, dzj, adu, add, adz, h0j, dhlj, dh0j, daj, dtj, ada, adt, inner;
  size_t inner_bytes, total;
};

SliceLayout slice_layout(int batch, int dim, int seqlen, int bc_groups, int io_dtype, int flags) {
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  const size_t bcs = align256((size_t)batch * bc_groups * kNS * seqlen * es);
  const size_t xs = align256((size_t)batch * dim * seqlen * es);
  const size_t xf = align256((size_t)batch * dim * seqlen * 4);
  const size_t st = align256((size_t)batch * dim * kNS * 4);
  const size_t vd = align256((size_t)dim * 4);
  SliceLayout l;
  size_t o = 0;
  l.bj = o; o += bcs;
  l.cj = o; o += bcs;
  l.dbj = o; o += bcs;
  l.dcj = o; o += bcs;
  l.duj = o; o += xs;
  l.ddj = o; o += xs;
  l.dzj = o; o += xs;
  l.adu = o; o += xf;
  l.add = o; o += xf;
  l.adz = o; o += xf;
  l.h0j = o; o += st;
  l.dhlj = o; o += st;
  l.dh0j = o; o += st;
  l.daj = o; o += vd;
  l.dtj = o; o += vd;
  l.ada = o; o += vd;
  l.adt = o; o += vd;
  l.inner = o;
  l.inner_bytes = align256(ssm_scan_bwd_ex_workspace_size(batch, dim, seqlen, kNS, bc_groups,
                                                          io_dtype, 0, flags));
  l.total = o + l.inner_bytes;
  return l;
}

int fail(int code, const char* msg) {
  set_last_error(msg);
  return code;
}

// Workspace layout of the slice forward (byte offsets).
struct FwdSliceLayout {
  size_t bj, cj, h0j, hlj, ckj, oj, inner, inner_bytes, total;
};

FwdSliceLayout fwd_slice_layout(int batch, int dim, int seqlen, int bc_groups, int io_dtype,
                                int flags) {
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  const size_t nblk = (seqlen + kBlk - 1) / kBlk;
  FwdSliceLayout l;
  size_t o = 0;
  l.bj = o; o += align256((size_t)batch * bc_groups * kNS * seqlen * es);
  l.cj = o; o += align256((size_t)batch * bc_groups * kNS * seqlen * es);
  l.h0j = o; o += align256((size_t)batch * dim * kNS * 4);
  l.hlj = o; o += align256((size_t)batch * dim * kNS * 4);
  l.ckj = o; o += align256((size_t)batch * dim * nblk * kNS * 4);
  l.oj = o; o += align256((size_t)batch * dim * seqlen * es);
  l.inner = o;
  l.inner_bytes = align256(ssm_scan_fwd_ex_workspace_size(batch, dim, seqlen, kNS, bc_groups,
                                                          io_dtype, flags));
  l.total = o + l.inner_bytes;
  return l;
}

}  // namespace

size_t scan_fwd_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                 int io_dtype, int flags) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR || !(flags & SSM_SCALAR_A) ||
      (flags & SSM_CHANNELS_LAST) || batch <= 0 || dim <= 0 || seqlen <= 0 || bc_groups < 1 ||
      io_dtype != SSM_F32)
    return 0;
  return fwd_slice_layout(batch, dim, seqlen, bc_groups, io_dtype, flags).total;
}

int scan_fwd_slices(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                    void* workspace, size_t workspace_bytes, int batch, int dim, int seqlen,
                    int dstate, int bc_groups, int io_dtype, int flags, void* stream) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR)
    return fail(SSM_EUNSUPPORTED, "scalar-decay f32 forward with dstate > 16 needs a multiple of 16 "
                                  "up to 128");
  if (flags & SSM_CHANNELS_LAST)
    return fail(SSM_EUNSUPPORTED, "scalar-decay forward with dstate > 16 takes the default layout");
  if (bc_groups == dim && bc_groups > 1)
    return fail(SSM_EUNSUPPORTED, "scalar-decay forward with dstate > 16 takes shared or grouped B/C");
  const size_t need = scan_fwd_slices_workspace(batch, dim, seqlen, dstate, bc_groups, io_dtype, flags);
  if (need == 0) return fail(SSM_EINVAL, "invalid sizes, groups or io_dtype");
  if (!workspace || workspace_bytes < need) {
    char msg[128];
    snprintf(msg, sizeof(msg), "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    return fail(SSM_EWORKSPACE, msg);
  }
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  int rc = check_device_ptr(workspace, need, 256, "workspace");
  if (rc != SSM_OK) return rc;
  const size_t es = 4;
  const size_t N = (size_t)dstate;
  const long long nbc = (long long)bc_groups * dstate * seqlen;
  const long long nblk = (seqlen + kBlk - 1) / kBlk;
  if ((rc = check_device_ptr(B, (size_t)batch * nbc * es, es, "B")) != SSM_OK) return rc;
  if ((rc = check_device_ptr(C, (size_t)batch * nbc * es, es, "C")) != SSM_OK) return rc;
  if ((rc = check_device_ptr(out, (size_t)batch * dim * seqlen * es, es, "out")) != SSM_OK) return rc;
  const size_t nst = (size_t)batch * dim * N * 4;
  if (h0 && (rc = check_device_ptr(h0, nst, 4, "h0")) != SSM_OK) return rc;
  if (hL && (rc = check_device_ptr(hL, nst, 4, "hL")) != SSM_OK) return rc;
  if (ckpt && (rc = check_device_ptr(ckpt, (size_t)batch * dim * nblk * N * 4, 4, "ckpt")) != SSM_OK)
    return rc;

  const FwdSliceLayout l = fwd_slice_layout(batch, dim, seqlen, bc_groups, io_dtype, flags);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nx = (long long)batch * dim * seqlen;
  const int k = dstate / kNS;
  const long long n_bc[4] = {batch, bc_groups, kNS, seqlen};
  const long long s_bc[4] = {(long long)bc_groups * dstate * seqlen, (long long)dstate * seqlen, seqlen, 1};
  const long long d_bc[4] = {(long long)bc_groups * kNS * seqlen, (long long)kNS * seqlen, seqlen, 1};
  const long long n_st[4] = {1, batch, dim, kNS};
  const long long s_st[4] = {0, (long long)dim * dstate, dstate, 1};
  const long long d_st[4] = {0, (long long)dim * kNS, kNS, 1};
  // a slice of the checkpoints [batch][dim][blocks][N]
  const long long n_ck[4] = {batch, dim, nblk, kNS};
  const long long s_ck[4] = {(long long)dim * nblk * dstate, (long long)nblk * dstate, dstate, 1};
  const long long d_ck[4] = {(long long)dim * nblk * kNS, (long long)nblk * kNS, kNS, 1};
  cudaError_t e = cudaSuccess;
#define CK(x)                                         \
  do {                                                \
    if ((e = (x)) != cudaSuccess) {                   \
      set_last_error(cudaGetErrorString(e));          \
      return SSM_ECUDA;                               \
    }                                                 \
  } while (0)
  for (int j = 0; j < k; ++j) {
    const size_t off = (size_t)j * kNS;
    void* Bj = w + l.bj;
    void* Cj = w + l.cj;
    CK(copy_view(reinterpret_cast<const char*>(B) + off * seqlen * es, n_bc, s_bc, Bj, d_bc, es, s));
    CK(copy_view(reinterpret_cast<const char*>(C) + off * seqlen * es, n_bc, s_bc, Cj, d_bc, es, s));
    float* h0j = h0 ? reinterpret_cast<float*>(w + l.h0j) : nullptr;
    if (h0j) CK(copy_view(h0 + off, n_st, s_st, h0j, d_st, 4, s));
    float* hLj = hL ? reinterpret_cast<float*>(w + l.hlj) : nullptr;
    float* ckj = ckpt ? reinterpret_cast<float*>(w + l.ckj) : nullptr;
    // the first slice (with D) writes out; the others add theirs to it
    void* oj = j == 0 ? out : w + l.oj;
    rc = ssm_scan_fwd_ex(u, delta, A, Bj, Cj, j == 0 ? D : nullptr, z, dt_bias, delta_softplus,
                         h0j, hLj, oj, ckj, w + l.inner, l.inner_bytes, batch, dim, seqlen, kNS,
                         bc_groups, io_dtype, flags, stream);
    if (rc != SSM_OK) return rc;
    if (j > 0) CK(accumulate(oj, reinterpret_cast<float*>(out), nx, false, es, s));
    if (hLj) CK(copy_view(hLj, n_st, d_st, hL + off, s_st, 4, s));
    if (ckj) CK(copy_view(ckj, n_ck, d_ck, ckpt + off, s_ck, 4, s));
  }
#undef CK
  return SSM_OK;
}

// Sequence summary (end state from zero, ΣΔ) of the f32 scalar-decay scan with dstate = 16 k: the
// 16-state summary of each slice of B gives that slice of the end state; ΣΔ does not depend on
// the states and is taken from the first slice.  The summary reads no C: each slice's call is
// given its B slice in C's place.
namespace {
struct SummarySliceLayout {
  size_t bj, hj, inner, inner_bytes, total;
};

SummarySliceLayout summary_slice_layout(int batch, int dim, int seqlen, int bc_groups, int flags) {
  SummarySliceLayout l;
  size_t o = 0;
  l.bj = o; o += align256((size_t)batch * bc_groups * kNS * seqlen * 4);
  l.hj = o; o += align256((size_t)batch * dim * kNS * 4);
  l.inner = o;
  l.inner_bytes = align256(ssm_scan_fwd_summary_workspace_size(batch, dim, seqlen, kNS, bc_groups,
                                                               SSM_F32, flags));
  l.total = l.inner_bytes == 0 ? 0 : o + l.inner_bytes;
  return l;
}
}  // namespace

size_t scan_summary_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                     int flags) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR || !(flags & SSM_SCALAR_A) ||
      batch <= 0 || dim <= 0 || seqlen <= 0 || bc_groups < 1)
    return 0;
  return summary_slice_layout(batch, dim, seqlen, bc_groups, flags).total;
}

int scan_summary_slices(const void* u, const void* delta, const float* A, const void* B,
                        const void* C, const float* dt_bias, int delta_softplus, float* hend,
                        float* dsum, void* workspace, size_t workspace_bytes, int batch, int dim,
                        int seqlen, int dstate, int bc_groups, int flags, void* stream) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR)
    return fail(SSM_EUNSUPPORTED, "an f32 sequence summary with dstate > 16 needs a multiple of 16 "
                                  "up to 128");
  if (bc_groups == dim && bc_groups > 1)
    return fail(SSM_EUNSUPPORTED, "sequence summaries take shared or grouped B/C");
  const size_t need = scan_summary_slices_workspace(batch, dim, seqlen, dstate, bc_groups, flags);
  if (need == 0) return fail(SSM_EINVAL, "invalid sizes or groups");
  if (!workspace || workspace_bytes < need) {
    char msg[128];
    snprintf(msg, sizeof(msg), "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    return fail(SSM_EWORKSPACE, msg);
  }
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  int rc = check_device_ptr(workspace, need, 256, "workspace");
  if (rc != SSM_OK) return rc;
  const long long nbc = (long long)bc_groups * dstate * seqlen;
  if ((rc = check_device_ptr(B, (size_t)batch * nbc * 4, 4, "B")) != SSM_OK) return rc;
  if ((rc = check_device_ptr(C, (size_t)batch * nbc * 4, 4, "C")) != SSM_OK) return rc;
  if ((rc = check_device_ptr(hend, (size_t)batch * dim * dstate * 4, 4, "hend")) != SSM_OK) return rc;
  const SummarySliceLayout l = summary_slice_layout(batch, dim, seqlen, bc_groups, flags);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long n_bc[4] = {batch, bc_groups, kNS, seqlen};
  const long long s_bc[4] = {(long long)bc_groups * dstate * seqlen, (long long)dstate * seqlen, seqlen, 1};
  const long long d_bc[4] = {(long long)bc_groups * kNS * seqlen, (long long)kNS * seqlen, seqlen, 1};
  const long long n_st[4] = {1, batch, dim, kNS};
  const long long s_st[4] = {0, (long long)dim * dstate, dstate, 1};
  const long long d_st[4] = {0, (long long)dim * kNS, kNS, 1};
  cudaError_t e = cudaSuccess;
  for (int j = 0; j < dstate / kNS; ++j) {
    const size_t off = (size_t)j * kNS;
    void* Bj = w + l.bj;
    float* hj = reinterpret_cast<float*>(w + l.hj);
    if ((e = copy_view(reinterpret_cast<const float*>(B) + off * seqlen, n_bc, s_bc, Bj, d_bc, 4,
                       s)) != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return SSM_ECUDA;
    }
    rc = ssm_scan_fwd_summary(u, delta, A, Bj, Bj, dt_bias, delta_softplus, hj,
                              j == 0 ? dsum : nullptr, w + l.inner, l.inner_bytes, batch, dim,
                              seqlen, kNS, bc_groups, SSM_F32, flags, stream);
    if (rc != SSM_OK) return rc;
    if ((e = copy_view(hj, n_st, d_st, hend + off, s_st, 4, s)) != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return SSM_ECUDA;
    }
  }
  return SSM_OK;
}

size_t scan_bwd_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                 int io_dtype, int flags) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR || !(flags & SSM_SCALAR_A) ||
      (flags & SSM_CHANNELS_LAST) || batch <= 0 || dim <= 0 || seqlen <= 0 || bc_groups < 1 ||
      (io_dtype != SSM_F32 && io_dtype != SSM_BF16))
    return 0;
  const SliceLayout l = slice_layout(batch, dim, seqlen, bc_groups, io_dtype, flags);
  return l.inner_bytes == 0 ? 0 : l.total;
}

int scan_bwd_slices(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, const void* dout, const float* dhL,
                    const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC,
                    float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                    size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                    int bc_groups, int io_dtype, int flags, void* stream) {
  if (dstate % kNS != 0 || dstate > SSM_MAX_DSTATE_SCALAR)
    return fail(SSM_EUNSUPPORTED, "scalar-decay backward with dstate > 16 needs dstate 32, 64 or 128");
  if (flags & SSM_CHANNELS_LAST)
    return fail(SSM_EUNSUPPORTED, "scalar-decay backward with dstate > 16 takes the default layout");
  if (ckpt)
    return fail(SSM_EUNSUPPORTED, "scalar-decay backward with dstate > 16 recomputes its states: "
                                  "ckpt must be NULL");
  if (bc_groups == dim && bc_groups > 1)
    return fail(SSM_EUNSUPPORTED, "scalar-decay backward with dstate > 16 takes shared or grouped B/C");
  const size_t need = scan_bwd_slices_workspace(batch, dim, seqlen, dstate, bc_groups, io_dtype, flags);
  if (need == 0) return fail(SSM_EINVAL, "invalid sizes, groups or io_dtype");
  if (!workspace || workspace_bytes < need) {
    char msg[128];
    snprintf(msg, sizeof(msg), "workspace of %zu bytes given, %zu needed", workspace_bytes, need);
    return fail(SSM_EWORKSPACE, msg);
  }
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(SSM_EINVAL, "workspace is not 256-byte aligned");
  int rc = check_device_ptr(workspace, need, 256, "workspace");
  if (rc != SSM_OK) return rc;
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  const size_t N = (size_t)dstate;
  const long long nbc = (long long)bc_groups * dstate * seqlen;  // elements per batch row
  // the full tensors must hold what the slices read and write
  if ((rc = check_device_ptr(B, (size_t)batch * nbc * es, es, "B")) != SSM_OK) return rc;
  if ((rc = check_device_ptr(C, (size_t)batch * nbc * es, es, "C")) != SSM_OK) return rc;
  if (dB && (rc = check_device_ptr(dB, (size_t)batch * nbc * es, es, "dB")) != SSM_OK) return rc;
  if (dC && (rc = check_device_ptr(dC, (size_t)batch * nbc * es, es, "dC")) != SSM_OK) return rc;
  const size_t nst = (size_t)batch * dim * N * 4;
  if (h0 && (rc = check_device_ptr(h0, nst, 4, "h0")) != SSM_OK) return rc;
  if (dhL && (rc = check_device_ptr(dhL, nst, 4, "dhL")) != SSM_OK) return rc;
  if (dh0 && (rc = check_device_ptr(dh0, nst, 4, "dh0")) != SSM_OK) return rc;
  if (dA && (rc = check_device_ptr(dA, (size_t)dim * 4, 4, "dA")) != SSM_OK) return rc;
  if (ddt_bias && (rc = check_device_ptr(ddt_bias, (size_t)dim * 4, 4, "ddt_bias")) != SSM_OK) return rc;

  const SliceLayout l = slice_layout(batch, dim, seqlen, bc_groups, io_dtype, flags);
  char* w = reinterpret_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nx = (long long)batch * dim * seqlen;
  const int k = dstate / kNS;
  // views: a 16-state slice of [batch][G][N][L] and of [batch][dim][N]
  const long long n_bc[4] = {batch, bc_groups, kNS, seqlen};
  const long long s_bc[4] = {(long long)bc_groups * dstate * seqlen, (long long)dstate * seqlen, seqlen, 1};
  const long long d_bc[4] = {(long long)bc_groups * kNS * seqlen, (long long)kNS * seqlen, seqlen, 1};
  const long long n_st[4] = {1, batch, dim, kNS};
  const long long s_st[4] = {0, (long long)dim * dstate, dstate, 1};
  const long long d_st[4] = {0, (long long)dim * kNS, kNS, 1};
  const bool any_slice_grad = du || ddelta || dz || dB || dC || dA || ddt_bias || dh0;
  cudaError_t e = cudaSuccess;
#define CK(x)                                         \
  do {                                                \
    if ((e = (x)) != cudaSuccess) {                   \
      set_last_error(cudaGetErrorString(e));          \
      return SSM_ECUDA;                               \
    }                                                 \
  } while (0)
  for (int j = 0; j < k; ++j) {
    if (j > 0 && !any_slice_grad) break;  // only dD was asked for: slice 0 gives it
    const size_t off = (size_t)j * kNS;
    void* Bj = w + l.bj;
    void* Cj = w + l.cj;
    CK(copy_view(reinterpret_cast<const char*>(B) + off * seqlen * es, n_bc, s_bc, Bj, d_bc, es, s));
    CK(copy_view(reinterpret_cast<const char*>(C) + off * seqlen * es, n_bc, s_bc, Cj, d_bc, es, s));
    float* h0j = h0 ? reinterpret_cast<float*>(w + l.h0j) : nullptr;
    float* dhLj = dhL ? reinterpret_cast<float*>(w + l.dhlj) : nullptr;
    if (h0j) CK(copy_view(h0 + off, n_st, s_st, h0j, d_st, 4, s));
    if (dhLj) CK(copy_view(dhL + off, n_st, s_st, dhLj, d_st, 4, s));
    void* duj = du ? w + l.duj : nullptr;
    void* ddj = ddelta ? w + l.ddj : nullptr;
    void* dzj = dz ? w + l.dzj : nullptr;
    void* dBj = dB ? w + l.dbj : nullptr;
    void* dCj = dC ? w + l.dcj : nullptr;
    float* dAj = dA ? reinterpret_cast<float*>(w + l.daj) : nullptr;
    float* dtj = ddt_bias ? reinterpret_cast<float*>(w + l.dtj) : nullptr;
    float* dh0j = dh0 ? reinterpret_cast<float*>(w + l.dh0j) : nullptr;
    rc = ssm_scan_bwd_ex(u, delta, A, Bj, Cj, j == 0 ? D : nullptr, z, dt_bias, delta_softplus,
                         h0j, dout, dhLj, nullptr, duj, ddj, dAj, dBj, dCj, j == 0 ? dD : nullptr,
                         dzj, dtj, dh0j, w + l.inner, l.inner_bytes, batch, dim, seqlen, kNS,
                         bc_groups, io_dtype, flags, stream);
    if (rc != SSM_OK) return rc;
    if (duj) CK(accumulate(duj, reinterpret_cast<float*>(w + l.adu), nx, j == 0, es, s));
    if (ddj) CK(accumulate(ddj, reinterpret_cast<float*>(w + l.add), nx, j == 0, es, s));
    if (dzj) CK(accumulate(dzj, reinterpret_cast<float*>(w + l.adz), nx, j == 0, es, s));
    if (dAj) CK(accumulate(dAj, reinterpret_cast<float*>(w + l.ada), dim, j == 0, 4, s));
    if (dtj) CK(accumulate(dtj, reinterpret_cast<float*>(w + l.adt), dim, j == 0, 4, s));
    if (dBj) CK(copy_view(dBj, n_bc, d_bc, reinterpret_cast<char*>(dB) + off * seqlen * es, s_bc, es, s));
    if (dCj) CK(copy_view(dCj, n_bc, d_bc, reinterpret_cast<char*>(dC) + off * seqlen * es, s_bc, es, s));
    if (dh0j) CK(copy_view(dh0j, n_st, d_st, dh0 + off, s_st, 4, s));
  }
  if (du) CK(store(reinterpret_cast<const float*>(w + l.adu), du, nx, es, s));
  if (ddelta) CK(store(reinterpret_cast<const float*>(w + l.add), ddelta, nx, es, s));
  if (dz) CK(store(reinterpret_cast<const float*>(w + l.adz), dz, nx, es, s));
  if (dA) CK(store(reinterpret_cast<const float*>(w + l.ada), dA, dim, 4, s));
  if (ddt_bias) CK(store(reinterpret_cast<const float*>(w + l.adt), ddt_bias, dim, 4, s));
#undef CK
  return SSM_OK;
}

}  // namespace ssm
