// Internal launch interface between the C-ABI layer (ssm_api.cu) and the kernel files.
// Not part of the public boundary; the public declarations are in include/ssm_scan.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr int kBlk = 16;   // time steps per block: one scalar / state / output phase
constexpr int kNS = 16;    // states per channel (dstate <= 16, padded with zeros)

// kFwdOut: gated output (+ optional checkpoints / final state); kFwdSummary: per-chunk end
// state and ΣΔ from a zero state (time-split first pass); kFwdCkpt: state recurrence only,
// writing the state entering every 16-step block (input of the backward pass).
enum FwdMode { kFwdOut = 0, kFwdSummary = 1, kFwdCkpt = 2 };

// Variant codes passed in place of a MUFU pair count (template KE = KO of the forward kernel,
// KP of the backward kernel).
constexpr int kKpScalar = -1;      // one decay rate per channel, first-order input term
constexpr int kKpZoh = -2;         // zero-order-hold input term, range-checked block
constexpr int kKpZohClamped = -3;  // zero-order-hold input term, exponent range clamped
constexpr int kKpScalarZoh = -4;   // one decay rate per channel, zero-order-hold input term

struct FwdArgs {
  const void* u;
  const void* delta;
  const void* z;        // may be NULL (no gate)
  const void* B;
  const void* C;
  const float* A;       // [dim][N], or [dim] when scalar_a
  const float* D;       // may be NULL
  const float* dt_bias; // may be NULL
  const float* h0;      // may be NULL (zero initial state)
  void* out;
  float* hL;            // may be NULL
  float* ckpt;          // may be NULL; [batch][dim][ceil(L/16)][N]
  float* summ;          // summary pass: per-chunk end state from zero [S][channels][16] (N: chunked form)
  float* dsum;          // summary pass: per-chunk sum of Δ          [S][channels]
  const float* hin;     // output pass with S > 1: state entering each chunk [S][channels][16] (N: chunked form)
  int batch, dim, L, N;
  int chunk_len;        // multiple of kBlk
  int nchunk;           // S
  int softplus;
  int scalar_a;         // one decay rate A_d per channel, shared by its N states
  int reverse;          // scan runs from t = L-1 down to 0 (time rows read/written mirrored)
  int zoh;              // zero-order-hold input term (e^{ΔA} - 1)/A B x instead of Δ B x
  int bc_groups;        // B, C are [batch][bc_groups][N][L]; channel d uses group d / (dim / bc_groups)
  int channels_last;    // u, delta, z, out are [batch][L][dim] and B, C [batch][L][bc_groups][N]
  int cl_tile;          // channels-last rows moved as 16-byte tiles (dim % 16 == 0, N == 16, aligned)
  int lpc;              // lanes per channel: 1, 2 or 4 (16 / lpc states each)
  int wide;             // few warps per SM: the 255-register form of the output kernel
  int rows16;           // rows along L in aligned 16-byte pieces (L * es % 16 == 0, aligned tensors)
  int warps_per_b;      // ceil(dim / (32 / lpc))
  long long nwarps;     // batch * warps_per_b
};

struct BwdArgs {
  const void* u;
  const void* delta;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* dt_bias;
  const void* dout;
  const float* dhL;
  const float* ckpt;    // [batch][dim][nblk][N]
  void* du;
  void* ddelta;
  void* dz;
  float* dh0;
  float* part_bc;       // [ngroups][batch][2][16][L] per-CTA partial sums of dB, dC
  float* part_adt;      // [nsplit][batch][dim][16 + 2] per-channel (and chunk) partial dA, dD, ddt_bias
  int batch, dim, L, N;
  int softplus;
  int warps_per_b;
  long long nwarps;
  int wpb;              // warps per CTA (channels per CTA = 16 * wpb)
  int ngroups;          // CTAs per batch row = ceil(warps_per_b / wpb)
  int kmufu;            // state pairs (of 4 per lane) whose exponential runs on MUFU: 2, 3 or 4
  int reverse;          // gradients of the reverse scan (time rows read/written mirrored)
  int zoh;              // gradients of the zero-order-hold input term
  int bc_groups;        // B, C (and dB, dC) are [batch][bc_groups][N][L]
  int channels_last;    // time rows strided: [batch][L][dim] and [batch][L][bc_groups][N]
  // time split of the register-history backward (nsplit <= 1: none): chunk c covers blocks
  // [c blk_per_chunk, (c + 1) blk_per_chunk); lam_in [nsplit][batch][dim][16] holds the adjoint
  // entering each chunk from later time, in reverse chunk order (slot nsplit-1-c)
  int nsplit;
  int blk_per_chunk;
  const float* lam_in;
};

struct DecodeArgs {
  float* state;
  const void* x;
  const void* dt;
  const void* z;
  const void* B;
  const void* C;
  const float* A;
  const float* D;
  const float* dt_bias;
  void* out;
  int batch, dim, N;
  int softplus;
  int scalar_a;   // A is [dim]: one decay rate per channel
  int zoh;        // zero-order-hold input coefficient (e^{ΔA} - 1)/A instead of Δ
  int bc_groups;  // B, C are [batch][bc_groups][N]; channel d uses group d / (dim / bc_groups)
};

// io: 0 = f32, 1 = bf16.  vec: rows are 16-byte aligned and L is a multiple of the vector width.
cudaError_t launch_fwd(const FwdArgs& a, int io, bool vec, int mode, int wpb, int kmufu,
                       cudaStream_t s);
// The one-lane-per-channel forward kernel (default variant only: no scalar_a, zoh, reverse or
// channels_last; rows allow 16-byte copies; a.warps_per_b = ceil(dim / 32); dim / bc_groups a
// multiple of 32).
cudaError_t launch_fwd_lane(const FwdArgs& a, int io, int mode, int kmufu, cudaStream_t s);
// Scalar decay with N = 32, 64 or 128 (bf16 io): the chunked matrix form on the tensor cores
// (ssm_ssd.cu).  B, C shared by each CTA's 64 channels (bc_groups == 1 or dim / bc_groups a
// multiple of 64); a.rows16 selects 16-byte row accesses.  Time segments of a.chunk_len steps
// (a multiple of 16), a.nchunk of them: the summary mode runs segments 0 .. nchunk-2 from zero and
// writes a.summ [seg][batch][dim][N] and a.dsum [seg][batch][dim]; the output launch runs every
// segment from a.hin [seg][batch][dim][N] when given (else segment 0 from a.h0).
// Backward of the chunked matrix form (ssm_ssd_bwd.cu): scalar decay, bf16 io, N = 16..128.
struct SsdBwdArgs {
  const uint16_t* u;
  const uint16_t* delta;
  const uint16_t* z;        // NULL: no gate
  const uint16_t* B;        // [batch][bc_groups][N][L]
  const uint16_t* C;
  const uint16_t* dout;
  const float* A;           // [dim]
  const float* D;
  const float* dt_bias;
  const float* dhL;
  const float* ck;          // [batch][dim][ceil(L/16)][N]: the state entering every chunk
  uint16_t* du;
  uint16_t* ddelta;
  uint16_t* dz;
  float* dh0;
  float* part_bc;           // [CTAs per row][batch][2][N][L]: each CTA's dB, dC
  float* part_adt;          // [nseg][batch][dim][3]: dA, dD, ddt_bias of each (segment, row, channel)
  // time split (nseg segments of cps chunks): the summary launch writes each segment's μ at its
  // start from μ = 0 at its end and its ΣΔ, in reverse segment order ([nseg][batch][dim][N] and
  // [nseg][batch][dim]); mu_in [nseg][batch][dim][N] is their chain (mu_in[0] = dhL)
  float* mu_sum;
  float* dsum;
  const float* mu_in;
  int nseg, cps;
  int batch, dim, L, N, bc_groups, softplus, rows16, need_bc;
  int zoh;  // zero-order-hold input coefficient (e^{ΔA} - 1)/A instead of Δ
};
// 64 channels per CTA (dim / bc_groups a multiple of 64 with groups); a.ck from launch_ssd_fwd's
// checkpoint mode.  The finishing launch sums part_bc over each group's CTAs into dB, dC (bf16)
// and part_adt over the batch into dA, dD, ddt_bias.
cudaError_t launch_ssd_bwd(const SsdBwdArgs& a, bool summary, cudaStream_t s);
cudaError_t launch_ssd_bwd_finish(const SsdBwdArgs& a, void* dB, void* dC, float* dA, float* dD,
                                  float* ddt_bias, cudaStream_t s);
int ssd_bwd_ctas_per_row(int dim);
// mode: kSsdOut (with a.ckpt also the checkpoints), kSsdSummary, or kSsdCkpt (no outputs; only
// the state entering every 16-step chunk into a.ckpt, f32 [batch][dim][ceil(L / 16)][N]).
// kSsdOutCkpt is kSsdOut with checkpoints (chosen by the launcher when a.ckpt is set).
enum SsdMode { kSsdOut = 0, kSsdSummary = 1, kSsdCkpt = 2, kSsdOutCkpt = 3 };
cudaError_t launch_ssd_fwd(const FwdArgs& a, int mode, cudaStream_t s);
cudaError_t launch_fwd_carry(const FwdArgs& a, const float* summ, const float* dsum, float* hin,
                             cudaStream_t s);
cudaError_t launch_bwd(const BwdArgs& a, int io, bool vec, cudaStream_t s);
// The backward of the default variant with the state history in registers (ssm_bwd_hist.cu):
// N = 16, forward direction, no ZOH, [batch][dim][L] rows with L % 8 == 0 and 16-byte aligned
// tensors and checkpoints; a.wpb = 2 or 4 warps per CTA (bwd_hist_pick_wpb), a.ngroups =
// ceil(ceil(dim / 16) / a.wpb), each CTA inside one B/C group.
// With a.nsplit > 1 the CTAs of chunk c (grid.y) start from the adjoint in a.lam_in and write
// chunk c's part of part_adt; only chunk 0 writes dh0.
cudaError_t launch_bwd_hist(const BwdArgs& a, int io, cudaStream_t s);
int bwd_hist_pick_wpb(int io, int batch, int dim);
// The adjoint summaries of chunks 1 .. nsplit-1 for the time-split history backward: for chunk c,
// the adjoint leaving its first step when none enters at its end (summ [slot][batch][dim][16])
// and its ΣΔ (dsum [slot][batch][dim]), stored at slot nsplit-1-c so that the forward carry pass
// (launch_fwd_carry, with dhL in place of h0) chains them from the last chunk to the first.
cudaError_t launch_bwd_summary(const BwdArgs& a, int io, float* summ, float* dsum, cudaStream_t s);
// Number of CTAs of the history backward that one SM holds at once for this shape.
int bwd_hist_ctas_per_sm(int io, int wpb);
// B/C per channel (bc_groups == dim, ssm_pcbc.cu): forward (mode kFwdOut or kFwdCkpt) and
// backward (writes du, ddelta, dz, dB, dC, dh0 and the per-channel dA/dD/ddt_bias partials).
cudaError_t launch_fwd_pcbc(const FwdArgs& a, int io, bool vec, int mode, cudaStream_t s);
cudaError_t launch_bwd_pcbc(const BwdArgs& a, int io, bool vec, void* dB, void* dC, cudaStream_t s);
// dA, dD, ddt_bias from the per-channel partials (the second half of launch_bwd_finish).
cudaError_t launch_bwd_finish_adt(const BwdArgs& a, float* dA, float* dD, float* ddt_bias,
                                  cudaStream_t s);
cudaError_t launch_bwd_finish(const BwdArgs& a, int io, void* dB, void* dC, float* dA, float* dD,
                              float* ddt_bias, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, int io, cudaStream_t s);
// Number of bounded waits that ran out in the streamed decode kernel since the library was loaded
// on the current device (0 when every copy completed); -1 if the count could not be read.
int decode_wait_timeouts(unsigned int* out);

// Sets the message returned by ssm_last_error() on the calling thread.
void set_last_error(const char* msg);
// Copies the 4-index view (sizes n, element strides ss) at src into the view with strides ds at
// dst, es = 2 or 4 bytes per element (ssm_strided.cu).
cudaError_t copy_view(const void* src, const long long* n, const long long* ss, void* dst,
                      const long long* ds, size_t es, cudaStream_t s);
// Rows [rows][L] of 16-bit elements mirrored along L from src into dst, or in place when
// src == dst (ssm_strided.cu).
cudaError_t mirror_rows(const void* src, void* dst, long long rows, int L, cudaStream_t s);
// Backward of the scalar-decay scan for dstate = 16 k (k = 2, 4, 8) as the sum of k 16-state
// backwards (ssm_slices.cu); arguments as ssm_scan_bwd_ex.
// The f32 forward of the scalar-decay scan for dstate = 16 k as the sum of k 16-state forwards
// (ssm_slices.cu); arguments as ssm_scan_fwd_ex.
size_t scan_fwd_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                 int io_dtype, int flags);
int scan_fwd_slices(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                    void* workspace, size_t workspace_bytes, int batch, int dim, int seqlen,
                    int dstate, int bc_groups, int io_dtype, int flags, void* stream);
// The f32 sequence summary of the scalar-decay scan for dstate = 16 k as k 16-state summaries
// (ssm_slices.cu); arguments as ssm_scan_fwd_summary.
size_t scan_summary_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                     int flags);
int scan_summary_slices(const void* u, const void* delta, const float* A, const void* B,
                        const void* C, const float* dt_bias, int delta_softplus, float* hend,
                        float* dsum, void* workspace, size_t workspace_bytes, int batch, int dim,
                        int seqlen, int dstate, int bc_groups, int flags, void* stream);
size_t scan_bwd_slices_workspace(int batch, int dim, int seqlen, int dstate, int bc_groups,
                                 int io_dtype, int flags);
int scan_bwd_slices(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* dt_bias,
                    int delta_softplus, const float* h0, const void* dout, const float* dhL,
                    const float* ckpt, void* du, void* ddelta, float* dA, void* dB, void* dC,
                    float* dD, void* dz, float* ddt_bias, float* dh0, void* workspace,
                    size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                    int bc_groups, int io_dtype, int flags, void* stream);
// The entry points' pointer check (device-accessible on the current device, allocation holds
// `bytes` bytes, `align`-byte aligned); returns an ssm_status and sets the error message.
int check_device_ptr(const void* p, size_t bytes, size_t align, const char* name);

}  // namespace ssm
