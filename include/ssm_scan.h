/*
 * ssm_scan.h -- C ABI of the B200 selective state-space (S6) scan library (libssm_b200.so).
 *
 * The operation (all three entry points compute parts of it):
 *   "Mamba: Linear-Time Sequence Modeling with Selective State Spaces" (Gu & Dao, arXiv
 *   2312.00752; Turkish summary page):
 *     section "Yöntem"                 -- diagonal SSM discretised with step Δ: Ā = exp(ΔA),
 *                                         recurrence h_t = Ā h_{t-1} + B̄ x_t, readout y_t = C h_t;
 *     section "Seçim Mekanizması (S6)" -- B_t, C_t are per-token N-vectors shared by all D
 *                                         channels; Δ_t = softplus(Parameter + s_Δ(x_t));
 *     section "Donanım Duyarlı Durum Genişletme" -- the expanded (batch, L, D, N) state is kept
 *                                         on chip and never written to HBM; the backward pass
 *                                         recomputes the states;
 *     section "Sorular"                -- generation keeps only a fixed D x N state per layer.
 *   Per channel (b, d), time t and state n < N this library computes
 *     Δ_t      = softplus(delta[b,d,t] + dt_bias[d])   (delta_softplus != 0)
 *              = delta[b,d,t] + dt_bias[d]              (delta_softplus == 0)
 *     h[n]     = exp(Δ_t A[d,n]) h[n] + Δ_t B[b,n,t] u[b,d,t]
 *     y        = Σ_n C[b,n,t] h[n] + D[d] u[b,d,t]
 *     out      = y * silu(z[b,d,t])        (out = y when z is NULL)
 *   The input term Δ_t B_t x_t is the first-order form of the zero-order-hold B̄; the state is
 *   updated before it is read out (y_t uses h_t).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers (or host memory registered/mapped for device access) on the
 *     CURRENT CUDA device, owned by the caller.  The library allocates no memory; scratch space
 *     comes from the caller through `workspace`.  Outputs must not alias inputs, except
 *     `state` in ssm_state_update, which is updated in place by design.
 *   - io_dtype (ssm_dtype) is the element type of every "io" tensor (u, delta, z, B, C, out,
 *     dout, du, ddelta, dz, dB, dC, x, dt): SSM_F32 or SSM_BF16.  A, D, dt_bias, h0, hL, ckpt,
 *     dhL, dh0, dA, dD, ddt_bias and state are always float32.
 *   - All tensors are dense and row-major (last index contiguous), with the layouts given per
 *     argument.  1 <= dstate <= 16 (SSM_EUNSUPPORTED above), except the scalar-decay forward
 *     scan, which also takes dstate 32, 64 and 128.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and the call
 *     returns without synchronising.  A launch failure is reported by the return value; an
 *     error raised later by the device is reported by CUDA on the stream as usual.
 *   - Errors are returned, never raised by abort/exit.  Arguments are validated on the host
 *     before anything is enqueued: NULL required pointers, non-positive sizes, bad dtype codes,
 *     misaligned pointers, pointers the current device cannot access, and device allocations
 *     smaller than the tensor they must hold all return SSM_EINVAL with nothing launched;
 *     ssm_last_error() gives a one-line description (per thread).
 *   - Not thread-safe with respect to concurrent use of the SAME workspace.
 */
#ifndef SSM_SCAN_H_
#define SSM_SCAN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define SSM_API __attribute__((visibility("default")))
#else
#define SSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Number of time steps between two stored states in the checkpoint tensor `ckpt`. */
#define SSM_CKPT_STEPS 16
/* Largest supported dstate (N). */
#define SSM_MAX_DSTATE 16
/* Largest dstate of the scalar-decay forward scan (SSM_SCALAR_A; N = 32, 64 or 128 above 16). */
#define SSM_MAX_DSTATE_SCALAR 128

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

typedef enum {
  SSM_OK = 0,
  SSM_EINVAL = 1,        /* invalid argument; nothing was launched */
  SSM_EUNSUPPORTED = 2,  /* valid request this build does not implement (e.g. dstate 48) */
  SSM_ECUDA = 3,         /* a CUDA runtime call or kernel launch failed */
  SSM_EWORKSPACE = 4     /* workspace NULL or smaller than the size function returned */
} ssm_status;

/* Static description of a status code. */
SSM_API const char* ssm_status_string(int status);
/* Description of the last failure on the calling thread ("" if none). */
SSM_API const char* ssm_last_error(void);
/* Library version string. */
SSM_API const char* ssm_version(void);

/*
 * Bytes of workspace ssm_scan_fwd may use for this shape on the current device (0 when the
 * launch plan needs none).  With less (or NULL) workspace ssm_scan_fwd still computes the same
 * result, without splitting the time axis (slower when batch*dim is small).
 */
SSM_API size_t ssm_scan_fwd_workspace_size(int batch, int dim, int seqlen, int dstate, int io_dtype);

/*
 * Forward selective scan ("Yöntem", "Seçim Mekanizması (S6)", "Donanım Duyarlı Durum Genişletme").
 *   u, delta, z [batch][dim][seqlen] io    inputs x_t, raw step s_Δ(x_t), gate input (z may be NULL)
 *   A         [dim][dstate] f32           diagonal state matrix (any real values)
 *   B, C      [batch][dstate][seqlen] io  input-dependent B_t, C_t, shared across dim
 *   D         [dim] f32 or NULL           skip term D x_t (added before the gate)
 *   dt_bias   [dim] f32 or NULL           the per-channel "Parameter" added to delta
 *   h0        [batch][dim][dstate] f32 or NULL   initial state (NULL = zero)
 *   hL        [batch][dim][dstate] f32 or NULL   OUT: final state h_{L-1}
 *   out       [batch][dim][seqlen] io     OUT: gated output
 *   ckpt      [batch][dim][ceil(seqlen/SSM_CKPT_STEPS)][dstate] f32 or NULL
 *             OUT: state entering every SSM_CKPT_STEPS-step block (block k holds h_{16k-1},
 *             block 0 holds h0); pass it to ssm_scan_bwd to skip its state replay pass.
 *   workspace, workspace_bytes            scratch (may be NULL/0), see the size function.
 * Returns SSM_OK or an error code (nothing launched on error).
 */
SSM_API int ssm_scan_fwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                 const float* D, const void* z, const float* dt_bias, int delta_softplus,
                 const float* h0, float* hL, void* out, float* ckpt, void* workspace,
                 size_t workspace_bytes, int batch, int dim, int seqlen, int dstate,
                 int io_dtype, void* stream);

/*
 * Bytes of workspace ssm_scan_bwd needs.  have_ckpt != 0: the caller will pass the `ckpt`
 * written by ssm_scan_fwd with the same inputs (smaller workspace, one pass fewer).
 */
SSM_API size_t ssm_scan_bwd_workspace_size(int batch, int dim, int seqlen, int dstate, int io_dtype,
                                   int have_ckpt);

/*
 * Backward pass of ssm_scan_fwd with state recomputation ("Donanım Duyarlı Durum Genişletme":
 * intermediate states are recomputed, not stored).  Gradients by the chain rule through the
 * forward recurrence:
 *   λ_t  = g_t C_t + exp(Δ_{t+1} A) λ_{t+1},  g_t = dout_t silu(z_t),  λ_{L-1} += dhL
 *   du_t = g_t D + Δ_t Σ_n λ_t B_t;   ddelta_t = (Σ_n λ_t (A Ā_t h_{t-1} + B_t u_t)) softplus'
 *   dB_t = Σ_d λ_t Δ_t u_t;   dC_t = Σ_d g_t h_t;   dA = Σ_{b,t} λ_t Δ_t Ā_t h_{t-1}
 *   dD = Σ_{b,t} g_t u_t;   ddt_bias = Σ_{b,t} ddelta_t;   dz_t = dout_t y_t silu'(z_t);
 *   dh0 = Ā_0 λ_0.
 * Inputs: as ssm_scan_fwd, plus
 *   dout      [batch][dim][seqlen] io     upstream gradient of `out`
 *   dhL       [batch][dim][dstate] f32 or NULL   upstream gradient of hL
 *   ckpt      as written by ssm_scan_fwd, or NULL (then recomputed into the workspace)
 * Outputs (each may be NULL to skip it, except that at least one must be given):
 *   du, ddelta, dz [batch][dim][seqlen] io (dz only when z != NULL)
 *   dB, dC    [batch][dstate][seqlen] io
 *   dA [dim][dstate] f32;  dD, ddt_bias [dim] f32;  dh0 [batch][dim][dstate] f32
 * All outputs are OVERWRITTEN (not accumulated).  Summed gradients are reduced in a fixed
 * order, so results are bitwise reproducible run to run.
 * workspace: at least ssm_scan_bwd_workspace_size(..., ckpt != NULL) bytes, 256-byte aligned.
 */
SSM_API int ssm_scan_bwd(const void* u, const void* delta, const float* A, const void* B, const void* C,
                 const float* D, const void* z, const float* dt_bias, int delta_softplus,
                 const float* h0, const void* dout, const float* dhL, const float* ckpt,
                 void* du, void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                 float* ddt_bias, float* dh0, void* workspace, size_t workspace_bytes,
                 int batch, int dim, int seqlen, int dstate, int io_dtype, void* stream);

/*
 * Scalar decay: one rate A_d per channel shared by its N states (the restriction of the
 * transition to a scalar that the "2024 Reading List: Neural Network" page notes for Mamba-2,
 * section on state-space models).  The recurrence is the one above with A[d][n] = A_d:
 *   Ā_t = exp(Δ_t A_d) (one exponential per channel and step),  h_t = Ā_t h_{t-1} + Δ_t B_t x_t,
 *   y_t = C_t . h_t + D_d x_t,  out_t = y_t * silu(z_t).
 * Arguments, layouts, ownership and errors are those of ssm_scan_fwd / ssm_scan_bwd except:
 *   A   [dim] f32 (not [dim][dstate]);   dA (backward)  [dim] f32 = sum over n of dL/dA[d][n].
 * The backward needs ssm_scan_bwd_scalar_a_workspace_size() bytes of workspace (256-byte
 * aligned): A broadcast to [dim][dstate] and the per-state dA, followed by the workspace of
 * ssm_scan_bwd for the same shape.  Checkpoints of ssm_scan_fwd_scalar_a feed the backward.
 * dstate may be up to SSM_MAX_DSTATE_SCALAR in the forward scan: above 16 (and at 16 for bf16
 * calls in the default layout with no other flag) it runs in the chunked matrix form (per
 * 16-step chunk and 64-channel tile, the products C B^T, masked with the decay factors, times
 * the step-scaled inputs, plus C times the entering state: the structured-matrix view of the
 * scan in the Mamba-2 notes of the same page) on the tensor cores.  That form takes bf16 io,
 * dstate 16, 32, 64 or 128, the default layout and B/C groups of whole 64-channel tiles (with
 * SSM_ZOH: the coefficient (e^{ΔA} - 1)/A by the library expm1f).  f32 io with dstate a
 * multiple of 16 up to 128 (default layout, B/C shared or grouped) runs as the sum of the f32
 * 16-state forwards of the state slices: the first slice (with D) writes out, each further
 * slice's gated output is added to it in f32, and hL and ckpt are written slice by slice; its
 * workspace (ssm_scan_fwd_ex_workspace_size) holds the slice copies of B, C, h0, one slice's
 * hL, checkpoints and output, and the 16-state forward's own workspace.  Other forward requests
 * with dstate > 16 return SSM_EUNSUPPORTED.  With SSM_REVERSE
 * (dstate > 16; ssm_scan_fwd_ex) it scans the inputs mirrored along time into the workspace
 * and mirrors the output back in place, so ssm_scan_fwd_ex_workspace_size() then covers those
 * copies (u, delta, z, B, C) too.  Its checkpoints (ckpt, 16-byte aligned) have the layout and meaning of the
 * per-state scan's: the f32 state entering every 16-step block, [batch][dim][ceil(L/16)][dstate].
 * For bf16 io, no flag but SSM_SCALAR_A, SSM_ZOH and SSM_REVERSE (mirrored copies of u, delta,
 * z, dout, B, C in the workspace, the gradients along time mirrored back in place) and B/C shared or in
 * groups of whole 64-channel tiles, the backward with dstate = 16, 32, 64 or 128 runs in the
 * chunked matrix form too: the chunks
 * are walked in reverse with the adjoint of the state (the chain rule through the products
 * above), from the caller's checkpoints (either forward's; 16-byte aligned) or, with
 * ckpt = NULL, from a checkpoint pass into the workspace.  Other requests with dstate > 16
 * (f32, other groupings) take ckpt = NULL and run as the sum of the 16-state
 * backwards of the state slices (the states of a scalar-decay scan do not interact; D enters
 * one slice); with dstate <= 16 they run the per-state backward.
 * ssm_scan_bwd_scalar_a_workspace_size() covers the scratch of the path the call takes (chunk
 * states unless given, and per-CTA dB/dC partials; slice copies of B, C, h0, dhL, per-slice
 * gradients and f32 sums; or A broadcast plus the per-state backward's workspace).
 */
SSM_API size_t ssm_scan_fwd_scalar_a_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                    int io_dtype);
SSM_API int ssm_scan_fwd_scalar_a(const void* u, const void* delta, const float* A, const void* B,
                                  const void* C, const float* D, const void* z,
                                  const float* dt_bias, int delta_softplus, const float* h0,
                                  float* hL, void* out, float* ckpt, void* workspace,
                                  size_t workspace_bytes, int batch, int dim, int seqlen,
                                  int dstate, int io_dtype, void* stream);
SSM_API size_t ssm_scan_bwd_scalar_a_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                    int io_dtype, int have_ckpt);
SSM_API int ssm_scan_bwd_scalar_a(const void* u, const void* delta, const float* A, const void* B,
                                  const void* C, const float* D, const void* z,
                                  const float* dt_bias, int delta_softplus, const float* h0,
                                  const void* dout, const float* dhL, const float* ckpt, void* du,
                                  void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                                  float* ddt_bias, float* dh0, void* workspace,
                                  size_t workspace_bytes, int batch, int dim, int seqlen,
                                  int dstate, int io_dtype, void* stream);

/*
 * Variants of the scan selected by a bit mask (the _ex entry points; 0 = ssm_scan_fwd/_bwd):
 *   SSM_SCALAR_A  A (and dA) is [dim]: one decay rate per channel, as ssm_scan_fwd_scalar_a.
 *   SSM_REVERSE   the scan runs backwards in time, t = L-1 down to 0:
 *                   h_t = exp(Δ_t A) h_{t+1} + Δ_t B_t x_t  (h0 enters at t = L-1; hL is the
 *                   state after t = 0),  y_t = C_t . h_t + D x_t,
 *                 the anti-causal half of a bidirectional layer ("2024 Reading List: Neural
 *                 Network", Hydra notes: a forward and a backward scan whose outputs are summed).
 *                 Every tensor keeps its layout; the kernels read and write the time rows
 *                 mirrored.  Checkpoints are indexed by blocks of 16 steps in scan order
 *                 (block k holds the state before scan steps 16k .. 16k+15, i.e. before time
 *                 index L-1-16k), and only feed ssm_scan_bwd_ex with the same flags.
 *   SSM_ZOH       the zero-order-hold input term of the discretisation ("Yöntem":
 *                 B̄ = (ΔA)^{-1}(exp(ΔA) - I) ΔB): h_t = Ā h_{t-1} + c B_t x_t with
 *                 c = (exp(Δ_t A) - 1)/A per state (c -> Δ_t as A -> 0) instead of Δ_t.
 *                 Combines with the other flags.
 *   SSM_CHANNELS_LAST  the (B, L, D) layout: u, delta, z, out, dout, du, ddelta, dz are
 *                 [batch][L][dim] and B, C, dB, dC are [batch][L][bc_groups][dstate] (the
 *                 projections' own output layout); everything else as above.  With
 *                 dim % 16 == 0, dstate == 16 and 16-byte aligned tensors each warp moves
 *                 16-byte pieces (8 consecutive channels or states of one step) and transposes
 *                 them through shared memory; otherwise it uses element accesses (slower, same
 *                 results).
 * Any other bit is rejected with SSM_EINVAL.  Arguments are those of ssm_scan_fwd /
 * ssm_scan_bwd plus flags and bc_groups:
 *   bc_groups     B, C (and dB, dC) are [batch][bc_groups][dstate][L]: the per-token B_t, C_t
 *                 of the selection mechanism ("Seçim Mekanizması (S6)") computed once per group
 *                 of dim / bc_groups consecutive channels instead of once for all channels (the
 *                 grouping Mamba-2 uses; 1 = shared by every channel).  dim must be a multiple of
 *                 bc_groups (else SSM_EINVAL) and dim / bc_groups a multiple of 16 (the channels
 *                 of one warp share a group; else SSM_EUNSUPPORTED).
 *                 bc_groups == dim gives B, C (and dB, dC) per channel, [batch][dim][dstate][L]
 *                 (B_t, C_t computed from each channel's own input); dB, dC are then per channel,
 *                 not summed over d.  Per-channel B/C combines with no flag (SSM_EUNSUPPORTED).
 */
#define SSM_SCALAR_A 1
#define SSM_REVERSE 2
#define SSM_ZOH 4
#define SSM_CHANNELS_LAST 8
SSM_API size_t ssm_scan_fwd_ex_workspace_size(int batch, int dim, int seqlen, int dstate,
                                              int bc_groups, int io_dtype, int flags);
SSM_API int ssm_scan_fwd_ex(const void* u, const void* delta, const float* A, const void* B,
                            const void* C, const float* D, const void* z, const float* dt_bias,
                            int delta_softplus, const float* h0, float* hL, void* out, float* ckpt,
                            void* workspace, size_t workspace_bytes, int batch, int dim,
                            int seqlen, int dstate, int bc_groups, int io_dtype, int flags,
                            void* stream);
SSM_API size_t ssm_scan_bwd_ex_workspace_size(int batch, int dim, int seqlen, int dstate,
                                              int bc_groups, int io_dtype, int have_ckpt,
                                              int flags);
SSM_API int ssm_scan_bwd_ex(const void* u, const void* delta, const float* A, const void* B,
                            const void* C, const float* D, const void* z, const float* dt_bias,
                            int delta_softplus, const float* h0, const void* dout,
                            const float* dhL, const float* ckpt, void* du, void* ddelta, float* dA,
                            void* dB, void* dC, float* dD, void* dz, float* ddt_bias, float* dh0,
                            void* workspace, size_t workspace_bytes, int batch, int dim,
                            int seqlen, int dstate, int bc_groups, int io_dtype, int flags,
                            void* stream);

/*
 * ssm_scan_fwd from and to HOST memory.  The pages have no counterpart: this is the call a user
 * makes when sequences live in host memory.  The batch is cut into chunks of rows that flow
 * through three streams (host-to-device copies, the scan, device-to-host copies), so the copies
 * of one chunk overlap the scan of another and the two copy directions overlap each other.
 *   u, delta, z, out  [batch][dim][L] io       HOST (page-locked memory lets the copies overlap;
 *   B, C              [batch][N][L] io         HOST   pageable memory works but serialises them)
 *   h0, hL            [batch][dim][N] f32      HOST, or NULL
 *   A, D, dt_bias     as for ssm_scan_fwd      DEVICE (model parameters stay on the GPU)
 *   workspace         DEVICE, 256-byte aligned, ssm_scan_fwd_host_workspace_size() bytes
 * Asynchronous with respect to the host: the output is complete once `stream` has reached this
 * point (e.g. after cudaStreamSynchronize(stream)); work queued on `stream` before the call runs
 * first.  The three streams and their events are created on a device's first call and kept until
 * the process exits; calls from several host threads on one device are serialised while they
 * enqueue.  Errors as for ssm_scan_fwd; a copy failure returns SSM_ECUDA.
 */
SSM_API size_t ssm_scan_fwd_host_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                int io_dtype);
SSM_API int ssm_scan_fwd_host(const void* u, const void* delta, const float* A, const void* B,
                              const void* C, const float* D, const void* z, const float* dt_bias,
                              int delta_softplus, const float* h0, float* hL, void* out,
                              void* workspace, size_t workspace_bytes, int batch, int dim,
                              int seqlen, int dstate, int io_dtype, void* stream);

/* Size of the static scratch array used by ssm_scan_fwd_noalloc (8 MiB per GPU). */
#define SSM_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * ssm_scan_fwd without a workspace, for callers that cannot allocate device memory (a process
 * that handed all device memory to its own pool at start-up, a plugin whose host application
 * owns every allocation, or a hot path that must not call cudaMalloc because it can synchronise
 * the device).  The pages have no counterpart: this is a deployment variant of the forward scan.
 * Arguments, layouts, results and errors are those of ssm_scan_fwd, minus the workspace.  The
 * time-split scratch comes from one static device array of SSM_NOALLOC_SCRATCH_BYTES that every
 * GPU loading the library keeps until the process exits; shapes whose plan needs more return
 * SSM_EUNSUPPORTED (ssm_last_error() says how much) and launch nothing.  No call allocates or
 * frees memory.  The first call on each device (and the first after that device's context
 * changes, e.g. after cudaDeviceReset) looks up the array's device address with that device
 * current; make that first call before any stream capture.  All calls on a device share
 * the array: calls whose GPU work overlaps (other streams, other host threads) race on it.
 */
SSM_API int ssm_scan_fwd_noalloc(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z,
                                 const float* dt_bias, int delta_softplus, const float* h0,
                                 float* hL, void* out, float* ckpt, int batch, int dim,
                                 int seqlen, int dstate, int io_dtype, void* stream);

/*
 * One-token recurrent step ("Sorular": fixed D x N state per layer, O(1) per token).
 *   state     [batch][dim][dstate] f32    IN/OUT, updated in place: h <- exp(ΔA) h + Δ B x
 *   x, dt, z  [batch][dim] io            token input, raw step, gate input (z may be NULL)
 *   A [dim][dstate] f32;  B, C [batch][dstate] io;  D, dt_bias [dim] f32 or NULL
 *   out       [batch][dim] io             OUT: (C.h + D x) * silu(z)
 * Calling it L times reproduces ssm_scan_fwd over L steps (same arithmetic per step).
 */
SSM_API int ssm_state_update(float* state, const void* x, const void* dt, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* dt_bias,
                     int delta_softplus, void* out, int batch, int dim, int dstate,
                     int io_dtype, void* stream);

/*
 * ssm_state_update with the variants of the scan: flags SSM_SCALAR_A (A is [dim]) and SSM_ZOH
 * (the zero-order-hold input coefficient); B, C are [batch][bc_groups][dstate] (channel d uses
 * group d / (dim / bc_groups); dim / bc_groups a multiple of 16 when 1 < bc_groups < dim;
 * bc_groups == dim gives B, C per channel, [batch][dim][dstate]).  A decode
 * step runs forward in time: SSM_REVERSE is rejected with SSM_EINVAL, as is any unknown bit.
 * Calling it L times reproduces ssm_scan_fwd_ex with the same flags and groups.  With
 * SSM_SCALAR_A, dstate may also be 32, 64 or 128 (the state sizes of the chunked scan; the
 * state 16-byte aligned, else SSM_EINVAL); other dstate > 16 return SSM_EUNSUPPORTED.
 */
SSM_API int ssm_state_update_ex(float* state, const void* x, const void* dt, const float* A,
                                const void* B, const void* C, const float* D, const void* z,
                                const float* dt_bias, int delta_softplus, void* out, int batch,
                                int dim, int dstate, int bc_groups, int io_dtype, int flags,
                                void* stream);

/*
 * Number of bounded waits that ran out on the current device since the library was loaded
 * (the pages have no counterpart: this reports on the library's own kernels).  The streamed
 * decode step waits on shared-memory barriers for its bulk copies; each wait gives up after a
 * fixed number of polls, counts a timeout here, lets the copies in flight land and returns
 * (that call's outputs are then incomplete).  0 means every wait completed.  Synchronises with
 * the device (it reads a device counter).  Returns SSM_OK, or SSM_EINVAL for a NULL pointer,
 * or SSM_ECUDA if the counter cannot be read.
 */
SSM_API int ssm_wait_timeouts(unsigned int* count);

/*
 * Sequence split (a long sequence cut into consecutive segments, e.g. one per GPU).  The scan is
 * a composition of affine maps of the state ("Temel Fikirler": the recurrence is a parallel
 * associative scan): a segment with steps Δ_t maps the state entering it to
 *   h_out = exp(A ΣΔ) h_in + hend,
 * where hend is the segment's end state from a zero state (per state n: exp(A_n ΣΔ)).
 *
 * ssm_scan_fwd_summary: the map of one segment.  Arguments as ssm_scan_fwd_ex (flags
 *   SSM_SCALAR_A and SSM_ZOH; shared or grouped B/C), plus
 *     hend  [batch][dim][dstate] f32   OUT: the state after the segment from a zero state
 *     dsum  [batch][dim] f32 or NULL   OUT: ΣΔ over the segment (Kahan-summed in f32)
 *   and ssm_scan_fwd_summary_workspace_size() bytes of workspace (256-byte aligned).
 *   With SSM_SCALAR_A, dstate may exceed 16 as in the scalar-decay scan: bf16 with dstate 32,
 *   64 or 128 and B/C shared or in groups of whole 64-channel tiles runs the chunked matrix
 *   form's summary pass over the planner's segments and chains them; f32 with dstate a multiple
 *   of 16 up to 128 sums 16-state slices (C is not read then).
 * ssm_scan_chain: the state entering each of nseg consecutive segments,
 *     hin[0] = h0 (zero if NULL),  hin[r+1] = exp(A dsum[r]) hin[r] + hend[r],
 *   hend, hin [nseg][batch][dim][dstate] f32, dsum [nseg][batch][dim] f32, A as for the scan
 *   (flags: SSM_SCALAR_A, which allows dstate up to SSM_MAX_DSTATE_SCALAR).  Running each
 *   segment's forward scan from its hin[r] gives the full-sequence results, up to rounding.
 * Errors as for the scans.
 */
SSM_API size_t ssm_scan_fwd_summary_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                   int bc_groups, int io_dtype, int flags);
SSM_API int ssm_scan_fwd_summary(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* dt_bias, int delta_softplus,
                                 float* hend, float* dsum, void* workspace,
                                 size_t workspace_bytes, int batch, int dim, int seqlen,
                                 int dstate, int bc_groups, int io_dtype, int flags, void* stream);
SSM_API int ssm_scan_chain(const float* hend, const float* dsum, const float* A, const float* h0,
                           float* hin, int nseg, int batch, int dim, int dstate, int flags,
                           void* stream);

/*
 * General element strides.  The entry points above take dense tensors (the layouts given per
 * argument, or the (B, L, D) layout of SSM_CHANNELS_LAST).  These take each io tensor with its
 * own element strides, e.g. views cut out of a larger projection output, transposed views, or B
 * and C broadcast over the batch with stride 0 ("Seçim Mekanizması (S6)": the selective
 * parameters come from projections of the input, in whatever layout those produce).  Strides
 * are in elements, one per index of the tensor's logical shape:
 *   [batch][dim][L] tensors (u, delta, z, out, dout, du, ddelta, dz): (batch, dim, t)
 *   [batch][bc_groups][dstate][L] tensors (B, C, dB, dC): (batch, group, state, t)
 * Strides must be >= 0; an output's strides must not map two of its elements to one address
 * (SSM_EINVAL otherwise).  Each tensor's allocation must hold every element the strides reach.
 * A tensor whose strides are the dense ones is used in place; any other is gathered into (or,
 * for an output, scattered from) a dense copy in the workspace by the library's own copy kernel
 * around the dense call, so the results equal those of the dense entry points bitwise.  f32
 * tensors (A, D, dt_bias, h0, hL, ckpt, dhL, dA, dD, ddt_bias, dh0) stay dense.  flags:
 * SSM_SCALAR_A, SSM_REVERSE, SSM_ZOH (SSM_CHANNELS_LAST is one set of strides: SSM_EINVAL).
 * The workspace holds the dense copies followed by the dense call's workspace; its size does not
 * depend on the strides.
 */
typedef struct ssm_strides {
  long long u[3], delta[3], z[3], out[3];      /* forward tensors: (batch, dim, t) */
  long long dout[3], du[3], ddelta[3], dz[3];  /* backward tensors: (batch, dim, t) */
  long long B[4], C[4], dB[4], dC[4];          /* (batch, group, state, t) */
} ssm_strides;

SSM_API size_t ssm_scan_fwd_strided_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                   int bc_groups, int io_dtype, int flags);
SSM_API int ssm_scan_fwd_strided(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z,
                                 const float* dt_bias, int delta_softplus, const float* h0,
                                 float* hL, void* out, float* ckpt, void* workspace,
                                 size_t workspace_bytes, int batch, int dim, int seqlen,
                                 int dstate, int bc_groups, int io_dtype, int flags,
                                 const ssm_strides* strides, void* stream);
SSM_API size_t ssm_scan_bwd_strided_workspace_size(int batch, int dim, int seqlen, int dstate,
                                                   int bc_groups, int io_dtype, int have_ckpt,
                                                   int flags);
SSM_API int ssm_scan_bwd_strided(const void* u, const void* delta, const float* A, const void* B,
                                 const void* C, const float* D, const void* z,
                                 const float* dt_bias, int delta_softplus, const float* h0,
                                 const void* dout, const float* dhL, const float* ckpt, void* du,
                                 void* ddelta, float* dA, void* dB, void* dC, float* dD, void* dz,
                                 float* ddt_bias, float* dh0, void* workspace,
                                 size_t workspace_bytes, int batch, int dim, int seqlen,
                                 int dstate, int bc_groups, int io_dtype, int flags,
                                 const ssm_strides* strides, void* stream);

/*
 * The decode step with general element strides (same rules as above):
 *   state (batch, dim, state) f32, updated in place;  x, dt, z, out (batch, dim) io;
 *   B, C (batch, group, state) io.
 * flags: SSM_SCALAR_A, SSM_ZOH.  Needs ssm_state_update_strided_workspace_size() bytes of
 * workspace (256-byte aligned) for the dense copies.
 */
typedef struct ssm_decode_strides {
  long long state[3];
  long long x[2], dt[2], z[2], out[2];
  long long B[3], C[3];
} ssm_decode_strides;

SSM_API size_t ssm_state_update_strided_workspace_size(int batch, int dim, int dstate,
                                                       int bc_groups, int io_dtype);
SSM_API int ssm_state_update_strided(float* state, const void* x, const void* dt, const float* A,
                                     const void* B, const void* C, const float* D, const void* z,
                                     const float* dt_bias, int delta_softplus, void* out,
                                     void* workspace, size_t workspace_bytes, int batch, int dim,
                                     int dstate, int bc_groups, int io_dtype, int flags,
                                     const ssm_decode_strides* strides, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H_ */
