/*
 * mamba_scan.h -- C ABI of the B200 (sm_100a) selective-scan library.
 *
 * The library computes the selective state-space (S6) layer of Mamba:
 *
 *   delta_t = softplus(delta_raw_t + delta_bias[d])        (softplus optional)
 *   Abar    = exp(delta_t * A[d, n])                       (zero-order hold of A)
 *   h_t[n]  = Abar * h_{t-1}[n] + delta_t * B[b, n, t] * u_t
 *   y_t     = sum_n C[b, n, t] * h_t[n] + D[d] * u_t
 *   out_t   = y_t * silu(z_t)                              (gate optional)
 *
 * Sources: "Mamba SSM concept and implementation in Keras and TensorFlow"
 * (sections on the continuous SSM, its zero-order-hold discretisation and the
 * recurrent form, the selective_scan listing with dA = delta*A,
 * dB_u = delta*u*B and y + u*D, and MambaBlock.call, y * swish(res));
 * "Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
 * Appendix E.5 (the scan fuses discretisation with the recurrence and does not
 * write the expanded (batch, L, dim, N) parameters to HBM); the state-spaces
 * mamba README (the selective-scan interface and the Mamba(d_model,
 * d_state=16, d_conv=4, expand=2) block that wraps it).
 *
 * Entry points
 * ------------
 *   forward scan      mamba_scan_fwd, _tuned, _ws (workspace: persistent
 *                     schedule), _noalloc, _init (from a given state),
 *                     _strided (any strides), _complex (complex mode),
 *                     _conv (causal conv1d + silu fused in), _host (sequences
 *                     in host memory); mamba_scan_plan, mamba_scan_plan_noworkspace,
 *                     mamba_scan_workspace_size,
 *                     mamba_scan_host_scratch_size
 *   decoding          mamba_state_update (one token), mamba_conv1d_update
 *   conv1d            mamba_conv1d_fwd
 *   backward          mamba_scan_bwd, mamba_scan_bwd_init, mamba_scan_bwd_workspace_size;
 *                     mamba_scan_fwd_ckpt / mamba_scan_bwd_ckpt (the forward
 *                     keeps the states the backward recomputes from),
 *                     mamba_scan_ckpt_size
 *   sequence split    mamba_delta_sum, mamba_state_fold
 *   status            mamba_scan_workspace_status, mamba_get_device_status,
 *                     mamba_status_string, mamba_abi_version;
 *                     mamba_debug_stall_group (test hook); the bounds-checked
 *                     build: mamba_bounds_checked, mamba_debug_bounds_status,
 *                     mamba_debug_shrink_output_extent (test hook)
 *
 * Conventions for every entry point
 * ---------------------------------
 * - Pointers are DEVICE pointers (cudaMalloc'd, managed, or mapped pinned host
 *   memory) of the current CUDA device, except where stated.  Tensors are
 *   dense, row-major and contiguous with the layouts given per function,
 *   except where strides are given.
 * - "act" tensors (u, delta, z, B, C, out) share one element type chosen by
 *   `act_dtype` (MAMBA_F32 or MAMBA_BF16).  A, D, delta_bias, states are
 *   always fp32.  All arithmetic is fp32.
 * - The caller owns every buffer.  The library allocates no memory (the
 *   host-memory scan creates and releases two streams and seven events per
 *   call) and only mamba_scan_workspace_status and mamba_get_device_status
 *   synchronise: work is enqueued on `stream` (0 = legacy default stream) and
 *   buffers must stay alive until that work completes.
 * - Argument validation is synchronous and happens before anything is
 *   enqueued; a non-zero return means nothing was enqueued, except
 *   MAMBA_ERR_CUDA, which reports a launch failure (cudaGetLastError).
 * - Alignment never fails: 16-byte-aligned act pointers with seqlen a multiple
 *   of the 16-byte vector width take the vectorised path, others a scalar path.
 * - `out` may alias exactly one of u, delta or z (same pointer, in-place);
 *   any other overlap between an output and an input is rejected.
 * - Calls are reentrant and thread-safe, with one exception:
 *   mamba_scan_fwd_noalloc calls share one scratch area per device, so the
 *   caller must serialise them (see there).  Library state: per device, the
 *   workspace pointer of the last persistent launch and the local schedule's
 *   timeout word (both for mamba_get_device_status), and the scratch area of
 *   mamba_scan_fwd_noalloc; process-wide, the mamba_debug_stall_group and
 *   mamba_debug_shrink_output_extent test hooks (off by default).
 */
#ifndef MAMBA_SCAN_H
#define MAMBA_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#ifndef __CUDA_RUNTIME_H__
typedef struct CUstream_st *cudaStream_t; /* identical to the CUDA runtime's typedef */
#endif

typedef enum {
    MAMBA_F32 = 0,  /* IEEE binary32 */
    MAMBA_BF16 = 1  /* bfloat16; stores round to nearest even */
} mamba_dtype_t;

typedef enum {
    MAMBA_OK = 0,
    MAMBA_ERR_NULL = -1,        /* a required pointer is NULL */
    MAMBA_ERR_SHAPE = -2,       /* a size is <= 0 or too large to index */
    MAMBA_ERR_UNSUPPORTED = -3, /* dstate outside [1, 64], unknown dtype, bad tuning */
    MAMBA_ERR_ALIGN = -4,       /* reserved (alignment selects a path, never fails) */
    MAMBA_ERR_CUDA = -5,        /* the CUDA runtime reported an error at launch */
    MAMBA_ERR_DEVICE = -6,      /* no usable CUDA device */
    MAMBA_ERR_OVERLAP = -7,     /* an output partially overlaps an input */
    MAMBA_ERR_WORKSPACE = -8,   /* workspace too small or misaligned */
    MAMBA_ERR_TIMEOUT = -9,     /* a persistent launch gave up waiting (see
                                   mamba_scan_workspace_status) */
    MAMBA_ERR_BOUNDS = -10      /* bounds-checked build only: a kernel access
                                   fell outside its tensor and was skipped */
} mamba_status_t;

/* Launch schedules of the scan. */
typedef enum {
    MAMBA_SCHEDULE_AUTO = 0,
    MAMBA_SCHEDULE_STATIC = 1,     /* one block per channel group walks the whole
                                      sequence; no workspace */
    MAMBA_SCHEDULE_PERSISTENT = 2, /* dstate <= 16: persistent warps, all
                                      resident; 2 or 4 lanes per channel split
                                      the (channel group, sub-chunk) grid into
                                      equal contiguous shares, 1 lane per
                                      channel takes (group, time chunk) units
                                      from a ready queue; states pass between
                                      pieces through the workspace */
    MAMBA_SCHEDULE_LOCAL = 3       /* dstate <= 16, 2 or 4 lanes per channel:
                                      one block per SM takes whole channel
                                      groups and splits their sub-chunks among
                                      its own warps; states pass between
                                      pieces through shared memory; no
                                      workspace */
} mamba_schedule_t;

/* Optional launch tuning.  Zero fields mean "choose automatically".
 *   lanes_per_channel : threads sharing one channel's states.  Static
 *                       schedule: 1, 2, 4, 8 or 16 (the padded dstate must be
 *                       a multiple, and at most 16 states stay in one
 *                       thread).  Persistent schedule: 1, 2 or 4.  Local
 *                       schedule: 2 or 4.
 *   threads_per_block : static schedule only: 128 or 256
 *   schedule          : a mamba_schedule_t
 *   chunk_timesteps   : persistent schedule only: timesteps per work unit
 *                       (rounded up to the kernel's staging granularity)
 */
typedef struct {
    int lanes_per_channel;
    int threads_per_block;
    int schedule;
    int chunk_timesteps;
} mamba_scan_tuning_t;

/*
 * mamba_scan_fwd -- fused selective scan forward over a whole sequence.
 *
 * Defining passage: the recurrent form of the discretised SSM and the
 * selective_scan listing of "Mamba SSM concept and implementation in Keras
 * and TensorFlow"; the fused, HBM-avoiding scan of Appendix E.5 of the Mamba
 * paper.
 *
 *   u, delta, z  : act (batch, dim, seqlen).  delta is the raw step before the
 *                  bias and softplus.  z may be NULL (no gate).
 *   A            : fp32 (dim, dstate); the (usually negative) real diagonal A.
 *   B, C         : act (batch, dstate, seqlen); shared by every channel of a
 *                  batch row.
 *   D            : fp32 (dim) or NULL (no skip term).
 *   delta_bias   : fp32 (dim) or NULL (zero bias).
 *   delta_softplus: non-zero applies softplus to delta_raw + delta_bias.
 *   out          : act (batch, dim, seqlen), written.
 *   last_state   : fp32 (batch, dim, dstate) or NULL; receives h_{seqlen-1}.
 *   The state starts from zero.
 *
 * Needs no workspace.  With dstate <= 16, 16-byte-aligned act tensors and
 * seqlen a multiple of the 16-byte vector width, shapes with enough channels
 * run the local schedule (MAMBA_SCHEDULE_LOCAL); others the static one.  A
 * local launch whose bounded wait between warps ran out (it cannot, except
 * under the mamba_debug_stall_group test hook) is reported by
 * mamba_get_device_status.
 *
 * Returns MAMBA_OK or a mamba_status_t error.
 */
int mamba_scan_fwd(const void *u, const void *delta, const float *A,
                   const void *B, const void *C, const float *D,
                   const void *z, const float *delta_bias, int delta_softplus,
                   void *out, float *last_state, int64_t batch, int64_t dim,
                   int64_t seqlen, int64_t dstate, int act_dtype,
                   cudaStream_t stream);

/* mamba_scan_fwd with an explicit launch configuration (same results up to
 * fp32 rounding order; NULL tuning is identical to mamba_scan_fwd).  Invalid
 * tuning returns MAMBA_ERR_UNSUPPORTED. */
int mamba_scan_fwd_tuned(const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *D,
                         const void *z, const float *delta_bias,
                         int delta_softplus, void *out, float *last_state,
                         int64_t batch, int64_t dim, int64_t seqlen,
                         int64_t dstate, int act_dtype,
                         const mamba_scan_tuning_t *tuning,
                         cudaStream_t stream);

/* The launch configuration mamba_scan_fwd_ws would pick for these sizes on
 * the current device, given a large enough workspace and 16-byte-aligned
 * tensors (fields filled in `plan`), without launching anything.
 * Returns MAMBA_OK or a validation error. */
int mamba_scan_plan(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                    int act_dtype, mamba_scan_tuning_t *plan);

/* The launch configuration mamba_scan_fwd (no workspace) would pick for these
 * sizes on the current device, with 16-byte-aligned tensors; as
 * mamba_scan_plan otherwise. */
int mamba_scan_plan_noworkspace(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                                int act_dtype, mamba_scan_tuning_t *plan);

/* Bytes of device workspace mamba_scan_fwd_ws may use for these sizes (an
 * upper bound valid on every device); 0 when the persistent schedule never
 * applies (dstate > 16).  Pure host arithmetic. */
size_t mamba_scan_workspace_size(int64_t batch, int64_t dim, int64_t seqlen,
                                 int64_t dstate, int act_dtype);

/*
 * mamba_scan_fwd_ws -- mamba_scan_fwd plus a caller-owned device workspace
 * (at least mamba_scan_workspace_size bytes, 16-byte aligned) that enables
 * the persistent, load-balanced schedule.  Same arguments and results as
 * mamba_scan_fwd.  The workspace holds the work queue and the states carried
 * between time chunks; its queue part is zeroed on `stream` before the
 * launch, so one workspace must not be used by two launches that can run at
 * the same time.  When the persistent schedule does not apply (dstate > 16,
 * unaligned tensors, too few channel groups to fill the GPU) the static
 * schedule runs and the workspace is not touched.  `tuning` may be NULL.
 */
int mamba_scan_fwd_ws(const void *u, const void *delta, const float *A,
                      const void *B, const void *C, const float *D,
                      const void *z, const float *delta_bias,
                      int delta_softplus, void *out, float *last_state,
                      int64_t batch, int64_t dim, int64_t seqlen,
                      int64_t dstate, int act_dtype,
                      const mamba_scan_tuning_t *tuning, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/*
 * mamba_scan_fwd_init -- mamba_scan_fwd_ws from a given initial state
 * instead of zeros: the recurrence starts from h_{-1} = h0 (the pages unroll
 * it from a zero state; a nonzero start continues an earlier scan -- pass
 * that scan's last_state -- without replaying it).
 *
 *   h0           : fp32 (batch, dim, dstate), required; read only.  It may
 *                  be the same buffer as last_state (exactly), which then
 *                  advances in place; any other overlap with an output is
 *                  rejected.
 *
 * All other arguments, results and errors as mamba_scan_fwd_ws (workspace
 * may be NULL: static schedule).
 */
int mamba_scan_fwd_init(const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, void *out,
                        float *last_state, int64_t batch, int64_t dim,
                        int64_t seqlen, int64_t dstate, int act_dtype,
                        const mamba_scan_tuning_t *tuning, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/*
 * mamba_scan_state -- the final state of the scan alone: last_state =
 * h_{L-1} of the recurrence of mamba_scan_fwd_init (steps a2-a4 and a7 of the
 * S6 forward), without the readout, gate or outputs.  This is what one shard
 * of a sequence split over several GPUs contributes before the exchange
 * (its state from a zero start; the shards are then folded with
 * mamba_state_fold), and the way to advance a state over a prompt whose
 * outputs are not wanted.
 *
 *   u, delta     : act (batch, dim, seqlen), as mamba_scan_fwd.
 *   A            : fp32 (dim, dstate); delta_bias fp32 (dim) or NULL.
 *   B            : act (batch, dstate, seqlen).  C, D and z take no part.
 *   h0           : fp32 (batch, dim, dstate) or NULL (zeros); may be
 *                  last_state exactly (advanced in place).
 *   last_state   : fp32 (batch, dim, dstate), required, written.
 *   workspace    : NULL (block-local lane-split kernel, no workspace) or at
 *                  least mamba_scan_workspace_size bytes, 16-byte aligned
 *                  (device-wide form).
 *
 * The lane-split kernel runs every piece of each channel group's sequence
 * state-only from a zero start (no C rows, readout, gate or stores; delta
 * summed in fp64) and combines it with the state before the piece as
 * exp(A sum(delta)) h_in + h_piece: about three quarters of a full scan.
 * Results agree with mamba_scan_fwd_init's last_state within the tolerance,
 * not bit for bit (the pieces are combined in another order).
 * Requires dstate <= 16 and 16-byte aligned rows of a whole number of
 * 16-byte vectors (as the lane-split schedules): else MAMBA_ERR_UNSUPPORTED.
 * Errors: MAMBA_ERR_NULL, MAMBA_ERR_SHAPE, MAMBA_ERR_OVERLAP (last_state over
 * an input, a workspace over anything), MAMBA_ERR_WORKSPACE (misaligned or
 * small), MAMBA_ERR_CUDA.
 */
int mamba_scan_state(const void *u, const void *delta, const float *A,
                     const void *B, const float *delta_bias, int delta_softplus,
                     const float *h0, float *last_state, int64_t batch,
                     int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                     void *workspace, size_t workspace_bytes,
                     cudaStream_t stream);

/* Element strides of one sequence tensor: along the batch, along its rows
 * (channels for u / delta / z / out, states for B / C) and along time. */
typedef struct {
    int64_t batch;
    int64_t row;
    int64_t time;
} mamba_stride3_t;

typedef struct {
    mamba_stride3_t u, delta, z, out, B, C;
} mamba_scan_strides_t;

/*
 * mamba_scan_fwd_strided -- mamba_scan_fwd_init with every sequence tensor
 * given by its own element strides instead of the dense (batch, dim, seqlen)
 * / (batch, dstate, seqlen) layout.  This reads a model's activations where
 * they already are: the (batch, seqlen, dim) layout the pages' Keras listing
 * uses (channels contiguous, "b l d"), slices of a wider projection output
 * (x and z as the two halves of one (batch, seqlen, 2 dim) tensor; B and C as
 * columns of one (batch, seqlen, R + 2 dstate) tensor), B or C shared by
 * every batch row (batch stride 0), or the dense layout itself.
 *
 *   strides      : element strides (>= 0) of u, delta, z, out, B and C;
 *                  NULL means dense.  z's entry is ignored when z is NULL.
 *   h0           : fp32 (batch, dim, dstate) or NULL (zeros); as for
 *                  mamba_scan_fwd_init.
 *   out          : its strides must not map two elements to one address.
 *                  out may be u, delta or z in place only with the same
 *                  pointer and strides; any other overlap of out, last_state
 *                  or h0 with an input is rejected (MAMBA_ERR_OVERLAP, judged
 *                  on each tensor's address span).
 *   tuning       : NULL, or schedule AUTO / LOCAL / STATIC with optional
 *                  lanes and threads (PERSISTENT needs the dense layout and a
 *                  workspace: MAMBA_ERR_UNSUPPORTED).
 *
 * The pages' own layout -- u, delta, z and out dense (batch, seqlen, dim),
 * i.e. strides (seqlen dim, 1, dim), and B, C dense (batch, seqlen, dstate),
 * strides (seqlen dstate, 1, dstate) -- runs on the block-local lane-split
 * kernel of mamba_scan_fwd (no workspace), staging each timestep's channels
 * with 16-byte copies: results bit-equal to mamba_scan_fwd on the same values
 * laid out densely with the same lane count.  It needs dstate <= 16, dim and
 * dstate multiples of 8 (bf16) or 4 (fp32), 16-byte-aligned pointers, lanes
 * 0 / 2 / 4 and no block size; schedule LOCAL insists on it
 * (MAMBA_ERR_UNSUPPORTED otherwise), AUTO falls back to the static kernel.
 * Every other layout, and schedule STATIC, uses the static schedule.  There
 * 16-byte copies are used where a tensor allows them: channel-contiguous u /
 * delta / z / out (row stride 1) with 16-byte-aligned pointers, batch and
 * time strides multiples of 8 (bf16) or 4 (fp32) elements and dim a multiple
 * of the same; time-contiguous ones likewise with the row stride and seqlen;
 * B and C likewise along time or along states.  Anything else is read and
 * written element by element (correct, slower).  Other arguments, results
 * and errors as mamba_scan_fwd.
 */
int mamba_scan_fwd_strided(const void *u, const void *delta, const float *A,
                           const void *B, const void *C, const float *D,
                           const void *z, const float *delta_bias,
                           int delta_softplus, const float *h0, void *out,
                           float *last_state, int64_t batch, int64_t dim,
                           int64_t seqlen, int64_t dstate, int act_dtype,
                           const mamba_scan_strides_t *strides,
                           const mamba_scan_tuning_t *tuning,
                           cudaStream_t stream);

/*
 * mamba_scan_fwd_complex -- the scan in complex-valued mode: a complex
 * diagonal A and complex, input-dependent B and C (the complex SSM the Mamba
 * paper compares with the real one on audio, Appendix E.4.1; the "complex
 * number mode" on the roadmap of the "Mamba x JAX" page).  The pages give no
 * formulas for it; this is the real recurrence over the complex numbers with
 * the real part of the readout as output:
 *
 *   delta = softplus(delta_raw + delta_bias[d])            (real)
 *   Abar  = exp(delta A[d,n])                               (complex)
 *   h[n]  = Abar h[n] + delta B[b,n,t] u[b,d,t]             (complex)
 *   y     = Re(sum_n C[b,n,t] h[n]) + D[d] u[b,d,t];  out = y silu(z)
 *
 *   u, delta, z, out : act (batch, dim, seqlen), as mamba_scan_fwd.
 *   A            : fp32 (dim, dstate, 2): (re, im) pairs.
 *   B, C         : act (batch, dstate, seqlen, 2): (re, im) pairs.
 *   h0           : fp32 (batch, dim, dstate, 2) or NULL (zeros); may be
 *                  last_state exactly.
 *   last_state   : fp32 (batch, dim, dstate, 2) or NULL.
 *   tuning       : NULL or schedule AUTO / STATIC with lanes_per_channel
 *                  0 (auto), 1, 2 or 4; other fields 0.
 *
 * dstate <= 16.  Each state-step takes three special-function ops (ex2, sin,
 * cos).  Aliasing rules and errors as mamba_scan_fwd.
 */
int mamba_scan_fwd_complex(const void *u, const void *delta, const float *A,
                           const void *B, const void *C, const float *D,
                           const void *z, const float *delta_bias,
                           int delta_softplus, const float *h0, void *out,
                           float *last_state, int64_t batch, int64_t dim,
                           int64_t seqlen, int64_t dstate, int act_dtype,
                           const mamba_scan_tuning_t *tuning,
                           cudaStream_t stream);

/*
 * mamba_scan_fwd_host -- mamba_scan_fwd_init for sequences in HOST memory:
 * the scan of a model whose activations do not stay on the GPU, or of a
 * problem larger than the device.  The (batch, channel) rows are cut into
 * chunks (channel ranges of one batch row); for each chunk the inputs are
 * copied host -> device on an internal stream, the scan runs on `stream`,
 * and the outputs are copied back on a second internal stream, through two
 * device slots, so both copy directions and the scans overlap.
 *
 *   u, delta, z, B, C : HOST, layouts of mamba_scan_fwd (z may be NULL).
 *                  Page-locked (pinned) memory lets the copies run
 *                  asynchronously; pageable memory works but serialises them.
 *   out          : HOST act (batch, dim, seqlen), written.
 *   last_state   : HOST fp32 (batch, dim, dstate) or NULL.
 *   A, D, delta_bias, h0 : DEVICE, as for mamba_scan_fwd_init (h0 may be NULL).
 *   scratch      : DEVICE, at least mamba_scan_host_scratch_size bytes,
 *                  16-byte aligned, caller-owned; must not overlap A, D,
 *                  delta_bias or h0.
 *
 * Stream-ordered like the other entry points: the copies start after the
 * work already queued on `stream`, and `stream` waits for the last copy
 * back; host buffers must stay valid (and out unread) until then.  Returns
 * MAMBA_OK or a mamba_status_t error (MAMBA_ERR_WORKSPACE for a missing or
 * small scratch; an error of a chunk's scan is returned as is).
 */
size_t mamba_scan_host_scratch_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                                    int act_dtype);
int mamba_scan_fwd_host(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, void *out, float *last_state,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        void *scratch, size_t scratch_bytes, cudaStream_t stream);

/*
 * mamba_scan_fwd_conv -- the causal depthwise conv1d + silu fused into the
 * scan's prologue: the step before the scan in the Mamba block ("Mamba SSM
 * concept and implementation in Keras and TensorFlow", MambaBlock: Conv1D
 * with one group per channel, causal padding, bias, then swish) computed
 * where the scan loads u, so u never makes a round trip through HBM:
 *
 *   u[b,d,t] = silu(conv_bias[d] + sum_{k<K} conv_weight[d,k] x[b,d,t-(K-1)+k]),
 *              x = 0 before the sequence, u rounded to the activation type,
 *   then the scan of mamba_scan_fwd_init on that u, softplus on.
 *
 * The result equals mamba_conv1d_fwd followed by mamba_scan_fwd_ws bit for
 * bit.
 *
 *   x            : act; channel d of batch row b is the seqlen-long row at
 *                  x + b * x_batch_stride + d * seqlen (0: dim * seqlen) --
 *                  e.g. the x half of the in-projection's (batch, 2 dim,
 *                  seqlen) output.
 *   conv_weight  : fp32 (dim, conv_width), conv_width 1 .. 4; conv_bias:
 *                  fp32 (dim) or NULL.
 *   z            : act or NULL, rows at z + b * z_batch_stride + d * seqlen
 *                  (0: dim * seqlen) -- e.g. the other half of the same
 *                  output; x and z may share one buffer.
 *   u_out        : act (batch, dim, seqlen) or NULL: the u it formed (what a
 *                  backward pass needs).
 *   h0           : fp32 (batch, dim, dstate) or NULL; may be last_state.
 *   other arguments as mamba_scan_fwd_ws; the workspace is required.
 *
 * The fused prologue lives in the persistent lane-split kernel, so the
 * call needs its layout: dstate <= 16, 16-byte-aligned tensors, seqlen and
 * both batch strides multiples of 8 (bf16) or 4 (fp32) elements; otherwise
 * MAMBA_ERR_UNSUPPORTED (run the two calls instead).  out, u_out and
 * last_state must not overlap any input (h0 == last_state excepted) or
 * each other.
 */
int mamba_scan_fwd_conv(const void *x, const float *conv_weight, const float *conv_bias,
                        int64_t conv_width, int64_t x_batch_stride, const void *delta,
                        const float *A, const void *B, const void *C, const float *D,
                        const void *z, int64_t z_batch_stride, const float *delta_bias,
                        const float *h0, void *out, float *last_state, void *u_out,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                        int act_dtype, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * Splitting one sequence across GPUs.  The recurrence is affine in the state
 * and its decays are diagonal, so a shard of timesteps maps an initial state
 * h to exp(A * S) (.) h + h_local, where S is the shard's sum of delta
 * (after bias and softplus) per (batch, channel) and h_local its final state
 * from a zero start (the recurrent form of "Mamba SSM concept and
 * implementation in Keras and TensorFlow", unrolled over the shard).  Rank r
 * scans its shard from zero (mamba_scan_fwd with last_state -> h_local),
 * sums delta (mamba_delta_sum -> S), exchanges (S, h_local) with the other
 * ranks, folds the summaries of ranks 0 .. r-1 into its true initial state
 * (mamba_state_fold) and scans its shard again from it (mamba_scan_fwd_init).
 *
 * mamba_delta_sum -- S[b, d] = sum_t softplus(delta[b, d, t] + delta_bias[d])
 * (without softplus when delta_softplus is 0), accumulated in fp64.
 *   delta        : act (batch, dim, seqlen); delta_bias: fp32 (dim) or NULL.
 *   out          : fp64 (batch, dim), written.
 */
int mamba_delta_sum(const void *delta, const float *delta_bias, int delta_softplus,
                    double *out, int64_t batch, int64_t dim, int64_t seqlen, int act_dtype,
                    cudaStream_t stream);

/*
 * mamba_state_fold -- h_out = the state after `count` shards starting from
 * h_init (NULL: zeros): for k = 0 .. count - 1,
 *   h <- exp(A[d, n] * delta_sums[k][b, d]) * h + h_local[k][b, d, n]
 * evaluated in fp64, rounded to fp32 once.
 *   h_init       : fp32 (batch, dim, dstate) or NULL.
 *   delta_sums   : fp64 (count, batch, dim); h_local: fp32 (count, batch, dim, dstate).
 *   A            : fp32 (dim, dstate).
 *   h_out        : fp32 (batch, dim, dstate), written; may be h_init or one of
 *                  the h_local slices exactly.
 * count may be 0 (h_out = h_init, or zeros).
 */
int mamba_state_fold(const float *h_init, const double *delta_sums, const float *A,
                     const float *h_local, float *h_out, int64_t batch, int64_t dim,
                     int64_t dstate, int64_t count, cudaStream_t stream);

/* The device-side status of this process's work on the current device:
 * synchronises `stream`, then returns MAMBA_ERR_CUDA if the stream or the
 * context reports an error; MAMBA_ERR_TIMEOUT if a local-schedule launch
 * (no workspace) on this device gave up a bounded wait since the previous
 * call (a device word the library keeps; reading it clears it), or if the
 * last persistent launch on this device (any entry point that was given a
 * workspace) gave up one -- the error word in its workspace, which must
 * still be allocated; in the bounds-checked build, MAMBA_ERR_BOUNDS (checked
 * first) if an instrumented kernel skipped an access outside its tensor
 * since the previous call (reading clears the record); else MAMBA_OK.  No
 * device code traps; this and mamba_scan_workspace_status are how failures
 * surface. */
int mamba_get_device_status(cudaStream_t stream);

/* Test hook for the failure-detection path: from the next launch on, the
 * persistent lane-split kernel's pieces of channel group `group` no longer
 * publish their carried state, so the piece after them waits until its time
 * limit (2 s) runs out, raises the workspace's error word and stops, and the
 * other pieces of the group stop on the error word; every other group
 * completes.  mamba_scan_workspace_status then reports MAMBA_ERR_TIMEOUT.
 * No wait is unbounded and nothing faults.  group < 0 turns the hook off
 * (the default).  Process-wide; returns the previous setting. */
int mamba_debug_stall_group(int group);

/*
 * The bounds-checked build (libmamba_scan_checked.so, compiled with
 * MSCAN_BOUNDS_CHECK; same entry points and results).  Every launch of the
 * lane-split scan kernel (mamba_scan_fwd, _ws, _noalloc, _init, _conv,
 * _ckpt, the (batch, L, dim) layout of mamba_scan_fwd_strided,
 * mamba_scan_state), of the
 * one-lane scan kernel (lanes_per_channel = 1 with a workspace), of the static
 * scan kernel (any layout of mamba_scan_fwd_strided, small problems of
 * mamba_scan_fwd), of the complex mode, of the backward (mamba_scan_bwd,
 * _init, _ckpt), of the decode step (mamba_state_update) and of the conv1d
 * kernels (mamba_conv1d_fwd, mamba_conv1d_update) carries the byte range of
 * every pointer argument and workspace part,
 * computed from the sizes given; each global access first checks that it
 * stays inside its range.  One that would not is skipped (a load reads
 * zeros, a store is dropped) and the first such access is recorded: its site
 * (the tensor: 1 A, 2 delta_bias, 3 D, 4 conv weight, 5 conv bias, 6 u / x,
 * 7 delta, 8 z, 9 B, 10 C, 11 conv input before a piece, 12 u written by the
 * fused conv, 13 out, 14 last_state, 15 h0, 16 checkpoints, 17 workspace
 * carries, 18 decode state, 19 conv1d input, 20 conv1d state; the backward
 * reports dout and du / ddelta / dz as 13, dlast as 14, dA / dD / dbias as
 * 1 / 3 / 2, dB / dC as 9 / 10 and its workspace parts as 16 and 17) and its
 * byte offset from the tensor's start.  Nothing traps.  In the normal build
 * the checks compile away.
 *
 * mamba_bounds_checked: 1 in the bounds-checked build, 0 otherwise.
 * mamba_debug_bounds_status: 1 with the first recorded violation (site and
 *   offset written when the pointers are not NULL), 0 without; clears the
 *   record.  Does not synchronise: call after the work has completed.
 *   MAMBA_ERR_CUDA if the record cannot be read.
 * mamba_debug_shrink_output_extent: test hook -- every later launch records
 *   its output range `bytes` short of the real one, so that the checks have a
 *   violation to find while every access still lands in allocated memory.
 *   Process-wide; 0 (the default) turns it off; returns the previous value.
 */
int mamba_bounds_checked(void);
int mamba_debug_bounds_status(int *site, long long *offset);
int mamba_debug_shrink_output_extent(int bytes);

/* Synchronises `stream`, then reads the status a persistent launch left in
 * `workspace`: MAMBA_OK, or MAMBA_ERR_TIMEOUT if a worker stopped waiting for
 * a predecessor chunk (the outputs of that launch are then incomplete).
 * This is the only entry point that synchronises. */
int mamba_scan_workspace_status(const void *workspace, cudaStream_t stream);

/*
 * mamba_scan_fwd_noalloc -- mamba_scan_fwd for callers that cannot allocate
 * device memory.  (No counterpart in the paper: this is an interface
 * convenience, not part of the method.)
 *
 * Some callers have no way to obtain a device workspace to hand over: a
 * plugin or foreign-language host that links only this library and is given
 * just its input and output buffers, or a process whose device memory is
 * owned by a pooling allocator that must not see extra cudaMalloc calls.
 * For them this entry point runs the same computation as mamba_scan_fwd_ws
 * (same arguments and results as mamba_scan_fwd) using a 4 MiB scratch area
 * built into the library instead of a caller workspace, and calls no
 * cudaMalloc, cudaFree or other allocating routine.  The caller still
 * provides every input and output.
 *
 * - The 4 MiB area is reserved on a device when the library's device code
 *   is loaded there, and held until the process exits.  With lazily loaded
 *   modules (CUDA_MODULE_LOADING=LAZY, the CUDA default) that happens at the
 *   first call on each device, which can then fail with MAMBA_ERR_CUDA if
 *   the device is out of memory: make the first call early, and before any
 *   stream capture begins.
 * - Problems whose workspace (mamba_scan_workspace_size) exceeds 4 MiB are
 *   rejected with MAMBA_ERR_WORKSPACE before anything is enqueued; that is
 *   about 2,000 groups of 32 channels (batch * ceil(dim / 32)) at moderate
 *   lengths.
 * - Every call looks the area's device address up in the current context
 *   (cudaGetSymbolAddress); nothing is cached between calls.
 * - All calls share the one area and each launch re-initialises the part
 *   that must start at zero; calls whose GPU work can overlap (other streams,
 *   other host threads) race on it and must be serialised by the caller.
 */
int mamba_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                           const void *B, const void *C, const float *D,
                           const void *z, const float *delta_bias,
                           int delta_softplus, void *out, float *last_state,
                           int64_t batch, int64_t dim, int64_t seqlen,
                           int64_t dstate, int act_dtype, cudaStream_t stream);

/*
 * mamba_state_update -- one recurrent step (one token) for every channel,
 * with the state held in HBM and updated in place: the decoding form used by
 * generation, one token per call (mamba-jax sample.py; the generation
 * benchmark of the state-spaces README).
 *
 *   state        : fp32 (batch, dim, dstate), read and overwritten.
 *   u, delta, z  : act (batch, dim); z may be NULL.
 *   A            : fp32 (dim, dstate).
 *   B, C         : act (batch, dstate).
 *   D, delta_bias: fp32 (dim) or NULL.
 *   out          : act (batch, dim), written.
 *
 * One call equals one iteration of mamba_scan_fwd's time loop.
 * Returns MAMBA_OK or a mamba_status_t error.
 */
int mamba_state_update(float *state, const void *u, const void *delta,
                       const float *A, const void *B, const void *C,
                       const float *D, const void *z, const float *delta_bias,
                       int delta_softplus, void *out, int64_t batch,
                       int64_t dim, int64_t dstate, int act_dtype,
                       cudaStream_t stream);

/*
 * mamba_scan_bwd -- gradients of mamba_scan_fwd with respect to every input,
 * for a loss L given dL/dout and optionally dL/dlast_state: reverse-mode
 * differentiation of the recurrence ("Mamba SSM concept and implementation
 * in Keras and TensorFlow", recurrent form, differentiated through the whole
 * sequence for training; recomputing the states in the backward pass, as the
 * Mamba paper's hardware-aware algorithm does, Section 3.3).  With
 * g = dL/dh_t carried backwards from dlast:
 *   dy = dout silu(z), dz = dout y silu'(z), dD += dy u, du = dy D,
 *   dC[n,t] += dy h_t[n], g[n] += dy C[n,t],
 *   ddelta += g[n] (h_{t-1}[n] Abar A[n] + B[n,t] u), dA[n] += g[n] h_{t-1}[n] Abar delta,
 *   dB[n,t] += g[n] delta u, du += g[n] delta B[n,t], g[n] *= Abar,
 *   ddelta_raw = ddelta sigmoid(delta_raw + bias) with softplus, dbias += ddelta_raw.
 *
 *   inputs       : exactly those of mamba_scan_fwd (same layouts and dtypes).
 *   dout         : act (batch, dim, seqlen).
 *   dlast_state  : fp32 (batch, dim, dstate) or NULL (no loss on the final state).
 *   du, ddelta   : act (batch, dim, seqlen), written.
 *   dz           : act (batch, dim, seqlen), written; required iff z is given.
 *   dA           : fp32 (dim, dstate); dB, dC: fp32 (batch, dstate, seqlen);
 *   dD, ddelta_bias : fp32 (dim) or NULL -- written (sums over batch rows,
 *                  channels and time).
 *   workspace    : at least mamba_scan_bwd_workspace_size bytes, 16-byte
 *                  aligned, caller-owned (the states every 32 timesteps
 *                  unless given, every 4th within a 32-step piece, and eight
 *                  partial copies of dB and dC).
 *
 * The states every 32 timesteps come from a first sweep over the inputs;
 * mamba_scan_bwd_ckpt takes them from the forward instead.  dstate <= 16.
 * dA, dB, dC, dD and ddelta_bias add partial sums with floating-point
 * atomics, so they may differ in the last bits between runs; du, ddelta and
 * dz do not.  Returns MAMBA_OK or a mamba_status_t error.
 */
int mamba_scan_bwd(const void *u, const void *delta, const float *A,
                   const void *B, const void *C, const float *D,
                   const void *z, const float *delta_bias, int delta_softplus,
                   const void *dout, const float *dlast_state,
                   void *du, void *ddelta, float *dA, float *dB, float *dC,
                   float *dD, void *dz, float *ddelta_bias,
                   int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                   int act_dtype, void *workspace, size_t workspace_bytes,
                   cudaStream_t stream);

/*
 * mamba_scan_bwd_init -- mamba_scan_bwd for a forward that started from the
 * state h0 (mamba_scan_fwd_init), which also returns the gradient with
 * respect to that state: dh0 = dL/dh_{-1}, the carried g after timestep 0
 * (g times that step's Abar).
 *
 *   h0           : fp32 (batch, dim, dstate), required; read only.
 *   dh0          : fp32 (batch, dim, dstate), written, or NULL; must not
 *                  overlap any other argument.
 *
 * All other arguments, results and errors as mamba_scan_bwd.
 */
int mamba_scan_bwd_init(const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, const void *dout,
                        const float *dlast_state, void *du, void *ddelta,
                        float *dA, float *dB, float *dC, float *dD, void *dz,
                        float *ddelta_bias, float *dh0, int64_t batch,
                        int64_t dim, int64_t seqlen, int64_t dstate,
                        int act_dtype, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* Bytes of workspace mamba_scan_bwd needs for these sizes (0 when dstate > 16
 * or the sizes are invalid).  Pure host arithmetic. */
size_t mamba_scan_bwd_workspace_size(int64_t batch, int64_t dim, int64_t seqlen,
                                     int64_t dstate);

/* Bytes of the checkpoints mamba_scan_fwd_ckpt writes and mamba_scan_bwd_ckpt
 * reads: the fp32 state entering every 32nd timestep, laid out [batch *
 * ceil(dim / 32)][ceil(seqlen / 32)][32 channels][16 states] (0 for invalid
 * sizes or dstate > 16).  Pure host arithmetic. */
size_t mamba_scan_ckpt_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate);

/*
 * mamba_scan_fwd_ckpt -- mamba_scan_fwd (from the state h0, or zeros when h0
 * is NULL) that also writes the checkpoints the backward pass recomputes
 * from (the Mamba paper's recomputation, Section 3.3: the forward keeps a
 * state every 32 steps, the backward recomputes the rest), so that
 * mamba_scan_bwd_ckpt needs no sweep of its own.
 *
 *   ckpt, ckpt_bytes : at least mamba_scan_ckpt_size bytes, 16-byte aligned,
 *                  written; must not overlap any other argument.
 *   all other arguments as mamba_scan_fwd_init (h0 may be NULL).
 *
 * Runs the local schedule of mamba_scan_fwd (no workspace); needs dstate <=
 * 16, 16-byte-aligned act tensors and seqlen a multiple of the 16-byte
 * vector width, else MAMBA_ERR_UNSUPPORTED.
 */
int mamba_scan_fwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, void *out, float *last_state,
                        float *ckpt, size_t ckpt_bytes, int64_t batch, int64_t dim,
                        int64_t seqlen, int64_t dstate, int act_dtype, cudaStream_t stream);

/*
 * mamba_scan_bwd_ckpt -- mamba_scan_bwd_init (h0 may be NULL: zeros) with
 * the states every 32 steps read from `ckpt`, as mamba_scan_fwd_ckpt wrote
 * them for the same inputs and h0, instead of a sweep over the inputs.
 *
 *   ckpt         : mamba_scan_ckpt_size bytes, 16-byte aligned, read only.
 *   dh0          : written when h0 is given (may be NULL), must be NULL
 *                  otherwise.
 *   all other arguments, results and errors as mamba_scan_bwd_init.
 */
int mamba_scan_bwd_ckpt(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, const float *ckpt, const void *dout,
                        const float *dlast_state, void *du, void *ddelta, float *dA, float *dB,
                        float *dC, float *dD, void *dz, float *ddelta_bias, float *dh0,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * mamba_conv1d_fwd -- the step that produces the scan's input u: a causal
 * depthwise convolution over time with a bias, then silu ("Mamba SSM concept
 * and implementation in Keras and TensorFlow", MambaBlock: a Conv1D with one
 * group per channel, channels-first, causal padding and a bias, cut to the
 * input length, then swish).  With K = width:
 *
 *   v[b,d,t]   = bias[d] + sum_{k=0}^{K-1} weight[d,k] * x[b,d,t-(K-1)+k],
 *                x[b,d,t] = 0 for t < 0
 *   out[b,d,t] = silu(v) if apply_silu, else v
 *
 *   x            : act; channel d of batch row b is the seqlen-long row at
 *                  x + b * x_batch_stride + d * seqlen (elements).
 *                  x_batch_stride = 0 means dim * seqlen (contiguous); a
 *                  larger stride takes x as the first dim channel rows of a
 *                  wider tensor, such as the x half of the input
 *                  projection's (batch, 2 dim, seqlen) output.
 *   weight       : fp32 (dim, width), width 1 .. 4.
 *   bias         : fp32 (dim) or NULL.
 *   out          : act (batch, dim, seqlen), contiguous, written; must not
 *                  overlap x.
 *
 * 16-byte-aligned x / out with seqlen and x_batch_stride multiples of 8
 * (bf16) or 4 (fp32) take the vector path; anything else a scalar one.
 * Returns MAMBA_OK or a mamba_status_t error (MAMBA_ERR_UNSUPPORTED for a
 * width outside 1 .. 4, MAMBA_ERR_SHAPE for a stride below dim * seqlen).
 */
int mamba_conv1d_fwd(const void *x, const float *weight, const float *bias,
                     int apply_silu, void *out, int64_t batch, int64_t dim,
                     int64_t seqlen, int64_t width, int64_t x_batch_stride,
                     int act_dtype, cudaStream_t stream);

/*
 * mamba_conv1d_update -- one token of mamba_conv1d_fwd, for decoding.
 *
 *   conv_state   : fp32 (batch, dim, width - 1): each row's last width - 1
 *                  inputs, oldest first (zeros before the sequence starts);
 *                  read, then shifted by one with the token's input
 *                  appended.  Unused (may be NULL) when width is 1.
 *   x            : act (batch, dim); row b at x + b * x_batch_stride
 *                  (0 means dim).
 *   weight, bias : as for mamba_conv1d_fwd.
 *   out          : act (batch, dim), written; must not overlap x or the state.
 *
 * A run of calls from a zero state equals mamba_conv1d_fwd over the tokens.
 * Returns MAMBA_OK or a mamba_status_t error.
 */
int mamba_conv1d_update(float *conv_state, const void *x, const float *weight,
                        const float *bias, int apply_silu, void *out,
                        int64_t batch, int64_t dim, int64_t width,
                        int64_t x_batch_stride, int act_dtype,
                        cudaStream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *mamba_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
int mamba_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_SCAN_H */
