// internal.h -- declarations shared by the C-ABI layer and the kernel files.
// Not part of the public interface (that is include/mamba_scan.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mscan {

enum ActType : int { kF32 = 0, kBF16 = 1 };

// Test hook of the bounds-checked build: the output extent every launch
// records is this many bytes short of the real one (0 in normal use).
extern int g_out_extent_shrink;

// The bounds-checked build's record of each instrumented translation unit
// (1: a violation, its site and byte offset; cleared), 0 without one, -1 on
// a read error.  Always 0 in the normal build.
int pairs_bounds_take(int *site, long long *off);
int spec_bounds_take(int *site, long long *off);
int static_bounds_take(int *site, long long *off);
int complex_bounds_take(int *site, long long *off);
int bwd_bounds_take(int *site, long long *off);
int state_update_bounds_take(int *site, long long *off);
int conv1d_bounds_take(int *site, long long *off);

// Element strides of one (batch, channel or state, time) tensor.
struct Stride3 {
    int64_t b, d, t;
};
// Strides of every sequence tensor of a scan; u, delta, z, out are (batch,
// channel, time) and B, C (batch, state, time).
struct ScanStrides {
    Stride3 u, delta, z, out, B, C;
};

struct ScanArgs {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    float *last_state;
    const float *h0;  // initial state (batch, dim, dstate) or null (zeros)
    const ScanStrides *strides;  // null: dense (batch, dim, L) / (batch, N, L), L contiguous
    // fused causal conv1d prologue (persistent lane-split kernel only): when
    // conv_w is set, u holds x, the conv input, and the kernel forms
    // u = silu(conv_b + sum_k conv_w[k] x[t - (conv_k - 1) + k]) itself
    const float *conv_w = nullptr;  // (dim, conv_k), conv_k <= 4
    const float *conv_b = nullptr;  // (dim) or null
    int conv_k = 0;
    void *u_out = nullptr;          // (batch, dim, L) act or null: the u it formed
    int64_t u_bstride = 0;          // batch stride of x when conv_w is set (elements); 0: dim * L
    int64_t z_bstride = 0;          // batch stride of z when conv_w is set; 0: dim * L
    // lane-split kernel only: checkpoints for the backward pass (the state
    // entering every scan_bwd_ckpt_interval() steps, its layout) or null
    float *ckpt = nullptr;
    // lane-split block-local kernel only: u / delta / z / out dense
    // (batch, L, dim) and B / C dense (batch, L, N) -- the layout of the
    // Keras page -- instead of (batch, dim, L) / (batch, N, L)
    bool channels_last = false;
    // lane-split kernel only: the final state alone -- no C, D, z, readout,
    // gate or out (dense layout, no conv, no checkpoints)
    bool state_only = false;
    int64_t batch, dim, seqlen;
    int dstate;
    int softplus;
    int act;  // ActType
};

struct ScanPlan {
    int padded_dstate;      // dstate rounded up to 8, 16, 32 or 64
    int lanes;              // threads per channel (R)
    int threads;            // threads per block
    int channels_per_block; // threads / lanes
    int chunk;              // timesteps staged per pass
    int vectorized;         // 16-byte loads/stores usable
    int64_t blocks;
    size_t smem_bytes;
};

struct StateUpdateArgs {
    float *state;
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    int64_t batch, dim;
    int dstate;
    int softplus;
    int act;
};

// Fills `plan` for the given sizes.  lanes/threads of 0 mean automatic.
// Returns 0 if the configuration is valid, -1 otherwise.
int make_scan_plan(const ScanArgs &a, int want_lanes, int want_threads,
                   int sm_count, ScanPlan *plan);

cudaError_t launch_scan_fwd(const ScanArgs &a, const ScanPlan &plan,
                            cudaStream_t stream);

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t stream);

// Causal depthwise conv1d (+ bias, + silu) producing u; width 1 .. 4.
struct Conv1dArgs {
    const void *x;           // row (b, d) at x + b * x_batch_stride + d * seqlen
    const float *weight;     // (dim, width)
    const float *bias;       // (dim) or null
    void *out;               // (batch, dim, seqlen)
    int64_t batch, dim, seqlen, x_batch_stride;
    int width, silu, act;
};
struct Conv1dUpdateArgs {
    float *state;            // (batch, dim, width - 1), oldest input first
    const void *x;           // (batch, dim): row b at x + b * x_batch_stride
    const float *weight, *bias;
    void *out;               // (batch, dim)
    int64_t batch, dim, x_batch_stride;
    int width, silu, act;
};
// Backward of the scan (dstate <= 16): every input gradient.
struct ScanBwdArgs {
    const void *u, *delta, *B, *C, *z, *dout;
    const float *A, *D, *delta_bias, *dlast;
    const float *h0;                                 // initial state (batch, dim, N) or null (zeros)
    void *du, *ddelta, *dz;                          // act (batch, dim, L)
    float *dA, *dB, *dC, *dD, *ddelta_bias;          // fp32, accumulated from zero
    float *dh0;                                      // fp32 (batch, dim, N) or null
    int64_t batch, dim, seqlen;
    int dstate, softplus, act;
};
size_t scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen);
// Checkpoints the backward reads: the state entering every
// scan_bwd_ckpt_interval() timesteps, fp32 [batch * ceil(dim / 32)][ceil(L /
// interval)][32 channels][16 states].  ckpt == null: the backward writes them
// itself (into the workspace) in a first sweep.
int64_t scan_bwd_ckpt_floats(int64_t batch, int64_t dim, int64_t seqlen);
int scan_bwd_ckpt_interval();
cudaError_t launch_scan_bwd(const ScanBwdArgs &a, void *workspace, const float *ckpt, int sm_count,
                            cudaStream_t stream);

cudaError_t launch_conv1d_fwd(const Conv1dArgs &a, cudaStream_t stream);
cudaError_t launch_conv1d_update(const Conv1dUpdateArgs &a, cudaStream_t stream);

// Persistent, queue-balanced scan (dstate <= 16), one or two lanes per channel.
bool persistent_supported(const ScanArgs &a);
// Layout and alignment rules of the channel-last block-local kernel.
bool channels_last_supported(const ScanArgs &a);
// Test hook: the lane-split kernel's pieces of this channel group stop
// publishing their carried state, so the next piece's bounded wait runs out
// (-1 turns it off).  Returns the previous value.
int set_stall_group(int group);
bool persistent_preferred(const ScanArgs &a, int sm_count);
int persistent_choose_lanes(const ScanArgs &a, int sm_count);  // 0 = not preferred
size_t persistent_workspace_bound(int64_t batch, int64_t dim, int64_t seqlen, int act);
// Sequence split across GPUs: per-row sums of delta, and the fold of shard
// summaries into an initial state (seqpar.cu).
cudaError_t launch_delta_sum(const void *delta, const float *bias, int softplus, double *out,
                             int64_t batch, int64_t dim, int64_t seqlen, int act, cudaStream_t stream);
cudaError_t launch_state_fold(const float *h_init, const double *sums, const float *A,
                              const float *h_local, float *h_out, int64_t batch, int64_t dim,
                              int64_t dstate, int count, cudaStream_t stream);

// Complex-valued mode (dstate <= 16): A (dim, N, 2), B / C (batch, N, L, 2),
// h0 / last_state (batch, dim, N, 2); lanes 1, 2 or 4 per channel.
int complex_scan_lanes(int64_t batch, int64_t dim, int sm_count);
cudaError_t launch_scan_fwd_complex(const ScanArgs &a, int lanes, cudaStream_t stream);

cudaError_t launch_scan_fwd_persistent(const ScanArgs &a, int lanes, int chunk_timesteps,
                                       void *workspace, size_t ws_bytes, int sm_count,
                                       cudaStream_t stream);

// The lane-split kernel without a workspace: one block per SM takes whole
// channel groups and splits them among its warps (dstate <= 16, the layout
// rules of persistent_supported).  local_choose_lanes: 2 or 4, or 0 when the
// static schedule should run.  local_error_take: 1 if a block-local launch on
// the current device stopped waiting since the last call (then cleared).
int local_choose_lanes(const ScanArgs &a, int sm_count);
cudaError_t launch_scan_fwd_local(const ScanArgs &a, int lanes, int sm_count, cudaStream_t stream);
int local_error_take();

}  // namespace mscan
