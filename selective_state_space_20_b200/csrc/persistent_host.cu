// persistent_host.cu -- planning for the persistent scan kernels: which
// variant (one lane or two lanes per channel), chunk length, workspace
// layout, grid size.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "persistent_kernels.h"

namespace mscan {

namespace {

int group_channels(int lanes) { return 32 / lanes; }
int states_per_lane(int lanes) { return persist::kNS / lanes; }
int sub_chunk(int lanes, int act) {
    return lanes == 1 ? persistent_spec_sub_chunk() : persistent_split_sub_chunk(lanes, act);
}
int blocks_per_sm(int lanes) {
    // blocks of kWarps workers; the one-lane kernel runs one block of kWarps pairs
    return lanes == 1 ? persistent_spec_pairs_per_sm() / persist::kWarps : persistent_split_blocks_per_sm(lanes);
}
int64_t n_groups(int64_t batch, int64_t dim, int lanes) {
    const int cw = group_channels(lanes);
    return batch * ((dim + cw - 1) / cw);
}

// Timesteps per work unit: about 4 units per worker (measured best on B200
// for the Mamba layer shapes: shorter units pay more per-unit costs -- pop,
// carry, pipeline ramp -- longer ones leave a longer drain at the end), and
// never fewer than 4 sub-chunks per unit.
int chunk_len(int64_t groups, int64_t seqlen, int workers, int tc) {
    const int64_t max_chunks = (seqlen + tc - 1) / tc;
    int64_t want = (4LL * workers + groups - 1) / groups;
    int64_t lim = (max_chunks + 3) / 4;
    if (lim < 1) lim = 1;
    if (want > lim) want = lim;
    if (want < 1) want = 1;
    int64_t tu = (seqlen + want - 1) / want;
    tu = (tu + tc - 1) / tc * tc;
    return (int)tu;
}

struct Layout {
    int64_t groups, chunks;
    size_t queue_off, carry_off, bytes;
};

Layout layout(int64_t batch, int64_t dim, int64_t seqlen, int lanes, int tu) {
    Layout l;
    l.groups = n_groups(batch, dim, lanes);
    l.chunks = (seqlen + tu - 1) / tu;
    const int64_t queue = l.groups * (l.chunks - 1);
    l.queue_off = 16;
    l.carry_off = 16 + (size_t)((queue * 4 + 255) / 256 * 256);
    l.bytes = l.carry_off + (size_t)(l.groups * 32 * states_per_lane(lanes)) * 4;
    return l;
}

// Balanced split (lanes 2 and 4): header, one progress word per group, one
// carried state per group.  Independent of the device.
Layout balanced_layout(int64_t batch, int64_t dim, int lanes) {
    Layout l;
    l.groups = n_groups(batch, dim, lanes);
    l.chunks = 1;
    l.queue_off = 16;  // progress words
    l.carry_off = 16 + (size_t)((l.groups * 4 + 255) / 256 * 256);
    l.bytes = l.carry_off + (size_t)(l.groups * 32 * states_per_lane(lanes)) * 4;
    return l;
}

// Largest workspace any device can need.  Queue schedule (one lane): the
// smallest unit (4 sub-chunks).
size_t bound_for(int64_t batch, int64_t dim, int64_t seqlen, int lanes, int act) {
    if (lanes != 1) return balanced_layout(batch, dim, lanes).bytes;
    const int tc = sub_chunk(lanes, act);
    const int64_t max_chunks = ((seqlen + tc - 1) / tc + 3) / 4;
    int64_t tu = (seqlen + max_chunks - 1) / max_chunks;
    tu = (tu + tc - 1) / tc * tc;
    return layout(batch, dim, seqlen, lanes, (int)tu).bytes;
}

}  // namespace

namespace {
int g_stall_group = -1;  // test hook (mamba_debug_stall_group)
}  // namespace

int g_out_extent_shrink = 0;  // test hook (mamba_debug_shrink_output_extent)

int set_stall_group(int group) {
    const int prev = g_stall_group;
    g_stall_group = group;
    return prev;
}

// The channel-last form of the block-local kernel: every 16-byte copy of a
// timestep's channels or states must be whole (dim and N multiples of 16
// bytes of the activation type) and start aligned.
bool channels_last_supported(const ScanArgs &a) {
    if (a.dstate > persist::kNS) return false;
    const int es = a.act == kBF16 ? 2 : 4;
    if ((a.dim * es) % 16 != 0 || (a.dstate * es) % 16 != 0) return false;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    if (!(al(a.u) && al(a.delta) && al(a.z) && al(a.B) && al(a.C) && al(a.out))) return false;
    const int64_t units = n_groups(a.batch, a.dim, 4) * ((a.seqlen + 15) / 16);
    return units < ((int64_t)1 << 30);
}

bool persistent_supported(const ScanArgs &a) {
    if (a.dstate > persist::kNS) return false;
    const int es = a.act == kBF16 ? 2 : 4;
    if (a.seqlen % (16 / es) != 0) return false;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    if (!(al(a.u) && al(a.delta) && al(a.z) && al(a.B) && al(a.C) && al(a.out))) return false;
    const int64_t units = n_groups(a.batch, a.dim, 4) * ((a.seqlen + 15) / 16);
    return units < ((int64_t)1 << 30);
}

// Preferred lanes per channel, or 0 when the static schedule should run.
// Measured on B200 (Mamba layer shapes, N = 16): two lanes per channel is
// fastest when its channel groups give every worker (2 blocks x 4 warps per
// SM) a chain of its own, minus 10 %; with fewer groups, four lanes (3 blocks
// per SM) as long as three quarters of its workers are busy.  With fewer
// groups still, long sequences (at least 8 sub-chunks per worker) go back to
// two lanes, where the balanced split cuts each group into pieces that run
// at once (two-phase pieces; the long-context layer, 1 x 2048 x 262144:
// 6.0 ms against 7.9 ms for the static schedule).  Below that the static
// schedule, which splits states further, keeps more warps busy.  One lane
// per channel (the warp-specialised kernel) is never preferred: it measured
// slower than two lanes on every Mamba shape; it runs on request.
int persistent_choose_lanes(const ScanArgs &a, int sm_count) {
    const int64_t w2 = (int64_t)sm_count * blocks_per_sm(2) * persist::kWarps;
    const int64_t g2 = n_groups(a.batch, a.dim, 2);
    if (g2 * 10 >= w2 * 9) return 2;
    const int64_t w4 = (int64_t)sm_count * blocks_per_sm(4) * persist::kWarps;
    if (n_groups(a.batch, a.dim, 4) * 4 >= w4 * 3) return 4;
    const int tc = sub_chunk(2, a.act);
    if (g2 * ((a.seqlen + tc - 1) / tc) >= 8 * w2) return 2;
    return 0;
}

bool persistent_preferred(const ScanArgs &a, int sm_count) {
    return persistent_choose_lanes(a, sm_count) != 0;
}

size_t persistent_workspace_bound(int64_t batch, int64_t dim, int64_t seqlen, int act) {
    size_t m = 0;
    for (int lanes : {1, 2, 4}) {
        const size_t b = bound_for(batch, dim, seqlen, lanes, act);
        if (b > m) m = b;
    }
    return m;
}

namespace {
// Kernel parameters shared by both launch forms of the lane-split kernel and
// the one-lane kernel (no workspace fields).
persist::Params base_params(const ScanArgs &a, int lanes, int tc) {
    persist::Params kp = {};
    kp.u = a.u; kp.delta = a.delta; kp.B = a.B; kp.C = a.C; kp.z = a.z;
    kp.A = a.A; kp.D = a.D; kp.delta_bias = a.delta_bias;
    kp.out = a.out; kp.last_state = a.last_state; kp.h0 = a.h0;
    kp.conv_w = a.conv_w; kp.conv_b = a.conv_b; kp.conv_k = a.conv_k; kp.u_out = a.u_out;
    kp.u_bstride = a.u_bstride > 0 ? a.u_bstride : a.dim * a.seqlen;
    kp.z_bstride = a.z_bstride > 0 ? a.z_bstride : a.dim * a.seqlen;
    kp.dim = a.dim; kp.seqlen = a.seqlen; kp.dstate = a.dstate; kp.softplus = a.softplus;
    kp.group_channels = group_channels(lanes);
    kp.groups_per_batch = (int)((a.dim + kp.group_channels - 1) / kp.group_channels);
    kp.n_groups = (int)n_groups(a.batch, a.dim, lanes);
    kp.subs_per_chain = (int)((a.seqlen + tc - 1) / tc);
    kp.stall_group = g_stall_group;
    kp.ckpt = a.ckpt;
    kp.ckpt_gpb = (int)((a.dim + 31) / 32);
    kp.ckpt_nsup = (int)((a.seqlen + 31) / 32);
    kp.channels_last = a.channels_last ? 1 : 0;
    kp.state_only = a.state_only ? 1 : 0;
#ifdef MSCAN_BOUNDS_CHECK
    // byte ranges of the pointer arguments (checked in the bounds-checked build)
    const unsigned long long es = a.act == kBF16 ? 2 : 4;
    const unsigned long long x = (unsigned long long)(a.batch * a.dim * a.seqlen) * es;
    const unsigned long long bc = (unsigned long long)(a.batch * a.dstate * a.seqlen) * es;
    const unsigned long long st = (unsigned long long)(a.batch * a.dim * a.dstate) * 4;
    const unsigned long long row = (unsigned long long)(a.dim * a.seqlen) * es;
    kp.x_u = extent_of(a.u, a.conv_w ? (unsigned long long)(a.batch - 1) * kp.u_bstride * es + row : x);
    kp.x_delta = extent_of(a.delta, x);
    kp.x_z = extent_of(a.z, a.conv_w ? (unsigned long long)(a.batch - 1) * kp.z_bstride * es + row : x);
    kp.x_B = extent_of(a.B, bc);
    kp.x_C = extent_of(a.C, bc);
    kp.x_A = extent_of(a.A, (unsigned long long)(a.dim * a.dstate) * 4);
    kp.x_D = extent_of(a.D, (unsigned long long)a.dim * 4);
    kp.x_bias = extent_of(a.delta_bias, (unsigned long long)a.dim * 4);
    kp.x_out = extent_of(a.out, x > (unsigned long long)g_out_extent_shrink ? x - g_out_extent_shrink : 0);
    kp.x_last = extent_of(a.last_state, st);
    kp.x_h0 = extent_of(a.h0, st);
    kp.x_conv_w = extent_of(a.conv_w, (unsigned long long)(a.dim * a.conv_k) * 4);
    kp.x_conv_b = extent_of(a.conv_b, (unsigned long long)a.dim * 4);
    kp.x_u_out = extent_of(a.u_out, x);
    kp.x_ckpt = extent_of(a.ckpt, (unsigned long long)a.batch * kp.ckpt_gpb * kp.ckpt_nsup * 32 * 16 * 4);
    kp.x_carry = extent_of(nullptr, 0);
#endif
    return kp;
}
}  // namespace

// Block-local form.  Each of the min(SMs, groups) blocks takes whole groups,
// so the slowest block holds ceil(groups / blocks) of them for its W warps.
// Measured on B200 (Mamba layer shapes, N = 16): two lanes per channel when
// those groups give every warp about one group or more (Mamba-2.8B: 9 groups
// for 8 warps, 524 us); else four lanes (8-channel groups, 12 warps per
// block) when they keep three quarters of the warps busy (Mamba-130M: 11
// groups for 12 warps, 205 us against 240 us with two lanes); else, on rows
// long enough for the two-phase pieces (>= 8 sub-chunks per warp), two lanes
// again (long context: 6.35 ms against 7.38 ms with four); else the static
// schedule, which splits states further.
int local_choose_lanes(const ScanArgs &a, int sm_count) {
    const int64_t g2 = n_groups(a.batch, a.dim, 2), g4 = n_groups(a.batch, a.dim, 4);
    const int64_t w2 = local_split_warps(2), w4 = local_split_warps(4);
    const int64_t b2 = g2 < sm_count ? g2 : sm_count, b4 = g4 < sm_count ? g4 : sm_count;
    const int64_t per2 = (g2 + b2 - 1) / b2, per4 = (g4 + b4 - 1) / b4;  // groups of the busiest block
    if (per2 * 10 >= w2 * 9) return 2;
    if (per4 * 4 >= w4 * 3) return 4;
    const int tc = sub_chunk(2, a.act);
    if (g2 * ((a.seqlen + tc - 1) / tc) >= 8 * w2 * b2) return 2;
    return 0;
}

// The final state alone runs on the dense layout without the fused conv1d or
// checkpoints.
static bool state_only_ok(const ScanArgs &a) {
    return !a.state_only || (!a.conv_w && !a.ckpt && !a.channels_last);
}

cudaError_t launch_scan_fwd_local(const ScanArgs &a, int lanes, int sm_count, cudaStream_t st) {
    if (lanes != 2 && lanes != 4) return cudaErrorInvalidValue;
    if (a.conv_w && !a.softplus) return cudaErrorInvalidValue;
    if (!state_only_ok(a)) return cudaErrorInvalidValue;
    persist::Params kp = base_params(a, lanes, sub_chunk(lanes, a.act));
    kp.n_chunks = 1;
    kp.chunk_len = (int)a.seqlen;
    kp.hdr = nullptr; kp.queue = nullptr; kp.progress = nullptr; kp.carry = nullptr;
    return launch_local_split(kp, lanes, a.act, sm_count, st);
}

int local_error_take() {
    unsigned v = 0;
    if (take_local_error(&v) != 0) return -1;
    return v != 0 ? 1 : 0;
}

cudaError_t launch_scan_fwd_persistent(const ScanArgs &a, int lanes, int chunk_timesteps,
                                       void *workspace, size_t ws_bytes, int sm_count,
                                       cudaStream_t st) {
    if (lanes == 0) lanes = persistent_choose_lanes(a, sm_count);
    if (lanes == 0) lanes = 1;
    if (lanes != 1 && lanes != 2 && lanes != 4) return cudaErrorInvalidValue;
    const int per_sm = blocks_per_sm(lanes);
    const int64_t workers = (int64_t)sm_count * per_sm * persist::kWarps;
    const int64_t groups = n_groups(a.batch, a.dim, lanes);
    const int tc = sub_chunk(lanes, a.act);

    if (a.conv_w && (lanes == 1 || !a.softplus)) return cudaErrorInvalidValue;  // lane-split kernel, softplus on
    if (a.state_only && (lanes == 1 || !state_only_ok(a))) return cudaErrorInvalidValue;
    persist::Params kp = base_params(a, lanes, tc);
    unsigned char *w = static_cast<unsigned char *>(workspace);
    kp.hdr = reinterpret_cast<unsigned *>(w);

    if (lanes != 1) {
        // balanced split over every resident worker; chunk_timesteps does not apply
        const Layout l = balanced_layout(a.batch, a.dim, lanes);
        if (ws_bytes < l.bytes) return cudaErrorInvalidValue;
        kp.n_chunks = 1;
        kp.chunk_len = (int)a.seqlen;
        kp.queue = nullptr;
        kp.progress = reinterpret_cast<unsigned *>(w + l.queue_off);
        kp.carry = reinterpret_cast<float *>(w + l.carry_off);
#ifdef MSCAN_BOUNDS_CHECK
        kp.x_carry = extent_of(kp.carry, l.bytes - l.carry_off);
#endif
        cudaError_t e = cudaMemsetAsync(w, 0, l.queue_off + (size_t)groups * 4, st);
        if (e != cudaSuccess) return e;
        return launch_persistent_split(kp, lanes, a.act, sm_count, st);
    }

    int tu = chunk_len(groups, a.seqlen, (int)workers, tc);
    if (chunk_timesteps > 0) {
        // explicit unit length, but never shorter than the bound's units
        // (4 sub-chunks or the whole sequence)
        int64_t want = ((int64_t)chunk_timesteps + tc - 1) / tc * tc;
        const int64_t min_tu = 4LL * tc < a.seqlen ? 4LL * tc : (a.seqlen + tc - 1) / tc * tc;
        if (want < min_tu) want = min_tu;
        if (want > a.seqlen) want = (a.seqlen + tc - 1) / tc * tc;
        tu = (int)want;
    }
    const Layout l = layout(a.batch, a.dim, a.seqlen, lanes, tu);
    if (ws_bytes < l.bytes) return cudaErrorInvalidValue;
    kp.n_chunks = (int)l.chunks;
    kp.chunk_len = tu;
    kp.queue = reinterpret_cast<unsigned *>(w + l.queue_off);
    kp.progress = nullptr;
    kp.carry = reinterpret_cast<float *>(w + l.carry_off);
#ifdef MSCAN_BOUNDS_CHECK
    kp.x_carry = extent_of(kp.carry, l.bytes - l.carry_off);
#endif
    // counters and queue entries start at zero; carries are written before read
    cudaError_t e = cudaMemsetAsync(w, 0, l.queue_off + (size_t)(l.groups * (l.chunks - 1)) * 4, st);
    if (e != cudaSuccess) return e;

    const int64_t units = l.groups * l.chunks;
    int64_t grid = (int64_t)sm_count * per_sm;
    const int64_t need = (units + persist::kWarps - 1) / persist::kWarps;
    if (grid > need) grid = need;
    return launch_persistent_spec(kp, a.act, (int)grid, st);
}

}  // namespace mscan
