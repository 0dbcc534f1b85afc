// api.cu -- the C ABI declared in include/mamba_scan.h: argument validation,
// launch planning and dispatch.  No computation happens here and nothing is
// allocated; only mamba_scan_workspace_status synchronises.
#include <cuda_runtime.h>
#include <stdint.h>

#include "mamba_scan.h"
#include "bounds.cuh"
#include "internal.h"

namespace {

constexpr int kMaxDstate = 64;
constexpr int kMaxDevices = 64;

int g_sm_count[kMaxDevices];  // 0 = not queried yet (benign races: same value)
// workspace of the last persistent launch per device (mamba_get_device_status)
const void *g_last_workspace[kMaxDevices];

void note_workspace(const void *ws) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) g_last_workspace[dev] = ws;
}

// The first recorded violation of the instrumented kernels (lane-split,
// one-lane, static and complex scans, backward, decode, conv1d), every
// record cleared:
// 1 with it, 0 without, -1 on a read error.
int take_bounds(int *site, long long *off) {
    int found = 0;
    int (*takes[])(int *, long long *) = {mscan::pairs_bounds_take, mscan::spec_bounds_take, mscan::static_bounds_take,
                                          mscan::complex_bounds_take, mscan::bwd_bounds_take,
                                          mscan::state_update_bounds_take, mscan::conv1d_bounds_take};
    for (auto take : takes) {
        int s = 0;
        long long o = 0;
        const int r = take(&s, &o);
        if (r < 0) return -1;
        if (r > 0 && !found) {
            found = 1;
            *site = s;
            *off = o;
        }
    }
    return found;
}

int current_sm_count(int *status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { *status = MAMBA_ERR_DEVICE; return 0; }
    if (dev >= 0 && dev < kMaxDevices && g_sm_count[dev] > 0) return g_sm_count[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        *status = MAMBA_ERR_DEVICE;
        return 0;
    }
    if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev] = sms;
    return sms;
}

size_t act_size(int act) { return act == MAMBA_BF16 ? 2 : 4; }

bool overlaps(const void *a, size_t abytes, const void *b, size_t bbytes) {
    if (!a || !b) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bbytes && b0 < a0 + abytes;
}

// An output may coincide exactly with one same-shaped input (in place) but
// must not otherwise overlap any input.
bool bad_alias(const void *out, size_t obytes, const void *in, size_t ibytes, bool exact_ok) {
    if (!overlaps(out, obytes, in, ibytes)) return false;
    return !(exact_ok && out == in && obytes == ibytes);
}

// Largest element count a launch may index with int64 arithmetic.
constexpr int64_t kMaxElems = (int64_t)1 << 50;

int check_sizes(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate) {
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0) return MAMBA_ERR_SHAPE;
    if (dstate > kMaxDstate) return MAMBA_ERR_UNSUPPORTED;
    if (batch > kMaxElems || dim > kMaxElems || seqlen > kMaxElems) return MAMBA_ERR_SHAPE;
    if ((double)batch * (double)dim * (double)seqlen > (double)kMaxElems) return MAMBA_ERR_SHAPE;
    if ((double)batch * (double)dstate * (double)seqlen > (double)kMaxElems) return MAMBA_ERR_SHAPE;
    return MAMBA_OK;
}

// Null and aliasing rules of a dense scan: out may replace u, delta or z in
// place; last_state may be h0 (in place); nothing else may overlap.
int check_scan_aliases(const void *u, const void *delta, const float *A, const void *B, const void *C,
                       const float *D, const void *z, const float *delta_bias, const float *h0, void *out,
                       float *last_state, int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                       int act_dtype) {
    if (!u || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim * seqlen) * es;
    const size_t nbc = (size_t)(batch * dstate * seqlen) * es;
    const size_t nA = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4;
    const size_t nls = (size_t)(batch * dim * dstate) * 4;
    if (bad_alias(out, nx, u, nx, true) || bad_alias(out, nx, delta, nx, true) ||
        bad_alias(out, nx, z, nx, true) || bad_alias(out, nx, B, nbc, false) ||
        bad_alias(out, nx, C, nbc, false) || bad_alias(out, nx, A, nA, false) ||
        bad_alias(out, nx, D, nd, false) || bad_alias(out, nx, delta_bias, nd, false))
        return MAMBA_ERR_OVERLAP;
    if (last_state &&
        (overlaps(last_state, nls, u, nx) || overlaps(last_state, nls, delta, nx) ||
         overlaps(last_state, nls, z, nx) || overlaps(last_state, nls, B, nbc) ||
         overlaps(last_state, nls, C, nbc) || overlaps(last_state, nls, A, nA) ||
         overlaps(last_state, nls, D, nd) || overlaps(last_state, nls, delta_bias, nd) ||
         overlaps(last_state, nls, out, nx)))
        return MAMBA_ERR_OVERLAP;
    if (h0 && (overlaps(h0, nls, out, nx) || bad_alias(last_state, nls, h0, nls, true)))
        return MAMBA_ERR_OVERLAP;
    return MAMBA_OK;
}

int scan_impl(const void *u, const void *delta, const float *A, const void *B, const void *C,
              const float *D, const void *z, const float *delta_bias, int delta_softplus,
              const float *h0, void *out, float *last_state, int64_t batch, int64_t dim, int64_t seqlen,
              int64_t dstate, int act_dtype, const mamba_scan_tuning_t *tuning,
              void *workspace, size_t ws_bytes, cudaStream_t stream, bool launch,
              mamba_scan_tuning_t *plan_out, bool plan_noworkspace = false) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (launch) {
        rc = check_scan_aliases(u, delta, A, B, C, D, z, delta_bias, h0, out, last_state, batch, dim, seqlen,
                                dstate, act_dtype);
        if (rc != MAMBA_OK) return rc;
        const size_t es = act_size(act_dtype);
        const size_t nx = (size_t)(batch * dim * seqlen) * es;
        const size_t nbc = (size_t)(batch * dstate * seqlen) * es;
        const size_t nA = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4;
        const size_t nls = (size_t)(batch * dim * dstate) * 4;
        if (workspace) {
            if ((reinterpret_cast<uintptr_t>(workspace) & 15) != 0) return MAMBA_ERR_WORKSPACE;
            const void *ins[] = {u, delta, z, B, C, A, D, delta_bias, out, last_state, h0};
            const size_t sz[] = {nx, nx, nx, nbc, nbc, nA, nd, nd, nx, nls, nls};
            for (int i = 0; i < 11; ++i)
                if (overlaps(workspace, ws_bytes, ins[i], sz[i])) return MAMBA_ERR_OVERLAP;
        }
    }
    int want_lanes = 0, want_threads = 0, want_sched = MAMBA_SCHEDULE_AUTO, want_chunk = 0;
    if (tuning) {
        want_lanes = tuning->lanes_per_channel;
        want_threads = tuning->threads_per_block;
        want_sched = tuning->schedule;
        want_chunk = tuning->chunk_timesteps;
        if (want_chunk < 0) return MAMBA_ERR_UNSUPPORTED;
        if (want_lanes != 0 && want_lanes != 1 && want_lanes != 2 && want_lanes != 4 &&
            want_lanes != 8 && want_lanes != 16)
            return MAMBA_ERR_UNSUPPORTED;
        if (want_threads != 0 && want_threads != 128 && want_threads != 256)
            return MAMBA_ERR_UNSUPPORTED;
        if (want_sched < MAMBA_SCHEDULE_AUTO || want_sched > MAMBA_SCHEDULE_LOCAL)
            return MAMBA_ERR_UNSUPPORTED;
    }
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;

    mscan::ScanArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out; a.last_state = last_state; a.h0 = h0;
    a.strides = nullptr;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;

    // Persistent schedule: needs a workspace (when launching), dstate <= 16,
    // aligned tensors and enough channel groups to occupy every worker.  The
    // local schedule (same kernel, no workspace) needs the same layout; it
    // runs when no workspace is given.
    const bool ws_ok = (!launch && !plan_noworkspace) || (workspace != nullptr &&
                                   ws_bytes >= mscan::persistent_workspace_bound(
                                                   batch, dim, seqlen, act_dtype));
    const bool supported = mscan::persistent_supported(a);
    int local_lanes = 0;
    if (want_sched == MAMBA_SCHEDULE_LOCAL) {
        if (!supported || want_threads != 0 || (want_lanes != 0 && want_lanes != 2 && want_lanes != 4))
            return MAMBA_ERR_UNSUPPORTED;
        local_lanes = want_lanes != 0 ? want_lanes : mscan::local_choose_lanes(a, sms);
        if (local_lanes == 0) local_lanes = 2;
    } else if (want_sched == MAMBA_SCHEDULE_AUTO && want_lanes == 0 && want_threads == 0 &&
               (launch || plan_noworkspace) && workspace == nullptr && supported) {
        local_lanes = mscan::local_choose_lanes(a, sms);
    }
    if (local_lanes != 0) {
        if (plan_out) {
            plan_out->lanes_per_channel = local_lanes;
            plan_out->threads_per_block = 32 * (local_lanes == 4 ? 12 : 8);
            plan_out->schedule = MAMBA_SCHEDULE_LOCAL;
            plan_out->chunk_timesteps = 0;
        }
        if (!launch) return MAMBA_OK;
        note_workspace(nullptr);
        return mscan::launch_scan_fwd_local(a, local_lanes, sms, stream) == cudaSuccess ? MAMBA_OK
                                                                                        : MAMBA_ERR_CUDA;
    }
    bool persist = false;
    int persist_lanes = 0;
    if (want_sched == MAMBA_SCHEDULE_PERSISTENT) {
        if (!supported || want_threads != 0 ||
            (want_lanes != 0 && want_lanes != 1 && want_lanes != 2 && want_lanes != 4))
            return MAMBA_ERR_UNSUPPORTED;
        if (!ws_ok) return MAMBA_ERR_WORKSPACE;
        persist = true;
        persist_lanes = want_lanes != 0 ? want_lanes : mscan::persistent_choose_lanes(a, sms);
        if (persist_lanes == 0) persist_lanes = 1;
    } else if (want_sched == MAMBA_SCHEDULE_AUTO && want_lanes == 0 && want_threads == 0) {
        persist_lanes = supported && ws_ok ? mscan::persistent_choose_lanes(a, sms) : 0;
        persist = persist_lanes != 0;
    }
    if (persist) {
        if (plan_out) {
            plan_out->lanes_per_channel = persist_lanes;
            plan_out->threads_per_block = 128;
            plan_out->schedule = MAMBA_SCHEDULE_PERSISTENT;
            plan_out->chunk_timesteps = want_chunk;
        }
        if (!launch) return MAMBA_OK;
        note_workspace(workspace);
        return mscan::launch_scan_fwd_persistent(a, persist_lanes, want_chunk, workspace, ws_bytes,
                                                 sms, stream) == cudaSuccess
                   ? MAMBA_OK : MAMBA_ERR_CUDA;
    }
    mscan::ScanPlan pl;
    if (mscan::make_scan_plan(a, want_lanes, want_threads, sms, &pl) != 0) return MAMBA_ERR_UNSUPPORTED;
    if (plan_out) {
        plan_out->lanes_per_channel = pl.lanes;
        plan_out->threads_per_block = pl.threads;
        plan_out->schedule = MAMBA_SCHEDULE_STATIC;
        plan_out->chunk_timesteps = 0;
    }
    if (!launch) return MAMBA_OK;
    return mscan::launch_scan_fwd(a, pl, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

// A strided tensor: its first byte and the bytes up to its last element
// (strides >= 0); false when an offset would not fit the int64 indexing.
struct Span {
    uintptr_t lo;
    size_t bytes;
};
bool strided_span(const void *p, const mamba_stride3_t &s, int64_t nb, int64_t nr, int64_t nt,
                  size_t es, Span *out) {
    if (s.batch < 0 || s.row < 0 || s.time < 0) return false;
    const double last = (double)(nb - 1) * (double)s.batch + (double)(nr - 1) * (double)s.row +
                        (double)(nt - 1) * (double)s.time;
    if (last > (double)kMaxElems) return false;
    out->lo = reinterpret_cast<uintptr_t>(p);
    out->bytes = p ? (size_t)((nb - 1) * s.batch + (nr - 1) * s.row + (nt - 1) * s.time + 1) * es : 0;
    return true;
}
bool spans_overlap(const Span &a, const Span &b) {
    if (!a.bytes || !b.bytes) return false;
    return a.lo < b.lo + b.bytes && b.lo < a.lo + a.bytes;
}
// No two elements at one address: ordered by stride, each extent's step
// clears everything the smaller strides reach (extents of 1 are ignored).
bool injective(const mamba_stride3_t &s, int64_t nb, int64_t nr, int64_t nt) {
    int64_t st[3] = {s.batch, s.row, s.time}, ex[3] = {nb, nr, nt};
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (ex[j] > 1 && (ex[i] <= 1 || st[j] < st[i])) {
                int64_t t = st[i]; st[i] = st[j]; st[j] = t;
                t = ex[i]; ex[i] = ex[j]; ex[j] = t;
            }
    int64_t reach = 0;  // largest offset reachable with the smaller strides
    for (int i = 0; i < 3; ++i) {
        if (ex[i] <= 1) continue;
        if (st[i] <= reach) return false;
        reach += (ex[i] - 1) * st[i];
    }
    return true;
}
bool same_stride(const mamba_stride3_t &a, const mamba_stride3_t &b) {
    return a.batch == b.batch && a.row == b.row && a.time == b.time;
}

}  // namespace

extern "C" {

int mamba_scan_fwd_strided(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *D, const void *z, const float *delta_bias,
                           int delta_softplus, const float *h0, void *out, float *last_state,
                           int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                           int act_dtype, const mamba_scan_strides_t *strides,
                           const mamba_scan_tuning_t *tuning, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (!u || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    int want_lanes = 0, want_threads = 0, want_sched = MAMBA_SCHEDULE_AUTO;
    if (tuning) {
        want_sched = tuning->schedule;
        if (want_sched != MAMBA_SCHEDULE_AUTO && want_sched != MAMBA_SCHEDULE_STATIC &&
            want_sched != MAMBA_SCHEDULE_LOCAL)
            return MAMBA_ERR_UNSUPPORTED;
        want_lanes = tuning->lanes_per_channel;
        want_threads = tuning->threads_per_block;
        if (want_lanes != 0 && want_lanes != 1 && want_lanes != 2 && want_lanes != 4 &&
            want_lanes != 8 && want_lanes != 16)
            return MAMBA_ERR_UNSUPPORTED;
        if (want_threads != 0 && want_threads != 128 && want_threads != 256)
            return MAMBA_ERR_UNSUPPORTED;
    }
    mamba_scan_strides_t st;
    if (strides) {
        st = *strides;
    } else {
        const mamba_stride3_t x{dim * seqlen, seqlen, 1}, bc{dstate * seqlen, seqlen, 1};
        st.u = st.delta = st.z = st.out = x;
        st.B = st.C = bc;
    }
    const size_t es = act_size(act_dtype);
    Span su, sd, sz, so, sb, sc;
    if (!strided_span(u, st.u, batch, dim, seqlen, es, &su) ||
        !strided_span(delta, st.delta, batch, dim, seqlen, es, &sd) ||
        !strided_span(z, st.z, batch, dim, seqlen, es, &sz) ||
        !strided_span(out, st.out, batch, dim, seqlen, es, &so) ||
        !strided_span(B, st.B, batch, dstate, seqlen, es, &sb) ||
        !strided_span(C, st.C, batch, dstate, seqlen, es, &sc))
        return MAMBA_ERR_SHAPE;
    if (!injective(st.out, batch, dim, seqlen)) return MAMBA_ERR_SHAPE;
    const Span sA{reinterpret_cast<uintptr_t>(A), (size_t)(dim * dstate) * 4};
    const Span sD{reinterpret_cast<uintptr_t>(D), D ? (size_t)dim * 4 : 0};
    const Span sbias{reinterpret_cast<uintptr_t>(delta_bias), delta_bias ? (size_t)dim * 4 : 0};
    const size_t nls = (size_t)(batch * dim * dstate) * 4;
    const Span sls{reinterpret_cast<uintptr_t>(last_state), last_state ? nls : 0};
    const Span sh0{reinterpret_cast<uintptr_t>(h0), h0 ? nls : 0};
    // out: in place over u, delta or z with the same map, else apart from every input
    auto in_place = [&](const void *in, const mamba_stride3_t &s) {
        return in == out && same_stride(s, st.out);
    };
    if ((spans_overlap(so, su) && !in_place(u, st.u)) ||
        (spans_overlap(so, sd) && !in_place(delta, st.delta)) ||
        (spans_overlap(so, sz) && !in_place(z, st.z)) || spans_overlap(so, sb) ||
        spans_overlap(so, sc) || spans_overlap(so, sA) || spans_overlap(so, sD) ||
        spans_overlap(so, sbias) || spans_overlap(so, sh0))
        return MAMBA_ERR_OVERLAP;
    const Span ins[] = {su, sd, sz, sb, sc, sA, sD, sbias, so};
    for (const Span &x : ins)
        if (spans_overlap(sls, x)) return MAMBA_ERR_OVERLAP;
    if (h0 && last_state && spans_overlap(sls, sh0) && h0 != last_state) return MAMBA_ERR_OVERLAP;

    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    mscan::ScanStrides ks;
    auto cvt = [](const mamba_stride3_t &s) { return mscan::Stride3{s.batch, s.row, s.time}; };
    ks.u = cvt(st.u); ks.delta = cvt(st.delta); ks.z = cvt(st.z); ks.out = cvt(st.out);
    ks.B = cvt(st.B); ks.C = cvt(st.C);
    mscan::ScanArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out; a.last_state = last_state; a.h0 = h0;
    a.strides = &ks;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    // The pages' own layout -- (batch, L, dim) activations and (batch, L, N)
    // B / C, each dense -- runs on the block-local lane-split kernel with
    // channel-last staging; any other layout, or an explicit static
    // schedule or block size, on the static kernel.
    const mamba_stride3_t xcl{seqlen * dim, 1, dim}, bccl{seqlen * dstate, 1, dstate};
    const bool cl_layout = same_stride(st.u, xcl) && same_stride(st.delta, xcl) && (!z || same_stride(st.z, xcl)) &&
                           same_stride(st.out, xcl) && same_stride(st.B, bccl) && same_stride(st.C, bccl);
    a.channels_last = true;
    const bool cl_ok = cl_layout && mscan::channels_last_supported(a);
    a.channels_last = false;
    if (want_sched == MAMBA_SCHEDULE_LOCAL &&
        (!cl_ok || want_threads != 0 || (want_lanes != 0 && want_lanes != 2 && want_lanes != 4)))
        return MAMBA_ERR_UNSUPPORTED;
    if (cl_ok && want_sched != MAMBA_SCHEDULE_STATIC && want_threads == 0 &&
        (want_lanes == 0 || want_lanes == 2 || want_lanes == 4)) {
        a.strides = nullptr;
        a.channels_last = true;
        int lanes = want_lanes != 0 ? want_lanes : mscan::local_choose_lanes(a, sms);
        if (lanes == 0 && want_sched == MAMBA_SCHEDULE_LOCAL) lanes = 2;
        if (lanes != 0) {
            note_workspace(nullptr);
            return mscan::launch_scan_fwd_local(a, lanes, sms, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
        }
        a.strides = &ks;
        a.channels_last = false;
    }
    mscan::ScanPlan pl;
    if (mscan::make_scan_plan(a, want_lanes, want_threads, sms, &pl) != 0) return MAMBA_ERR_UNSUPPORTED;
    return mscan::launch_scan_fwd(a, pl, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_scan_fwd_complex(const void *u, const void *delta, const float *A, const void *B,
                           const void *C, const float *D, const void *z, const float *delta_bias,
                           int delta_softplus, const float *h0, void *out, float *last_state,
                           int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                           int act_dtype, const mamba_scan_tuning_t *tuning, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (dstate > 16) return MAMBA_ERR_UNSUPPORTED;
    if ((double)batch * (double)dstate * (double)seqlen * 2.0 > (double)kMaxElems) return MAMBA_ERR_SHAPE;
    if (!u || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    int lanes = 0;
    if (tuning) {
        if (tuning->schedule != MAMBA_SCHEDULE_AUTO && tuning->schedule != MAMBA_SCHEDULE_STATIC)
            return MAMBA_ERR_UNSUPPORTED;
        if (tuning->threads_per_block != 0 || tuning->chunk_timesteps != 0) return MAMBA_ERR_UNSUPPORTED;
        lanes = tuning->lanes_per_channel;
        if (lanes != 0 && lanes != 1 && lanes != 2 && lanes != 4) return MAMBA_ERR_UNSUPPORTED;
    }
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim * seqlen) * es;
    const size_t nbc = (size_t)(batch * dstate * seqlen) * 2 * es;
    const size_t nA = (size_t)(dim * dstate) * 8, nd = (size_t)dim * 4;
    const size_t nls = (size_t)(batch * dim * dstate) * 8;
    if (bad_alias(out, nx, u, nx, true) || bad_alias(out, nx, delta, nx, true) ||
        bad_alias(out, nx, z, nx, true) || bad_alias(out, nx, B, nbc, false) ||
        bad_alias(out, nx, C, nbc, false) || bad_alias(out, nx, A, nA, false) ||
        bad_alias(out, nx, D, nd, false) || bad_alias(out, nx, delta_bias, nd, false))
        return MAMBA_ERR_OVERLAP;
    if (last_state &&
        (overlaps(last_state, nls, u, nx) || overlaps(last_state, nls, delta, nx) ||
         overlaps(last_state, nls, z, nx) || overlaps(last_state, nls, B, nbc) ||
         overlaps(last_state, nls, C, nbc) || overlaps(last_state, nls, A, nA) ||
         overlaps(last_state, nls, D, nd) || overlaps(last_state, nls, delta_bias, nd) ||
         overlaps(last_state, nls, out, nx)))
        return MAMBA_ERR_OVERLAP;
    if (h0 && (overlaps(h0, nls, out, nx) || bad_alias(last_state, nls, h0, nls, true)))
        return MAMBA_ERR_OVERLAP;
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    if (lanes == 0) lanes = mscan::complex_scan_lanes(batch, dim, sms);
    mscan::ScanArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out; a.last_state = last_state; a.h0 = h0;
    a.strides = nullptr;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    return mscan::launch_scan_fwd_complex(a, lanes, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_scan_fwd_conv(const void *x, const float *conv_weight, const float *conv_bias,
                        int64_t conv_width, int64_t x_batch_stride, const void *delta,
                        const float *A, const void *B, const void *C, const float *D, const void *z,
                        int64_t z_batch_stride, const float *delta_bias, const float *h0, void *out,
                        float *last_state, void *u_out, int64_t batch, int64_t dim, int64_t seqlen,
                        int64_t dstate, int act_dtype, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (conv_width < 1 || conv_width > 4) return MAMBA_ERR_UNSUPPORTED;
    if (!x || !conv_weight || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    const int64_t dense = dim * seqlen;
    if (x_batch_stride == 0) x_batch_stride = dense;
    if (z_batch_stride == 0) z_batch_stride = dense;
    if (x_batch_stride < dense || z_batch_stride < dense) return MAMBA_ERR_SHAPE;
    if ((double)batch * (double)x_batch_stride > (double)kMaxElems ||
        (double)batch * (double)z_batch_stride > (double)kMaxElems)
        return MAMBA_ERR_SHAPE;
    const size_t es = act_size(act_dtype);
    const int64_t V = 16 / (int64_t)es;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    // the fused prologue lives in the persistent lane-split kernel: its layout rules
    if (dstate > 16 || seqlen % V != 0 || x_batch_stride % V != 0 || z_batch_stride % V != 0 ||
        !al(x) || !al(delta) || !al(z) || !al(B) || !al(C) || !al(out) || !al(u_out))
        return MAMBA_ERR_UNSUPPORTED;
    const size_t nx = (size_t)(batch * dense) * es;
    const size_t nxs = (size_t)((batch - 1) * x_batch_stride + dense) * es;
    const size_t nzs = (size_t)((batch - 1) * z_batch_stride + dense) * es;
    const size_t nbc = (size_t)(batch * dstate * seqlen) * es;
    const size_t nA = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4;
    const size_t nls = (size_t)(batch * dim * dstate) * 4, nw = (size_t)(dim * conv_width) * 4;
    // outputs apart from every input and from each other (a worker reads the
    // conv inputs just before its piece while another writes outputs)
    const void *ins[] = {x, delta, z, B, C, A, D, delta_bias, conv_weight, conv_bias, h0};
    const size_t insz[] = {nxs, nx, nzs, nbc, nbc, nA, nd, nd, nw, nd, nls};
    void *outs[] = {out, u_out, last_state};
    const size_t outsz[] = {nx, nx, nls};
    for (int i = 0; i < 3; ++i) {
        for (int k = 0; k < 11; ++k) {
            if (i == 2 && k == 10 && h0 == last_state) continue;  // the state may advance in place
            if (overlaps(outs[i], outsz[i], ins[k], insz[k])) return MAMBA_ERR_OVERLAP;
        }
        for (int k = 0; k < i; ++k)
            if (overlaps(outs[i], outsz[i], outs[k], outsz[k])) return MAMBA_ERR_OVERLAP;
    }
    const size_t need = mscan::persistent_workspace_bound(batch, dim, seqlen, act_dtype);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15) != 0)
        return MAMBA_ERR_WORKSPACE;
    for (int k = 0; k < 11; ++k)
        if (overlaps(workspace, workspace_bytes, ins[k], insz[k])) return MAMBA_ERR_OVERLAP;
    for (int i = 0; i < 3; ++i)
        if (overlaps(workspace, workspace_bytes, outs[i], outsz[i])) return MAMBA_ERR_OVERLAP;
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    mscan::ScanArgs a;
    a.u = x; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out; a.last_state = last_state; a.h0 = h0;
    a.strides = nullptr;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = 1; a.act = act_dtype;
    a.conv_w = conv_weight; a.conv_b = conv_bias; a.conv_k = (int)conv_width; a.u_out = u_out;
    a.u_bstride = x_batch_stride; a.z_bstride = z_batch_stride;
    int lanes = mscan::persistent_choose_lanes(a, sms);
    if (lanes != 2 && lanes != 4) lanes = 2;  // the balanced split covers any shape
    note_workspace(workspace);
    return mscan::launch_scan_fwd_persistent(a, lanes, 0, workspace, workspace_bytes, sms, stream) == cudaSuccess
               ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_delta_sum(const void *delta, const float *delta_bias, int delta_softplus,
                    double *out, int64_t batch, int64_t dim, int64_t seqlen, int act_dtype,
                    cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, 1);
    if (rc != MAMBA_OK) return rc;
    if (!delta || !out) return MAMBA_ERR_NULL;
    const size_t nx = (size_t)(batch * dim * seqlen) * act_size(act_dtype);
    if (overlaps(out, (size_t)(batch * dim) * 8, delta, nx) ||
        overlaps(out, (size_t)(batch * dim) * 8, delta_bias, (size_t)dim * 4))
        return MAMBA_ERR_OVERLAP;
    return mscan::launch_delta_sum(delta, delta_bias, delta_softplus ? 1 : 0, out, batch, dim, seqlen,
                                   act_dtype, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_state_fold(const float *h_init, const double *delta_sums, const float *A,
                     const float *h_local, float *h_out, int64_t batch, int64_t dim,
                     int64_t dstate, int64_t count, cudaStream_t stream) {
    int rc = check_sizes(batch, dim, 1, dstate);
    if (rc != MAMBA_OK) return rc;
    if (count < 0 || count > (1 << 20)) return MAMBA_ERR_SHAPE;
    if (!A || !h_out || (count > 0 && (!delta_sums || !h_local))) return MAMBA_ERR_NULL;
    const size_t ns = (size_t)(batch * dim * dstate) * 4;
    if ((double)count * (double)ns > (double)kMaxElems) return MAMBA_ERR_SHAPE;
    const size_t nsum = (size_t)count * (size_t)(batch * dim) * 8;
    // h_out may be h_init or one of the h_local slices exactly; nothing else
    if (h_init && overlaps(h_out, ns, h_init, ns) && h_out != h_init) return MAMBA_ERR_OVERLAP;
    if (count > 0 && overlaps(h_out, ns, h_local, (size_t)count * ns)) {
        const uintptr_t off = reinterpret_cast<uintptr_t>(h_out) - reinterpret_cast<uintptr_t>(h_local);
        if (reinterpret_cast<uintptr_t>(h_out) < reinterpret_cast<uintptr_t>(h_local) || off % ns != 0)
            return MAMBA_ERR_OVERLAP;
    }
    if (overlaps(h_out, ns, delta_sums, nsum) || overlaps(h_out, ns, A, (size_t)(dim * dstate) * 4))
        return MAMBA_ERR_OVERLAP;
    return mscan::launch_state_fold(h_init, delta_sums, A, h_local, h_out, batch, dim, dstate, (int)count,
                                    stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                   const void *C, const float *D, const void *z, const float *delta_bias,
                   int delta_softplus, void *out, float *last_state, int64_t batch,
                   int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                   cudaStream_t stream) {
    return scan_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, out, last_state,
                     batch, dim, seqlen, dstate, act_dtype, nullptr, nullptr, 0, stream, true,
                     nullptr);
}

int mamba_scan_fwd_tuned(const void *u, const void *delta, const float *A, const void *B,
                         const void *C, const float *D, const void *z,
                         const float *delta_bias, int delta_softplus, void *out,
                         float *last_state, int64_t batch, int64_t dim, int64_t seqlen,
                         int64_t dstate, int act_dtype, const mamba_scan_tuning_t *tuning,
                         cudaStream_t stream) {
    return scan_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, out, last_state,
                     batch, dim, seqlen, dstate, act_dtype, tuning, nullptr, 0, stream, true,
                     nullptr);
}

int mamba_scan_fwd_ws(const void *u, const void *delta, const float *A, const void *B,
                      const void *C, const float *D, const void *z, const float *delta_bias,
                      int delta_softplus, void *out, float *last_state, int64_t batch,
                      int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                      const mamba_scan_tuning_t *tuning, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
    return scan_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, out, last_state,
                     batch, dim, seqlen, dstate, act_dtype, tuning, workspace, workspace_bytes,
                     stream, true, nullptr);
}

int mamba_scan_fwd_init(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, void *out, float *last_state,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        const mamba_scan_tuning_t *tuning, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
    if (!h0) return MAMBA_ERR_NULL;
    return scan_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, out, last_state,
                     batch, dim, seqlen, dstate, act_dtype, tuning, workspace, workspace_bytes,
                     stream, true, nullptr);
}

int mamba_scan_state(const void *u, const void *delta, const float *A, const void *B,
                     const float *delta_bias, int delta_softplus, const float *h0, float *last_state,
                     int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (!u || !delta || !A || !B || !last_state) return MAMBA_ERR_NULL;
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim * seqlen) * es;
    const size_t nbc = (size_t)(batch * dstate * seqlen) * es;
    const size_t nA = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4;
    const size_t nls = (size_t)(batch * dim * dstate) * 4;
    if (overlaps(last_state, nls, u, nx) || overlaps(last_state, nls, delta, nx) ||
        overlaps(last_state, nls, B, nbc) || overlaps(last_state, nls, A, nA) ||
        overlaps(last_state, nls, delta_bias, nd) || bad_alias(last_state, nls, h0, nls, true))
        return MAMBA_ERR_OVERLAP;
    if (workspace) {
        if ((reinterpret_cast<uintptr_t>(workspace) & 15) != 0) return MAMBA_ERR_WORKSPACE;
        const void *ins[] = {u, delta, B, A, delta_bias, last_state, h0};
        const size_t sz[] = {nx, nx, nbc, nA, nd, nls, nls};
        for (int i = 0; i < 7; ++i)
            if (overlaps(workspace, workspace_bytes, ins[i], sz[i])) return MAMBA_ERR_OVERLAP;
        if (workspace_bytes < mscan::persistent_workspace_bound(batch, dim, seqlen, act_dtype))
            return MAMBA_ERR_WORKSPACE;
    }
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    mscan::ScanArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = nullptr; a.z = nullptr;
    a.A = A; a.D = nullptr; a.delta_bias = delta_bias; a.out = nullptr; a.last_state = last_state; a.h0 = h0;
    a.strides = nullptr;
    a.state_only = true;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    // the lane-split kernel only: dstate <= 16, 16-byte aligned rows
    if (!mscan::persistent_supported(a)) return MAMBA_ERR_UNSUPPORTED;
    if (workspace) {
        int lanes = mscan::persistent_choose_lanes(a, sms);
        if (lanes != 2 && lanes != 4) lanes = 2;
        note_workspace(workspace);
        return mscan::launch_scan_fwd_persistent(a, lanes, 0, workspace, workspace_bytes, sms, stream) == cudaSuccess
                   ? MAMBA_OK : MAMBA_ERR_CUDA;
    }
    int lanes = mscan::local_choose_lanes(a, sms);
    if (lanes == 0) lanes = 2;
    note_workspace(nullptr);
    return mscan::launch_scan_fwd_local(a, lanes, sms, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

size_t mamba_scan_workspace_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                                 int act_dtype) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return 0;
    if (check_sizes(batch, dim, seqlen, dstate) != MAMBA_OK || dstate > 16) return 0;
    return mscan::persistent_workspace_bound(batch, dim, seqlen, act_dtype);
}

int mamba_scan_workspace_status(const void *workspace, cudaStream_t stream) {
    if (!workspace) return MAMBA_ERR_NULL;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MAMBA_ERR_CUDA;
    unsigned hdr[4] = {0, 0, 0, 0};
    if (cudaMemcpy(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MAMBA_ERR_CUDA;
    return hdr[2] != 0 ? MAMBA_ERR_TIMEOUT : MAMBA_OK;
}

int mamba_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MAMBA_ERR_CUDA;
    const cudaError_t sticky = cudaPeekAtLastError();
    if (sticky != cudaSuccess) return MAMBA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MAMBA_ERR_DEVICE;
    int site = 0;
    long long off = 0;
    const int bounds = take_bounds(&site, &off);  // bounds-checked build only
    if (bounds < 0) return MAMBA_ERR_CUDA;
    if (bounds > 0) return MAMBA_ERR_BOUNDS;
    const int local = mscan::local_error_take();  // block-local launches since the last call
    if (local < 0) return MAMBA_ERR_CUDA;
    if (local > 0) return MAMBA_ERR_TIMEOUT;
    const void *ws = (dev >= 0 && dev < kMaxDevices) ? g_last_workspace[dev] : nullptr;
    if (!ws) return MAMBA_OK;
    unsigned hdr[4] = {0, 0, 0, 0};
    if (cudaMemcpy(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess) return MAMBA_ERR_CUDA;
    return hdr[2] != 0 ? MAMBA_ERR_TIMEOUT : MAMBA_OK;
}

int mamba_scan_plan(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                    mamba_scan_tuning_t *plan) {
    if (!plan) return MAMBA_ERR_NULL;
    return scan_impl(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 1,
                     nullptr, nullptr, nullptr, batch, dim, seqlen, dstate, act_dtype, nullptr, nullptr, 0,
                     nullptr, false, plan);
}

int mamba_scan_plan_noworkspace(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                                mamba_scan_tuning_t *plan) {
    if (!plan) return MAMBA_ERR_NULL;
    return scan_impl(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 1,
                     nullptr, nullptr, nullptr, batch, dim, seqlen, dstate, act_dtype, nullptr, nullptr, 0,
                     nullptr, false, plan, true);
}

int mamba_state_update(float *state, const void *u, const void *delta, const float *A,
                       const void *B, const void *C, const float *D, const void *z,
                       const float *delta_bias, int delta_softplus, void *out, int64_t batch,
                       int64_t dim, int64_t dstate, int act_dtype, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, 1, dstate);
    if (rc != MAMBA_OK) return rc;
    if (!state || !u || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim) * es, nbc = (size_t)(batch * dstate) * es;
    const size_t ns = (size_t)(batch * dim * dstate) * 4, nA = (size_t)(dim * dstate) * 4;
    const size_t nd = (size_t)dim * 4;
    if (bad_alias(out, nx, u, nx, true) || bad_alias(out, nx, delta, nx, true) ||
        bad_alias(out, nx, z, nx, true) || bad_alias(out, nx, B, nbc, false) ||
        bad_alias(out, nx, C, nbc, false) || bad_alias(out, nx, A, nA, false) ||
        bad_alias(out, nx, D, nd, false) || bad_alias(out, nx, delta_bias, nd, false) ||
        overlaps(out, nx, state, ns))
        return MAMBA_ERR_OVERLAP;
    if (overlaps(state, ns, u, nx) || overlaps(state, ns, delta, nx) || overlaps(state, ns, z, nx) ||
        overlaps(state, ns, B, nbc) || overlaps(state, ns, C, nbc) || overlaps(state, ns, A, nA) ||
        overlaps(state, ns, D, nd) || overlaps(state, ns, delta_bias, nd))
        return MAMBA_ERR_OVERLAP;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MAMBA_ERR_DEVICE;
    mscan::StateUpdateArgs a;
    a.state = state; a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out;
    a.batch = batch; a.dim = dim; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    return mscan::launch_state_update(a, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

size_t mamba_scan_bwd_workspace_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate) {
    if (check_sizes(batch, dim, seqlen, dstate) != MAMBA_OK || dstate > 16) return 0;
    return mscan::scan_bwd_workspace_bytes(batch, dim, seqlen);
}

namespace {
int scan_bwd_impl(const void *u, const void *delta, const float *A, const void *B, const void *C,
                  const float *D, const void *z, const float *delta_bias, int delta_softplus,
                  const float *h0, const void *dout, const float *dlast_state, void *du,
                  void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz,
                  float *ddelta_bias, float *dh0, int64_t batch, int64_t dim, int64_t seqlen,
                  int64_t dstate, int act_dtype, void *workspace, size_t workspace_bytes,
                  cudaStream_t stream, const float *ckpt = nullptr) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (dstate > 16) return MAMBA_ERR_UNSUPPORTED;
    if (!u || !delta || !A || !B || !C || !dout || !du || !ddelta || !dA || !dB || !dC) return MAMBA_ERR_NULL;
    if ((z != nullptr) != (dz != nullptr)) return MAMBA_ERR_NULL;
    const size_t need = mscan::scan_bwd_workspace_bytes(batch, dim, seqlen);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15))
        return MAMBA_ERR_WORKSPACE;
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim * seqlen) * es, nbc = (size_t)(batch * dstate * seqlen) * es;
    const size_t nbc32 = (size_t)(batch * dstate * seqlen) * 4, nA = (size_t)(dim * dstate) * 4;
    const size_t nd = (size_t)dim * 4, ns = (size_t)(batch * dim * dstate) * 4;
    const size_t nck = ckpt ? (size_t)mscan::scan_bwd_ckpt_floats(batch, dim, seqlen) * 4 : 0;
    if (ckpt && (reinterpret_cast<uintptr_t>(ckpt) & 15) != 0) return MAMBA_ERR_ALIGN;
    const void *ins[] = {u, delta, z, dout, B, C, A, D, delta_bias, dlast_state, workspace, h0, ckpt};
    const size_t inb[] = {nx, nx, nx, nx, nbc, nbc, nA, nd, nd, ns, need, ns, nck};
    void *outs[] = {du, ddelta, dz, dA, dB, dC, dD, ddelta_bias, dh0};
    const size_t outb[] = {nx, nx, nx, nA, nbc32, nbc32, nd, nd, ns};
    if (ckpt && overlaps(ckpt, nck, workspace, need)) return MAMBA_ERR_OVERLAP;
    for (int i = 0; i < 9; ++i) {
        for (int k = 0; k < 13; ++k)
            if (overlaps(outs[i], outb[i], ins[k], inb[k])) return MAMBA_ERR_OVERLAP;
        for (int k = 0; k < i; ++k)
            if (overlaps(outs[i], outb[i], outs[k], outb[k])) return MAMBA_ERR_OVERLAP;
    }
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    mscan::ScanBwdArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z; a.dout = dout;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.dlast = dlast_state; a.h0 = h0;
    a.du = du; a.ddelta = ddelta; a.dz = dz;
    a.dA = dA; a.dB = dB; a.dC = dC; a.dD = dD; a.ddelta_bias = ddelta_bias; a.dh0 = dh0;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    return mscan::launch_scan_bwd(a, workspace, ckpt, sms, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}
}  // namespace

int mamba_scan_bwd(const void *u, const void *delta, const float *A, const void *B, const void *C,
                   const float *D, const void *z, const float *delta_bias, int delta_softplus,
                   const void *dout, const float *dlast_state, void *du, void *ddelta, float *dA,
                   float *dB, float *dC, float *dD, void *dz, float *ddelta_bias, int64_t batch,
                   int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype, void *workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
    return scan_bwd_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, nullptr, dout,
                         dlast_state, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, nullptr, batch,
                         dim, seqlen, dstate, act_dtype, workspace, workspace_bytes, stream);
}

int mamba_scan_bwd_init(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, const void *dout,
                        const float *dlast_state, void *du, void *ddelta, float *dA, float *dB,
                        float *dC, float *dD, void *dz, float *ddelta_bias, float *dh0,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!h0) return MAMBA_ERR_NULL;
    return scan_bwd_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, dout,
                         dlast_state, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0, batch,
                         dim, seqlen, dstate, act_dtype, workspace, workspace_bytes, stream);
}

size_t mamba_scan_ckpt_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate) {
    if (check_sizes(batch, dim, seqlen, dstate) != MAMBA_OK || dstate > 16) return 0;
    return (size_t)mscan::scan_bwd_ckpt_floats(batch, dim, seqlen) * 4;
}

int mamba_scan_fwd_ckpt(const void *u, const void *delta, const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *delta_bias, int delta_softplus,
                        const float *h0, void *out, float *last_state, float *ckpt, size_t ckpt_bytes,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, dstate);
    if (rc != MAMBA_OK) return rc;
    if (!ckpt) return MAMBA_ERR_NULL;
    rc = check_scan_aliases(u, delta, A, B, C, D, z, delta_bias, h0, out, last_state, batch, dim, seqlen, dstate,
                            act_dtype);
    if (rc != MAMBA_OK) return rc;
    if (dstate > 16) return MAMBA_ERR_UNSUPPORTED;
    const size_t need = mamba_scan_ckpt_size(batch, dim, seqlen, dstate);
    if (ckpt_bytes < need || (reinterpret_cast<uintptr_t>(ckpt) & 15) != 0) return MAMBA_ERR_WORKSPACE;
    const size_t es = act_size(act_dtype);
    const size_t nx = (size_t)(batch * dim * seqlen) * es, nbc = (size_t)(batch * dstate * seqlen) * es;
    const size_t nA = (size_t)(dim * dstate) * 4, nd = (size_t)dim * 4, nls = (size_t)(batch * dim * dstate) * 4;
    const void *all[] = {u, delta, z, B, C, A, D, delta_bias, h0, out, last_state};
    const size_t sz[] = {nx, nx, nx, nbc, nbc, nA, nd, nd, nls, nx, nls};
    for (int i = 0; i < 11; ++i)
        if (overlaps(ckpt, need, all[i], sz[i])) return MAMBA_ERR_OVERLAP;
    int status = MAMBA_OK;
    const int sms = current_sm_count(&status);
    if (status != MAMBA_OK) return status;
    mscan::ScanArgs a;
    a.u = u; a.delta = delta; a.B = B; a.C = C; a.z = z;
    a.A = A; a.D = D; a.delta_bias = delta_bias; a.out = out; a.last_state = last_state; a.h0 = h0;
    a.strides = nullptr;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.dstate = (int)dstate;
    a.softplus = delta_softplus ? 1 : 0; a.act = act_dtype;
    a.ckpt = ckpt;
    if (!mscan::persistent_supported(a)) return MAMBA_ERR_UNSUPPORTED;
    int lanes = mscan::local_choose_lanes(a, sms);
    if (lanes == 0) lanes = 2;  // the block-local form covers any shape
    note_workspace(nullptr);
    return mscan::launch_scan_fwd_local(a, lanes, sms, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_scan_bwd_ckpt(const void *u, const void *delta, const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *delta_bias, int delta_softplus,
                        const float *h0, const float *ckpt, const void *dout, const float *dlast_state,
                        void *du, void *ddelta, float *dA, float *dB, float *dC, float *dD, void *dz,
                        float *ddelta_bias, float *dh0, int64_t batch, int64_t dim, int64_t seqlen,
                        int64_t dstate, int act_dtype, void *workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
    if (!ckpt) return MAMBA_ERR_NULL;
    if (dh0 && !h0) return MAMBA_ERR_NULL;
    return scan_bwd_impl(u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, dout, dlast_state, du,
                         ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0, batch, dim, seqlen, dstate, act_dtype,
                         workspace, workspace_bytes, stream, ckpt);
}

int mamba_conv1d_fwd(const void *x, const float *weight, const float *bias, int apply_silu,
                     void *out, int64_t batch, int64_t dim, int64_t seqlen, int64_t width,
                     int64_t x_batch_stride, int act_dtype, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, seqlen, 1);
    if (rc != MAMBA_OK) return rc;
    if (width < 1 || width > 4) return MAMBA_ERR_UNSUPPORTED;
    if (!x || !weight || !out) return MAMBA_ERR_NULL;
    if (x_batch_stride == 0) x_batch_stride = dim * seqlen;
    if (x_batch_stride < dim * seqlen || x_batch_stride > kMaxElems) return MAMBA_ERR_SHAPE;
    if ((double)batch * (double)x_batch_stride > (double)kMaxElems) return MAMBA_ERR_SHAPE;
    const size_t es = act_size(act_dtype);
    const size_t nout = (size_t)(batch * dim * seqlen) * es;
    const size_t nx = (size_t)((batch - 1) * x_batch_stride + dim * seqlen) * es;
    if (overlaps(out, nout, x, nx) || overlaps(out, nout, weight, (size_t)(dim * width) * 4) ||
        overlaps(out, nout, bias, (size_t)dim * 4))
        return MAMBA_ERR_OVERLAP;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MAMBA_ERR_DEVICE;
    mscan::Conv1dArgs a;
    a.x = x; a.weight = weight; a.bias = bias; a.out = out;
    a.batch = batch; a.dim = dim; a.seqlen = seqlen; a.x_batch_stride = x_batch_stride;
    a.width = (int)width; a.silu = apply_silu ? 1 : 0; a.act = act_dtype;
    return mscan::launch_conv1d_fwd(a, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

int mamba_conv1d_update(float *conv_state, const void *x, const float *weight, const float *bias,
                        int apply_silu, void *out, int64_t batch, int64_t dim, int64_t width,
                        int64_t x_batch_stride, int act_dtype, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    int rc = check_sizes(batch, dim, 1, 1);
    if (rc != MAMBA_OK) return rc;
    if (width < 1 || width > 4) return MAMBA_ERR_UNSUPPORTED;
    if (!x || !weight || !out || (width > 1 && !conv_state)) return MAMBA_ERR_NULL;
    if (x_batch_stride == 0) x_batch_stride = dim;
    if (x_batch_stride < dim || x_batch_stride > kMaxElems) return MAMBA_ERR_SHAPE;
    const size_t es = act_size(act_dtype);
    const size_t nout = (size_t)(batch * dim) * es;
    const size_t nx = (size_t)((batch - 1) * x_batch_stride + dim) * es;
    const size_t ns = (size_t)(batch * dim * (width - 1)) * 4;
    if (overlaps(out, nout, x, nx) || overlaps(out, nout, conv_state, ns) ||
        overlaps(out, nout, weight, (size_t)(dim * width) * 4) || overlaps(out, nout, bias, (size_t)dim * 4) ||
        overlaps(conv_state, ns, x, nx) || overlaps(conv_state, ns, weight, (size_t)(dim * width) * 4) ||
        overlaps(conv_state, ns, bias, (size_t)dim * 4))
        return MAMBA_ERR_OVERLAP;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MAMBA_ERR_DEVICE;
    mscan::Conv1dUpdateArgs a;
    a.state = conv_state; a.x = x; a.weight = weight; a.bias = bias; a.out = out;
    a.batch = batch; a.dim = dim; a.x_batch_stride = x_batch_stride;
    a.width = (int)width; a.silu = apply_silu ? 1 : 0; a.act = act_dtype;
    return mscan::launch_conv1d_update(a, stream) == cudaSuccess ? MAMBA_OK : MAMBA_ERR_CUDA;
}

const char *mamba_status_string(int status) {
    switch (status) {
        case MAMBA_OK: return "ok";
        case MAMBA_ERR_NULL: return "a required pointer is NULL";
        case MAMBA_ERR_SHAPE: return "a size is non-positive or too large";
        case MAMBA_ERR_UNSUPPORTED: return "unsupported dstate, dtype or tuning";
        case MAMBA_ERR_ALIGN: return "misaligned pointer";
        case MAMBA_ERR_CUDA: return "CUDA runtime error at launch";
        case MAMBA_ERR_DEVICE: return "no usable CUDA device";
        case MAMBA_ERR_OVERLAP: return "an output overlaps an input or the workspace";
        case MAMBA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case MAMBA_ERR_TIMEOUT: return "a persistent launch stopped waiting for a predecessor chunk";
        case MAMBA_ERR_BOUNDS: return "a kernel access fell outside its tensor (bounds-checked build)";
        default: return "unknown status";
    }
}

int mamba_debug_stall_group(int group) { return mscan::set_stall_group(group < 0 ? -1 : group); }

int mamba_bounds_checked(void) { return mscan::kBoundsChecked ? 1 : 0; }

int mamba_debug_bounds_status(int *site, long long *offset) {
    int s = 0;
    long long o = 0;
    const int r = take_bounds(&s, &o);
    if (r < 0) return MAMBA_ERR_CUDA;
    if (site) *site = s;
    if (offset) *offset = o;
    return r;
}

int mamba_debug_shrink_output_extent(int bytes) {
    const int prev = mscan::g_out_extent_shrink;
    mscan::g_out_extent_shrink = bytes < 0 ? 0 : bytes;
    return prev;
}

int mamba_abi_version(void) { return (1 << 16) | 8; }

}  // extern "C"
