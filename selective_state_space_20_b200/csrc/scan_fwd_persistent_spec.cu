// scan_fwd_persistent_spec.cu -- persistent selective-scan (S6) forward with
// warp specialisation: one lane per channel, all states of the channel in that
// lane, and every scan warp paired with a helper warp.
//
// The arithmetic is that of the other persistent kernels (softplus(delta +
// bias), the zero-order-hold decay exp(delta A), the diagonal recurrence, the
// C readout, the D skip and the silu gate; "Mamba SSM concept and
// implementation in Keras and TensorFlow", recurrent form and selective_scan /
// MambaBlock; fused as in the Mamba paper, Appendix E.5).  What differs is who
// does it.  A block holds four (scan warp, helper warp) pairs, warp w and warp
// w + 4, one pair per SM sub-partition.  The scan warp runs nothing but the
// recurrence: per timestep and lane, 16 decays (14 on the MUFU, 2 on the FMA
// pipe through ex2_poly2, which balances the two pipes), 16 state updates and
// the 16-term readout.  The helper warp does everything else, overlapped with
// the scan of the neighbouring sub-chunk:
//   * stages the raw u / delta / z rows and the B / C rows of a sub-chunk of
//     kTC timesteps with cp.async, NRAW sub-chunks ahead;
//   * prologue: delta = softplus(delta_raw + bias) and delta * u per element,
//     written as (delta_t, delta_t u_t) pairs; B and C widened to fp32 [t][n]
//     rows that the scan reads with broadcast loads;
//   * epilogue: out = (y + D u) * silu(z) from the scan's fp32 readouts and the
//     staged u / z rows, packed and stored to global memory.
// fp32 activations take the accurate decay and softplus of device_math.cuh
// (Decay<true>) for all 16 states instead, with the states and the readout in
// fp64.
// The pair hands sub-chunks back and forth through two processed-data slots,
// each guarded by a pair of mbarriers (full: helper -> scan, done: scan ->
// helper).  Every wait is bounded in time; a timeout raises the error word.
//
// Work units and the ready queue are those of persistent_common.cuh.  The
// helper claims units ahead of use; a claimed unit whose predecessor has not
// finished yet is not waited for -- the helper hands the scan warp an empty
// (skip) sub-chunk and polls again next time, so the pair never blocks on a
// unit that it may itself have to finish.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "device_math.cuh"
#include "internal.h"
#include "persistent_common.cuh"
#include "persistent_kernels.h"

namespace mscan {
namespace {

using namespace persist;

constexpr int kPairs = 4;           // (scan, helper) pairs per block
constexpr int kTC = 16;             // timesteps per sub-chunk
constexpr int kChannels = 32;       // channels per unit: one per lane
constexpr uint64_t kWaitNs = 2000000000ull;  // give up a wait after 2 s

constexpr unsigned kFirst = 1u, kLast = 2u, kEnd = 4u, kSkip = 8u;

// One sub-chunk of a unit, as the helper hands it along (48 bytes).
struct Desc {
    unsigned unit;
    int sub;           // sub-chunk within the unit
    unsigned flags;
    int tvalid;        // timesteps of the sub-chunk inside the sequence
    int g, j;          // channel group, time chunk
    int b, d0;         // batch, first channel of the group
    long long rowidx;  // b * dim + d0: row of the group's first channel
    long long t0;      // first timestep
};
static_assert(sizeof(Desc) == 48, "descriptor layout");

template <typename T>
struct SpecSmem {
    static constexpr int V = 16 / (int)sizeof(T);         // elements per 16 bytes
    static constexpr int CPR = kTC / V;                   // 16-byte chunks per raw row
    static constexpr int ROWB = kTC * (int)sizeof(T) + 16;  // raw row pitch
    static constexpr int ROW_U = 0, ROW_D = 32, ROW_Z = 64, ROW_B = 96, ROW_C = 112;
    static constexpr int RAW_ROWS = 128;
    static constexpr int HDR = (int)sizeof(Desc);
    static constexpr int RAW = HDR + RAW_ROWS * ROWB;     // descriptor, then rows
    static constexpr int NRAW = sizeof(T) == 2 ? 4 : 3;   // raw slots in flight
    static constexpr int DLB = kTC * 8 + 16;              // (delta, delta u) row pitch
    static constexpr int DL_OFF = HDR;
    static constexpr int BC_OFF = DL_OFF + kChannels * DLB;
    static constexpr int C_FLOATS = kTC * kNS + 16;       // C starts 64 bytes after B's end
    static constexpr int PROC = BC_OFF + (kTC * kNS + C_FLOATS) * 4;
    static constexpr int YB = kTC * 4 + 16;               // readout row pitch
    static constexpr int Y = kChannels * YB;
    static constexpr int PROC_OFF = NRAW * RAW;
    static constexpr int Y_OFF = PROC_OFF + 2 * PROC;     // three readout slots
    static constexpr int BAR_OFF = Y_OFF + 3 * Y;         // 4 mbarriers
    static constexpr int PAIR = BAR_OFF + 32;
    static_assert(RAW % 16 == 0 && PROC % 16 == 0 && Y % 16 == 0 && BAR_OFF % 16 == 0, "16-byte alignment");
    static_assert(ROW_C == ROW_B + kNS && ROW_C + kNS == RAW_ROWS, "B rows, then C rows");
};

// ------------------------------------------------------------- mbarriers
__device__ __forceinline__ unsigned saddr(const void *p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(saddr(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(saddr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase with the given parity to complete; false after a timeout
// (which raises the error word) or when another worker raised it.
__device__ __noinline__ bool mbar_wait(uint64_t *bar, unsigned parity, unsigned *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (ld_acquire(err) != 0u) return false;
        if (global_ns() - t0 > kWaitNs) {
            atomicOr(err, 2u);
            return false;
        }
    }
}

template <typename T>
__device__ __forceinline__ void unpack_row(const unsigned char *src, float (&f)[kTC]) {
    constexpr int V = 16 / (int)sizeof(T);
#pragma unroll
    for (int c = 0; c < kTC / V; ++c)
        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(src + c * 16), f + c * V);
}

// ---------------------------------------------------------- the helper warp
template <typename T>
struct Helper {
    using W = SpecSmem<T>;
    const Params &p;
    unsigned char *pair;  // this pair's shared memory
    int lane;
    // unit generator (all lanes hold the same values)
    unsigned unit;        // unit being handed out, or kUnitDone when a new one is needed
    int sub, nsub, g, j, b, d0;
    long long rowidx;
    long long pending;    // claimed queue slot not yet ready, or -1
    bool finished;
    uint64_t skip_since;  // lane 0: when the pending slot was first found empty
    // per-lane source offsets of this lane's 16-byte copies (elements, before
    // the sub-chunk's first timestep is added)
    long long off_x[W::CPR], off_bc[W::CPR];
    int row_x[W::CPR], n_bc[W::CPR], c_x;

    __device__ Helper(const Params &p_, unsigned char *pair_, int lane_)
        : p(p_), pair(pair_), lane(lane_), unit(kUnitDone), sub(0), nsub(0), g(0), j(0), b(0), d0(0),
          rowidx(0), pending(-1), finished(false), skip_since(0) {
        // copy i = lane + 32 it covers row i / CPR, 16-byte chunk i % CPR
        c_x = lane % W::CPR;
#pragma unroll
        for (int it = 0; it < W::CPR; ++it) {
            const int i = lane + 32 * it;
            row_x[it] = i / W::CPR;
            off_x[it] = (long long)row_x[it] * p.seqlen + c_x * W::V;
            const int rem = i % (kNS * W::CPR);
            n_bc[it] = rem / W::CPR;
            off_bc[it] = (long long)n_bc[it] * p.seqlen + c_x * W::V;
        }
    }

    __device__ unsigned char *raw(int k) const { return pair + (k % W::NRAW) * W::RAW; }
    __device__ unsigned char *proc(int k) const { return pair + W::PROC_OFF + (k & 1) * W::PROC; }
    __device__ unsigned char *ybuf(int k) const { return pair + W::Y_OFF + (k % 3) * W::Y; }

    // Descriptor of the next sub-chunk in this pair's stream.
    __device__ Desc next() {
        Desc d{};
        d.flags = kEnd;
        if (finished) return d;
        if (unit == kUnitDone) {
            const unsigned n_units = (unsigned)p.n_groups * (unsigned)p.n_chunks;
            if (pending < 0) {
                unsigned s = 0;
                if (lane == 0) s = atomicAdd(p.hdr + 0, 1u);
                s = __shfl_sync(0xffffffffu, s, 0);
                if (s >= n_units) {
                    finished = true;
                    return d;
                }
                if (s < (unsigned)p.n_groups) unit = s;
                else pending = (long long)(s - (unsigned)p.n_groups);
            }
            if (pending >= 0) {
                unsigned v = 0;
                if (lane == 0) v = ld_acquire(p.queue + pending);
                v = __shfl_sync(0xffffffffu, v, 0);
                if (v == 0u) {
                    unsigned bad = 0;
                    if (lane == 0) {
                        const uint64_t now = global_ns();
                        if (skip_since == 0) skip_since = now;
                        bad = ld_acquire(p.hdr + 2) != 0u || now - skip_since > kWaitNs;
                        if (bad) atomicOr(p.hdr + 2, 1u);
                    }
                    if (__shfl_sync(0xffffffffu, bad, 0)) {
                        finished = true;
                        return d;
                    }
                    d.flags = kSkip;
                    return d;
                }
                unit = v - 1u;
                pending = -1;
                skip_since = 0;
            }
            g = (int)(unit % (unsigned)p.n_groups);
            j = (int)(unit / (unsigned)p.n_groups);
            b = g / p.groups_per_batch;
            d0 = (g % p.groups_per_batch) * kChannels;
            rowidx = (long long)b * p.dim + d0;
            const long long ts = (long long)j * p.chunk_len;
            const long long len = (p.seqlen - ts) < p.chunk_len ? (p.seqlen - ts) : p.chunk_len;
            sub = 0;
            nsub = (int)((len + kTC - 1) / kTC);
        }
        d.unit = unit;
        d.sub = sub;
        d.flags = (sub == 0 ? kFirst : 0u) | (sub + 1 == nsub ? kLast : 0u);
        d.g = g; d.j = j; d.b = b; d.d0 = d0;
        d.rowidx = rowidx;
        d.t0 = (long long)j * p.chunk_len + (long long)sub * kTC;
        d.tvalid = (p.seqlen - d.t0) < kTC ? (int)(p.seqlen - d.t0) : kTC;
        if (++sub == nsub) unit = kUnitDone;
        return d;
    }

    // Stage sub-chunk k's raw rows (one cp.async group, possibly empty).
    __device__ void issue(int k, const Desc &d) {
        unsigned char *rb = raw(k);
        if (lane == 0) *reinterpret_cast<Desc *>(rb) = d;
        if ((d.flags & (kEnd | kSkip)) == 0) {
            const long long L = p.seqlen;
            const long long base_x = d.rowidx * L + d.t0;
            const long long base_bc = (long long)d.b * p.dstate * L + d.t0;
            const int nrows = (p.dim - d.d0) < kChannels ? (int)(p.dim - d.d0) : kChannels;
            const bool tok = d.t0 + c_x * W::V < L;
            const T *gu = static_cast<const T *>(p.u);
            const T *gd = static_cast<const T *>(p.delta);
            const T *gz = static_cast<const T *>(p.z);
            const T *gB = static_cast<const T *>(p.B);
            const T *gC = static_cast<const T *>(p.C);
            unsigned char *rows = rb + W::HDR + c_x * 16;
#pragma unroll
            for (int it = 0; it < W::CPR; ++it) {
                const bool ok = tok && row_x[it] < nrows;
                const long long off = ok ? base_x + off_x[it] : 0;
                cp16(rows + (W::ROW_U + row_x[it]) * W::ROWB, gu + off, ok && MSCAN_WITHIN(p.x_u, gu + off, 16, kSiteU));
                cp16(rows + (W::ROW_D + row_x[it]) * W::ROWB, gd + off,
                     ok && MSCAN_WITHIN(p.x_delta, gd + off, 16, kSiteDelta));
                if (gz)
                    cp16(rows + (W::ROW_Z + row_x[it]) * W::ROWB, gz + off, ok && MSCAN_WITHIN(p.x_z, gz + off, 16, kSiteZ));
            }
#pragma unroll
            for (int it = 0; it < W::CPR; ++it) {
                const int which = (lane + 32 * it) / (kNS * W::CPR);
                const bool ok = tok && n_bc[it] < p.dstate;
                const long long off = ok ? base_bc + off_bc[it] : 0;
                cp16(rows + (W::ROW_B + which * kNS + n_bc[it]) * W::ROWB, (which ? gC : gB) + off,
                     ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, (which ? gC : gB) + off, 16, which ? kSiteC : kSiteB));
            }
        }
        cp_commit();
    }

    // Prologue of sub-chunk k (raw rows landed): per-element delta and
    // delta * u, B and C in fp32 [t][n]; the descriptor goes along.
    template <bool SP>
    __device__ void prologue(int k, const Desc &d) {
        unsigned char *pb = proc(k);
        if (lane == 0) *reinterpret_cast<Desc *>(pb) = d;
        if (d.flags & (kEnd | kSkip)) return;
        const unsigned char *rows = raw(k) + W::HDR;
        const int dc = d.d0 + lane;
        const float bias = (dc < p.dim && p.delta_bias && MSCAN_WITHIN(p.x_bias, p.delta_bias + dc, 4, kSiteBias))
                               ? __ldg(p.delta_bias + dc) : 0.f;
        float fu[kTC], fd[kTC];
        unpack_row<T>(rows + (W::ROW_U + lane) * W::ROWB, fu);
        unpack_row<T>(rows + (W::ROW_D + lane) * W::ROWB, fd);
        unsigned char *dl = pb + W::DL_OFF + lane * W::DLB;
#pragma unroll
        for (int t = 0; t < kTC; t += 2) {
            float2 x = __fadd2_rn(f2(fd[t], fd[t + 1]), f2(bias, bias));
            if (SP) x = Decay<sizeof(T) == 4>::softplus2(x);
            x.x = t < d.tvalid ? x.x : 0.f;  // past the end: decay 1, no input
            x.y = t + 1 < d.tvalid ? x.y : 0.f;
            const float2 xu = __fmul2_rn(x, f2(fu[t], fu[t + 1]));
            *reinterpret_cast<float4 *>(dl + t * 8) = make_float4(x.x, xu.x, x.y, xu.y);
        }
        // B (lanes 0-15) and C (lanes 16-31), one state row each
        float *bc = reinterpret_cast<float *>(pb + W::BC_OFF) + (lane >> 4) * (kTC * kNS + 16) + (lane & 15);
        float fb[kTC];
        unpack_row<T>(rows + (W::ROW_B + lane) * W::ROWB, fb);
#pragma unroll
        for (int t = 0; t < kTC; ++t) bc[t * kNS] = fb[t];
    }

    // Epilogue of sub-chunk k (scan done): out = (y + D u) * silu(z).
    template <bool GATE>
    __device__ void epilogue(int k, const Desc &d) {
        if (d.flags & (kEnd | kSkip)) return;
        const int dc = d.d0 + lane;
        if (dc >= p.dim) return;
        const unsigned char *rows = raw(k) + W::HDR;
        const float Dd = (p.D && MSCAN_WITHIN(p.x_D, p.D + dc, 4, kSiteD)) ? __ldg(p.D + dc) : 0.f;
        float fu[kTC], fz[kTC], y[kTC];
        unpack_row<T>(rows + (W::ROW_U + lane) * W::ROWB, fu);
        if (GATE) unpack_row<T>(rows + (W::ROW_Z + lane) * W::ROWB, fz);
        const float4 *yr = reinterpret_cast<const float4 *>(ybuf(k) + lane * W::YB);
#pragma unroll
        for (int i = 0; i < kTC / 4; ++i) {
            const float4 v = yr[i];
            y[4 * i] = v.x; y[4 * i + 1] = v.y; y[4 * i + 2] = v.z; y[4 * i + 3] = v.w;
        }
        float o[kTC];
#pragma unroll
        for (int t = 0; t < kTC; t += 2) {
            const float2 yy = __ffma2_rn(f2(Dd, Dd), f2(fu[t], fu[t + 1]), f2(y[t], y[t + 1]));
            const float2 oo = GATE ? __fmul2_rn(yy, silu2_f(f2(fz[t], fz[t + 1]))) : yy;
            o[t] = oo.x;
            o[t + 1] = oo.y;
        }
        T *dst = static_cast<T *>(p.out) + (d.rowidx + lane) * p.seqlen + d.t0;
#pragma unroll
        for (int c = 0; c < W::CPR; ++c)
            if (c * W::V < d.tvalid && MSCAN_WITHIN(p.x_out, dst + c * W::V, 16, kSiteOut))
                stg16_stream(dst + c * W::V, Elem<T>::pack(o + c * W::V));
    }
};

// ------------------------------------------------------------ the kernel
template <typename T, bool SP, bool GATE>
__global__ void __launch_bounds__(2 * kPairs * 32, 1) scan_fwd_spec_kernel(const Params p) {
    using W = SpecSmem<T>;
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair_id = warp % kPairs;
    const bool is_helper = warp >= kPairs;
    unsigned char *pair = smem + pair_id * W::PAIR;
    uint64_t *full = reinterpret_cast<uint64_t *>(pair + W::BAR_OFF);  // [2]
    uint64_t *done = full + 2;                                          // [2]
    unsigned *err = p.hdr + 2;
    if (is_helper && lane == 0) {
        mbar_init(full + 0, 1); mbar_init(full + 1, 1);
        mbar_init(done + 0, 1); mbar_init(done + 1, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (is_helper) {
        // Iteration k (the scan warp runs sub-chunk k): once the scan is done
        // with k-1, prepare k+1 in its processed slot and hand it over; then
        // finish k-1 and refill k-1's raw slot with sub-chunk k + NRAW - 1.
        Helper<T> h(p, pair, lane);
        constexpr int NR = W::NRAW;
        for (int k = 0; k < NR - 1; ++k) h.issue(k, h.next());
        cp_wait<NR - 2>();
        __syncwarp();
        Desc dcur = *reinterpret_cast<const Desc *>(h.raw(0));
        h.template prologue<SP>(0, dcur);
        __syncwarp();
        if (lane == 0) mbar_arrive(full + 0);
        bool ok = true;
        Desc dprev{};
        dprev.flags = kSkip;
        int k = 0;
        while (!(dcur.flags & kEnd)) {
            if (k >= 1 && !mbar_wait(done + ((k - 1) & 1), ((k - 1) >> 1) & 1, err)) {
                ok = false;
                break;
            }
            cp_wait<NR - 3>();  // sub-chunk k+1's rows have landed
            __syncwarp();
            const Desc dnext = *reinterpret_cast<const Desc *>(h.raw(k + 1));
            h.template prologue<SP>(k + 1, dnext);
            __syncwarp();
            if (lane == 0) mbar_arrive(full + ((k + 1) & 1));
            if (k >= 1) {
                h.template epilogue<GATE>(k - 1, dprev);
                __syncwarp();  // k-1's raw rows are read before the slot is refilled
            }
            h.issue(k + NR - 1, h.next());
            dprev = dcur;
            dcur = dnext;
            ++k;
        }
        // dcur (sub-chunk k) is the end marker; k-1 still needs its epilogue
        if (ok && k >= 1 && mbar_wait(done + ((k - 1) & 1), ((k - 1) >> 1) & 1, err))
            h.template epilogue<GATE>(k - 1, dprev);
        cp_wait<0>();
        return;
    }

    // ---- scan warp: lane = channel, all states in registers (pairs: fp32
    // for bf16 activations, fp64 for fp32 ones; Decay's note says why)
    constexpr bool ACC = sizeof(T) == 4;
    using HV = typename std::conditional<ACC, double2, float2>::type;
    auto hv = [](float a, float b) {
        HV r;
        r.x = a;
        r.y = b;
        return r;
    };
    int cur_group = -1;
    float2 A2[kNS / 2];
    HV hs[kNS / 2];
#pragma unroll
    for (int q = 0; q < kNS / 2; ++q) { A2[q] = f2(0.f, 0.f); hs[q] = hv(0.f, 0.f); }
    const int N = p.dstate;
    for (int k = 0;; ++k) {
        if (!mbar_wait(full + (k & 1), (k >> 1) & 1, err)) return;
        const unsigned char *pb = pair + W::PROC_OFF + (k & 1) * W::PROC;
        const Desc d = *reinterpret_cast<const Desc *>(pb);
        if (d.flags & kEnd) return;
        if (!(d.flags & kSkip)) {
            const int dc = d.d0 + lane;
            float *carry = p.carry + ((int64_t)d.g * 32 + lane) * kNS;
            if (d.flags & kFirst) {
                if (d.g != cur_group) {
                    cur_group = d.g;
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q) {
                        const int n0 = 2 * q, n1 = 2 * q + 1;
                        const float *a = p.A + (int64_t)dc * N;
                        const float a0 = (dc < p.dim && n0 < N && MSCAN_WITHIN(p.x_A, a + n0, 4, kSiteA)) ? __ldg(a + n0) : 0.f;
                        const float a1 = (dc < p.dim && n1 < N && MSCAN_WITHIN(p.x_A, a + n1, 4, kSiteA)) ? __ldg(a + n1) : 0.f;
                        A2[q] = f2(a0 * Decay<sizeof(T) == 4>::kScale, a1 * Decay<sizeof(T) == 4>::kScale);
                    }
                }
                if (d.j == 0) {  // the initial state, or zeros
                    const float *src = p.h0 + (d.rowidx + lane) * N;
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q)
                        hs[q] = (p.h0 && dc < p.dim)
                                    ? hv((2 * q < N && MSCAN_WITHIN(p.x_h0, src + 2 * q, 4, kSiteH0)) ? __ldcg(src + 2 * q) : 0.f,
                                         (2 * q + 1 < N && MSCAN_WITHIN(p.x_h0, src + 2 * q + 1, 4, kSiteH0))
                                             ? __ldcg(src + 2 * q + 1) : 0.f)
                                    : hv(0.f, 0.f);
                } else {
#pragma unroll
                    for (int q = 0; q < kNS / 4; ++q) {
                        const float4 v = MSCAN_WITHIN(p.x_carry, reinterpret_cast<const float4 *>(carry) + q, 16, kSiteCarry)
                                             ? __ldcg(reinterpret_cast<const float4 *>(carry) + q)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                        hs[2 * q] = hv(v.x, v.y);
                        hs[2 * q + 1] = hv(v.z, v.w);
                    }
                }
            }
            const float4 *dlrow = reinterpret_cast<const float4 *>(pb + W::DL_OFF + lane * W::DLB);
            const float *sB = reinterpret_cast<const float *>(pb + W::BC_OFF);
            const float *sC = sB + kTC * kNS + 16;
            float4 *yrow = reinterpret_cast<float4 *>(pair + W::Y_OFF + (k % 3) * W::Y + lane * W::YB);
#pragma unroll 1
            for (int tb = 0; tb < kTC; tb += 8) {
                float4 dd[4];  // (delta_t, delta_t u_t, delta_t+1, delta_t+1 u_t+1)
#pragma unroll
                for (int i = 0; i < 4; ++i) dd[i] = dlrow[tb / 2 + i];
                float2 y2[8];  // readout partial sums (fp64 in yd with fp32 activations)
                double yd[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    y2[e] = f2(0.f, 0.f);
                    yd[e] = 0.0;
                }
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int t = tb + e;
                        const float dl = (e & 1) ? dd[e >> 1].z : dd[e >> 1].x;
                        const float du = (e & 1) ? dd[e >> 1].w : dd[e >> 1].y;
                        const float4 bb = *reinterpret_cast<const float4 *>(sB + t * kNS + 4 * q);
                        const float4 cc = *reinterpret_cast<const float4 *>(sC + t * kNS + 4 * q);
                        const float2 x0 = __fmul2_rn(f2(dl, dl), A2[2 * q]);
                        const float2 x1 = __fmul2_rn(f2(dl, dl), A2[2 * q + 1]);
                        const float2 bu0 = __fmul2_rn(f2(du, du), f2(bb.x, bb.y));
                        const float2 bu1 = __fmul2_rn(f2(du, du), f2(bb.z, bb.w));
                        if constexpr (ACC) {  // fp32 activations: the accurate decay, fp64 state
                            hs[2 * q].x = Decay<true>::step(x0.x, hs[2 * q].x, bu0.x);
                            hs[2 * q].y = Decay<true>::step(x0.y, hs[2 * q].y, bu0.y);
                            hs[2 * q + 1].x = Decay<true>::step(x1.x, hs[2 * q + 1].x, bu1.x);
                            hs[2 * q + 1].y = Decay<true>::step(x1.y, hs[2 * q + 1].y, bu1.y);
                            yd[e] = fma((double)cc.x, hs[2 * q].x, yd[e]);
                            yd[e] = fma((double)cc.y, hs[2 * q].y, yd[e]);
                            yd[e] = fma((double)cc.z, hs[2 * q + 1].x, yd[e]);
                            yd[e] = fma((double)cc.w, hs[2 * q + 1].y, yd[e]);
                        } else {
                            const float2 a0 = f2(ex2_mufu(x0.x), ex2_mufu(x0.y));
                            // states 14 and 15 on the FMA pipe
                            const float2 a1 = q == kNS / 4 - 1 ? ex2_poly2(x1) : f2(ex2_mufu(x1.x), ex2_mufu(x1.y));
                            hs[2 * q] = __ffma2_rn(a0, hs[2 * q], bu0);
                            hs[2 * q + 1] = __ffma2_rn(a1, hs[2 * q + 1], bu1);
                            y2[e] = __ffma2_rn(f2(cc.x, cc.y), hs[2 * q], y2[e]);
                            y2[e] = __ffma2_rn(f2(cc.z, cc.w), hs[2 * q + 1], y2[e]);
                        }
                    }
                }
                float yv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) yv[e] = ACC ? (float)yd[e] : y2[e].x + y2[e].y;
                yrow[tb / 4] = make_float4(yv[0], yv[1], yv[2], yv[3]);
                yrow[tb / 4 + 1] = make_float4(yv[4], yv[5], yv[6], yv[7]);
            }
            if (d.flags & kLast) {
                if (d.j + 1 < p.n_chunks) {
#pragma unroll
                    for (int q = 0; q < kNS / 4; ++q)
                        if (MSCAN_WITHIN(p.x_carry, reinterpret_cast<float4 *>(carry) + q, 16, kSiteCarry))
                            __stcg(reinterpret_cast<float4 *>(carry) + q,
                                   make_float4((float)hs[2 * q].x, (float)hs[2 * q].y, (float)hs[2 * q + 1].x,
                                               (float)hs[2 * q + 1].y));
                    push_unit(p, lane, (unsigned)((d.j + 1) * p.n_groups + d.g));
                } else if (p.last_state != nullptr && dc < p.dim) {
                    float *ls = p.last_state + (d.rowidx + lane) * N;
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q) {
                        if (2 * q < N && MSCAN_WITHIN(p.x_last, ls + 2 * q, 4, kSiteLastState)) ls[2 * q] = (float)hs[q].x;
                        if (2 * q + 1 < N && MSCAN_WITHIN(p.x_last, ls + 2 * q + 1, 4, kSiteLastState))
                            ls[2 * q + 1] = (float)hs[q].y;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(done + (k & 1));
    }
}

template <typename T, bool SP, bool GATE>
cudaError_t launch_t(const Params &kp, int grid, cudaStream_t st) {
    const int smem = kPairs * SpecSmem<T>::PAIR;
    auto kern = scan_fwd_spec_kernel<T, SP, GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 2 * kPairs * 32, smem, st>>>(kp);
    return cudaGetLastError();
}

}  // namespace

MSCAN_BOUNDS_TAKE(spec_bounds_take)

int persistent_spec_sub_chunk() { return kTC; }
int persistent_spec_pairs_per_sm() { return kPairs; }

cudaError_t launch_persistent_spec(const Params &kp, int act, int grid, cudaStream_t st) {
    const bool gate = kp.z != nullptr;
    if (act == kBF16) {
        if (kp.softplus) return gate ? launch_t<__nv_bfloat16, true, true>(kp, grid, st)
                                     : launch_t<__nv_bfloat16, true, false>(kp, grid, st);
        return gate ? launch_t<__nv_bfloat16, false, true>(kp, grid, st)
                    : launch_t<__nv_bfloat16, false, false>(kp, grid, st);
    }
    if (kp.softplus) return gate ? launch_t<float, true, true>(kp, grid, st) : launch_t<float, true, false>(kp, grid, st);
    return gate ? launch_t<float, false, true>(kp, grid, st) : launch_t<float, false, false>(kp, grid, st);
}

}  // namespace mscan
