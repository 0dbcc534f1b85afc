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

struct Desc {
    unsigned unit;
    int sub;
    unsigned flags;
    int tvalid;
};

template <typename T>
struct SpecSmem {
    static constexpr int V = 16 / (int)sizeof(T);         // elements per 16 bytes
    static constexpr int CPR = kTC / V;                   // 16-byte chunks per raw row
    static constexpr int ROWB = kTC * (int)sizeof(T) + 16;  // raw row pitch
    static constexpr int ROW_U = 0, ROW_D = 32, ROW_Z = 64, ROW_B = 96, ROW_C = 112;
    static constexpr int RAW_ROWS = 128;
    static constexpr int RAW = 16 + RAW_ROWS * ROWB;      // descriptor, then rows
    static constexpr int NRAW = sizeof(T) == 2 ? 4 : 3;   // raw slots in flight
    static constexpr int DLB = kTC * 8 + 16;              // (delta, delta u) row pitch
    static constexpr int DL_OFF = 16;                     // after the descriptor
    static constexpr int BC_OFF = DL_OFF + kChannels * DLB;
    static constexpr int C_FLOATS = kTC * kNS + 16;       // C starts 64 bytes after B's end
    static constexpr int YB = kTC * 4 + 16;               // readout row pitch
    static constexpr int Y_OFF = BC_OFF + (kTC * kNS + C_FLOATS) * 4;
    static constexpr int PROC = Y_OFF + kChannels * YB;
    static constexpr int BAR_OFF = NRAW * RAW + 2 * PROC;  // 4 mbarriers
    static constexpr int PAIR = BAR_OFF + 32;
    static_assert(RAW % 16 == 0 && PROC % 16 == 0 && BAR_OFF % 16 == 0, "16-byte alignment");
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
    // unit generator
    unsigned unit;        // current unit, or kUnitDone when a new one is needed
    int sub, nsub;
    long long pending;    // claimed queue slot not yet ready, or -1
    bool finished;
    uint64_t skip_since;

    __device__ Helper(const Params &p_, unsigned char *pair_, int lane_)
        : p(p_), pair(pair_), lane(lane_), unit(kUnitDone), sub(0), nsub(0), pending(-1),
          finished(false), skip_since(0) {}

    __device__ unsigned char *raw(int k) const { return pair + (k % W::NRAW) * W::RAW; }
    __device__ unsigned char *proc(int k) const { return pair + W::NRAW * W::RAW + (k & 1) * W::PROC; }

    __device__ int unit_subs(unsigned u) const {
        const int j = (int)(u / (unsigned)p.n_groups);
        const int64_t t0 = (int64_t)j * p.chunk_len;
        const int64_t len = (p.seqlen - t0) < p.chunk_len ? (p.seqlen - t0) : p.chunk_len;
        return (int)((len + kTC - 1) / kTC);
    }

    // Descriptor of the next sub-chunk in this pair's stream.
    __device__ Desc next() {
        Desc d{0u, 0, kEnd, 0};
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
            sub = 0;
            nsub = unit_subs(unit);
        }
        d.unit = unit;
        d.sub = sub;
        d.flags = (sub == 0 ? kFirst : 0u) | (sub + 1 == nsub ? kLast : 0u);
        const int j = (int)(unit / (unsigned)p.n_groups);
        const int64_t t0 = (int64_t)j * p.chunk_len + (int64_t)sub * kTC;
        d.tvalid = (p.seqlen - t0) < kTC ? (int)(p.seqlen - t0) : kTC;
        if (++sub == nsub) unit = kUnitDone;
        return d;
    }

    // Stage sub-chunk k's raw rows (one cp.async group, possibly empty).
    __device__ void issue(int k, const Desc &d) {
        unsigned char *rb = raw(k);
        if (lane == 0) *reinterpret_cast<Desc *>(rb) = d;
        if ((d.flags & (kEnd | kSkip)) == 0) {
            const int g = (int)(d.unit % (unsigned)p.n_groups);
            const int j = (int)(d.unit / (unsigned)p.n_groups);
            const int64_t b = g / p.groups_per_batch;
            const int64_t d0 = (int64_t)(g % p.groups_per_batch) * kChannels;
            const int nrows = (p.dim - d0) < kChannels ? (int)(p.dim - d0) : kChannels;
            const int64_t L = p.seqlen;
            const int64_t t0 = (int64_t)j * p.chunk_len + (int64_t)d.sub * kTC;
            const int64_t row0 = (b * p.dim + d0) * L;
            const int64_t bc0 = b * (int64_t)p.dstate * L;
            const T *gu = static_cast<const T *>(p.u);
            const T *gd = static_cast<const T *>(p.delta);
            const T *gz = static_cast<const T *>(p.z);
            const T *gB = static_cast<const T *>(p.B);
            const T *gC = static_cast<const T *>(p.C);
            unsigned char *rows = rb + 16;
#pragma unroll
            for (int i = lane; i < kChannels * W::CPR; i += 32) {
                const int r = i / W::CPR, c = i % W::CPR;
                const int64_t t = t0 + c * W::V;
                const bool ok = r < nrows && t < L;
                const int64_t off = ok ? row0 + r * L + t : 0;
                cp16(rows + (W::ROW_U + r) * W::ROWB + c * 16, gu + off, ok);
                cp16(rows + (W::ROW_D + r) * W::ROWB + c * 16, gd + off, ok);
                if (gz) cp16(rows + (W::ROW_Z + r) * W::ROWB + c * 16, gz + off, ok);
            }
#pragma unroll
            for (int i = lane; i < 2 * kNS * W::CPR; i += 32) {
                const int which = i / (kNS * W::CPR), rem = i % (kNS * W::CPR);
                const int n = rem / W::CPR, c = rem % W::CPR;
                const int64_t t = t0 + c * W::V;
                const bool ok = n < p.dstate && t < L;
                const int64_t off = ok ? bc0 + (int64_t)n * L + t : 0;
                cp16(rows + (W::ROW_B + which * kNS + n) * W::ROWB + c * 16, (which ? gC : gB) + off, ok);
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
        const unsigned char *rows = raw(k) + 16;
        const int g = (int)(d.unit % (unsigned)p.n_groups);
        const int64_t d0 = (int64_t)(g % p.groups_per_batch) * kChannels;
        const int64_t dc = d0 + lane;
        const float bias = (dc < p.dim && p.delta_bias) ? __ldg(p.delta_bias + dc) : 0.f;
        float fu[kTC], fd[kTC];
        unpack_row<T>(rows + (W::ROW_U + lane) * W::ROWB, fu);
        unpack_row<T>(rows + (W::ROW_D + lane) * W::ROWB, fd);
        unsigned char *dl = pb + W::DL_OFF + lane * W::DLB;
#pragma unroll
        for (int t = 0; t < kTC; t += 2) {
            float2 x = __fadd2_rn(f2(fd[t], fd[t + 1]), f2(bias, bias));
            if (SP) x = softplus2_f(x);
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
        const unsigned char *rows = raw(k) + 16;
        const unsigned char *pb = proc(k);
        const int g = (int)(d.unit % (unsigned)p.n_groups);
        const int j = (int)(d.unit / (unsigned)p.n_groups);
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (int64_t)(g % p.groups_per_batch) * kChannels;
        const int64_t dc = d0 + lane;
        if (dc >= p.dim) return;
        const float Dd = p.D ? __ldg(p.D + dc) : 0.f;
        float fu[kTC], fz[kTC], y[kTC];
        unpack_row<T>(rows + (W::ROW_U + lane) * W::ROWB, fu);
        if (GATE) unpack_row<T>(rows + (W::ROW_Z + lane) * W::ROWB, fz);
        const float4 *yr = reinterpret_cast<const float4 *>(pb + W::Y_OFF + lane * W::YB);
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
        T *gout = static_cast<T *>(p.out);
        const int64_t t0 = (int64_t)j * p.chunk_len + (int64_t)d.sub * kTC;
        T *dst = gout + (b * p.dim + dc) * p.seqlen + t0;
#pragma unroll
        for (int c = 0; c < W::CPR; ++c)
            if (c * W::V < d.tvalid) stg16_stream(dst + c * W::V, Elem<T>::pack(o + c * W::V));
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
        Helper<T> h(p, pair, lane);
        constexpr int NR = W::NRAW;
        // fill the pipeline: sub-chunks 0 .. NR-2 staged, 0 prepared
        for (int k = 0; k < NR - 1; ++k) h.issue(k, h.next());
        cp_wait<NR - 2>();
        __syncwarp();
        Desc dcur = *reinterpret_cast<const Desc *>(h.raw(0));
        h.template prologue<SP>(0, dcur);
        __syncwarp();
        if (lane == 0) mbar_arrive(full + 0);
        bool ok = true;
        Desc dprev{0u, 0, kSkip, 0};
        int k = 0;
        while (!(dcur.flags & kEnd)) {
            // the scan runs sub-chunk k; finish k-1, then prepare k+1
            if (k >= 1) {
                if (!mbar_wait(done + ((k - 1) & 1), ((k - 1) >> 1) & 1, err)) { ok = false; break; }
                h.template epilogue<GATE>(k - 1, dprev);
                __syncwarp();  // raw slot of k-1 is read before it is refilled
            }
            h.issue(k + NR - 1, h.next());
            cp_wait<NR - 2>();
            __syncwarp();
            const Desc dnext = *reinterpret_cast<const Desc *>(h.raw(k + 1));
            h.template prologue<SP>(k + 1, dnext);
            __syncwarp();
            if (lane == 0) mbar_arrive(full + ((k + 1) & 1));
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

    // ---- scan warp: lane = channel, all states in registers
    int cur_group = -1;
    float2 A2[kNS / 2];
    float2 hs[kNS / 2];
#pragma unroll
    for (int q = 0; q < kNS / 2; ++q) { A2[q] = f2(0.f, 0.f); hs[q] = f2(0.f, 0.f); }
    const int N = p.dstate;
    for (int k = 0;; ++k) {
        uint64_t *bar = full + (k & 1);
        if (!mbar_wait(bar, (k >> 1) & 1, err)) return;
        unsigned char *pb = pair + W::NRAW * W::RAW + (k & 1) * W::PROC;
        const Desc d = *reinterpret_cast<const Desc *>(pb);
        if (d.flags & kEnd) return;
        if (!(d.flags & kSkip)) {
            const int g = (int)(d.unit % (unsigned)p.n_groups);
            const int j = (int)(d.unit / (unsigned)p.n_groups);
            const int64_t b = g / p.groups_per_batch;
            const int64_t dc = (int64_t)(g % p.groups_per_batch) * kChannels + lane;
            float *carry = p.carry + ((int64_t)g * 32 + lane) * kNS;
            if (d.flags & kFirst) {
                if (g != cur_group) {
                    cur_group = g;
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q) {
                        const int n0 = 2 * q, n1 = 2 * q + 1;
                        const float a0 = (dc < p.dim && n0 < N) ? __ldg(p.A + dc * N + n0) : 0.f;
                        const float a1 = (dc < p.dim && n1 < N) ? __ldg(p.A + dc * N + n1) : 0.f;
                        A2[q] = f2(a0 * kLog2e, a1 * kLog2e);
                    }
                }
                if (j == 0) {
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q) hs[q] = f2(0.f, 0.f);
                } else {
#pragma unroll
                    for (int q = 0; q < kNS / 4; ++q) {
                        const float4 v = __ldcg(reinterpret_cast<const float4 *>(carry) + q);
                        hs[2 * q] = f2(v.x, v.y);
                        hs[2 * q + 1] = f2(v.z, v.w);
                    }
                }
            }
            const float4 *dlrow = reinterpret_cast<const float4 *>(pb + W::DL_OFF + lane * W::DLB);
            const float *sB = reinterpret_cast<const float *>(pb + W::BC_OFF);
            const float *sC = sB + kTC * kNS + 16;
            float4 *yrow = reinterpret_cast<float4 *>(pb + W::Y_OFF + lane * W::YB);
#pragma unroll 1
            for (int tb = 0; tb < kTC; tb += 8) {
                float4 dd[4];  // (delta_t, delta_t u_t, delta_t+1, delta_t+1 u_t+1)
#pragma unroll
                for (int i = 0; i < 4; ++i) dd[i] = dlrow[tb / 2 + i];
                float2 y2[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y2[e] = f2(0.f, 0.f);
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
                        const float2 a0 = f2(ex2_mufu(x0.x), ex2_mufu(x0.y));
                        // states 14 and 15 on the FMA pipe
                        const float2 a1 = q == kNS / 4 - 1 ? ex2_poly2(x1) : f2(ex2_mufu(x1.x), ex2_mufu(x1.y));
                        const float2 bu0 = __fmul2_rn(f2(du, du), f2(bb.x, bb.y));
                        const float2 bu1 = __fmul2_rn(f2(du, du), f2(bb.z, bb.w));
                        hs[2 * q] = __ffma2_rn(a0, hs[2 * q], bu0);
                        hs[2 * q + 1] = __ffma2_rn(a1, hs[2 * q + 1], bu1);
                        y2[e] = __ffma2_rn(f2(cc.x, cc.y), hs[2 * q], y2[e]);
                        y2[e] = __ffma2_rn(f2(cc.z, cc.w), hs[2 * q + 1], y2[e]);
                    }
                }
                yrow[tb / 4] = make_float4(y2[0].x + y2[0].y, y2[1].x + y2[1].y, y2[2].x + y2[2].y,
                                           y2[3].x + y2[3].y);
                yrow[tb / 4 + 1] = make_float4(y2[4].x + y2[4].y, y2[5].x + y2[5].y, y2[6].x + y2[6].y,
                                               y2[7].x + y2[7].y);
            }
            if (d.flags & kLast) {
                if (j + 1 < p.n_chunks) {
#pragma unroll
                    for (int q = 0; q < kNS / 4; ++q)
                        __stcg(reinterpret_cast<float4 *>(carry) + q,
                               make_float4(hs[2 * q].x, hs[2 * q].y, hs[2 * q + 1].x, hs[2 * q + 1].y));
                    push_unit(p, lane, (unsigned)((j + 1) * p.n_groups + g));
                } else if (p.last_state != nullptr && dc < p.dim) {
                    float *ls = p.last_state + (b * p.dim + dc) * N;
#pragma unroll
                    for (int q = 0; q < kNS / 2; ++q) {
                        if (2 * q < N) ls[2 * q] = hs[q].x;
                        if (2 * q + 1 < N) ls[2 * q + 1] = hs[q].y;
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
