// scan_fwd_persistent_pairs.cu -- persistent selective-scan (S6) forward
// with each channel's states split over R = 2 or 4 lanes.
//
// Computes softplus(delta + bias), the zero-order-hold decay exp(delta A),
// the diagonal recurrence, the C readout, the D skip and the silu gate ("Mamba
// SSM concept and implementation in Keras and TensorFlow", recurrent form and
// selective_scan / MambaBlock; fused as in the Mamba paper, Appendix E.5).
// Splitting the 16 states of a channel over R lanes multiplies the number of
// warps a problem provides -- e.g. 1280 instead of 640 for the Mamba-2.8B
// layer at R = 2 -- so every SM sub-partition runs two or more workers and one
// hides the other's dependency stalls; with one warp per sub-partition the
// MUFU idles whenever that warp is in a non-exp stretch.
//
// Work: the balanced split of persistent_common.cuh -- each warp runs a
// contiguous share of the (channel group, sub-chunk) grid, at most three
// pieces.  Two launch forms:
//   * device-wide (LOCAL = false): every resident warp of the device takes a
//     share of all groups; carried states pass between warps through the
//     caller's workspace (cooperative launch, blocks of kWarps warps);
//   * block-local (LOCAL = true): one block per SM of LocalWarps<R> warps
//     takes a contiguous range of whole groups and splits it among its own
//     warps, so carried states only pass between warps of one block, through
//     shared memory -- no workspace at all.
// Per piece, per sub-chunk of TC timesteps:
//   1. cp.async stages the raw u / delta / z rows and the B / C rows of the
//      next sub-chunk (double buffer) while this one is processed;
//   2. prologue: B and C are widened to fp32 as [t][n] rows for broadcast
//      reads; every element's delta = softplus(delta_raw + bias) and delta * u
//      are computed once (lane = channel & timestep slice) into shared
//      (delta, delta, delta u, delta u) quads;
//   3. scan: lane (channel c, slice r) advances states (16/R) r .. through
//      blocks of 8 timesteps (state pairs on FMUL2 / FFMA2, the decays on the
//      MUFU); the R slices' readouts are combined with transposed shuffle
//      rounds, leaving each lane 8/R consecutive complete outputs, which it
//      gates -- (y + D u) * silu(z) from the staged raw rows -- and packs into
//      the output tile;
//   4. the tile is written with coalesced 16-byte stores.
// Shared arrays are padded so that every quarter-warp access is free of bank
// conflicts.  fp32 activations take the accurate decay and softplus of
// device_math.cuh (Decay<true>) in place of the MUFU ones.
// Channel-last form (CL, block-local only): the activations of the Keras
// page's layout -- (batch, L, dim), B and C (batch, L, N) -- are staged a
// timestep row at a time (16-byte copies of a row's channels or states), the
// prologue lane takes one timestep's channels, and the epilogue reads and
// writes the transposed rows; steps 2 (the quads and fp32 B / C rows) and 3
// are unchanged, so the results equal the dense layout's bit for bit.
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

template <typename T, int R>
struct PairSmem {
    static constexpr int kTC = 64 / (int)sizeof(T);        // timesteps per sub-chunk (64-byte rows)
    static constexpr int V = 16 / (int)sizeof(T);          // elements per 16 bytes
    static constexpr int CPR = kTC / V;                    // 16-byte chunks per raw row
    static constexpr int CW = 32 / R;                      // channels per unit
    static constexpr int ROWB = kTC * (int)sizeof(T) + 16;  // raw / output row pitch (bytes)
    static constexpr int RAW_ROWS = 3 * CW + 2 * kNS;      // u, delta, z rows, then B, C rows
    static constexpr int STAGE = RAW_ROWS * ROWB;
    // fp32 B then C as [t][n] rows of 64 bytes; every V rows (one staged
    // 16-byte chunk of timesteps) are followed by 32 bytes of padding, which
    // makes the transposing 16-byte stores free of bank conflicts
    static constexpr int BLKB = V * kNS * 4 + 32;
    static constexpr int BARR = (kTC / V) * BLKB;          // one of B, C
    static constexpr int BC32 = 2 * BARR;
    static constexpr int QUADB = kTC * 16 + 16;             // float4 row pitch (bytes)
    static constexpr int DDU = CW * QUADB;                  // (delta, delta, delta*u, delta*u) [c][t]
    static constexpr int OUTB = CW * ROWB;                  // packed outputs [c][t]
    static constexpr int BYTES = 2 * STAGE + BC32 + DDU + OUTB;
};

template <typename T>
__device__ __forceinline__ void store4(unsigned char *dst, const float *o);
template <>
__device__ __forceinline__ void store4<float>(unsigned char *dst, const float *o) {
    *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(unsigned char *dst, const float *o) {
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(Elem<__nv_bfloat16>::pack2(o[0], o[1]), Elem<__nv_bfloat16>::pack2(o[2], o[3]));
}
template <typename T>
__device__ __forceinline__ void store2(unsigned char *dst, const float *o);
template <>
__device__ __forceinline__ void store2<float>(unsigned char *dst, const float *o) {
    *reinterpret_cast<float2 *>(dst) = make_float2(o[0], o[1]);
}
template <>
__device__ __forceinline__ void store2<__nv_bfloat16>(unsigned char *dst, const float *o) {
    *reinterpret_cast<uint32_t *>(dst) = Elem<__nv_bfloat16>::pack2(o[0], o[1]);
}

// OWN (2 or 4) consecutive activations from shared memory, widened to fp32.
template <typename T, int OWN>
__device__ __forceinline__ void load_small(const unsigned char *src, float *f);
template <>
__device__ __forceinline__ void load_small<float, 4>(const unsigned char *src, float *f) {
    const float4 v = *reinterpret_cast<const float4 *>(src);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load_small<float, 2>(const unsigned char *src, float *f) {
    const float2 v = *reinterpret_cast<const float2 *>(src);
    f[0] = v.x; f[1] = v.y;
}
template <>
__device__ __forceinline__ void load_small<__nv_bfloat16, 4>(const unsigned char *src, float *f) {
    const uint2 v = *reinterpret_cast<const uint2 *>(src);
    Elem<__nv_bfloat16>::unpack2(v.x, f[0], f[1]);
    Elem<__nv_bfloat16>::unpack2(v.y, f[2], f[3]);
}
template <>
__device__ __forceinline__ void load_small<__nv_bfloat16, 2>(const unsigned char *src, float *f) {
    Elem<__nv_bfloat16>::unpack2(*reinterpret_cast<const uint32_t *>(src), f[0], f[1]);
}

// Sum the 8 per-timestep partial readouts of a block over the R lanes of a
// channel, transposed: afterwards lane r holds the complete outputs of
// timesteps r * 8/R .. r * 8/R + 8/R - 1 in v[0 ..].  Round K halves the live
// values: the lane with bit K set keeps the upper half, sends the lower.
template <int K, int CNT>
struct LaneReduce {
    __device__ __forceinline__ static void run(float (&v)[8], int r) {
        constexpr int HALF = CNT / 2;
        const bool upper = (r & K) != 0;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
            const float send = upper ? v[i] : v[i + HALF];
            const float keep = upper ? v[i + HALF] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, K);
        }
        LaneReduce<K / 2, HALF>::run(v, r);
    }
};
template <int CNT>
struct LaneReduce<0, CNT> {
    __device__ __forceinline__ static void run(float (&)[8], int) {}
};

template <int R> struct LanesOccupancy;
template <> struct LanesOccupancy<2> { static constexpr int kBlocks = 2; };
template <> struct LanesOccupancy<4> { static constexpr int kBlocks = 3; };

// Block-local form: warps per block (one block per SM, the same warps per SM
// as the device-wide form's kBlocks x kWarps).
template <int R> struct LocalWarps;
template <> struct LocalWarps<2> { static constexpr int value = 8; };
template <> struct LocalWarps<4> { static constexpr int value = 12; };

template <int R, bool LOCAL>
struct PairLaunch {
    static constexpr int kWorkers = LOCAL ? LocalWarps<R>::value : kWarps;  // warps per block
    static constexpr int kMinBlocks = LOCAL ? 1 : LanesOccupancy<R>::kBlocks;
};

// Block-local carries: slot w holds what warp w hands on to the next warp
// with a non-empty share ([32 lanes][16 / R floats]), then one flag word per
// slot (the sub-chunk position the carry covers; 0 = not yet published) and
// the block's abort word (set by a warp whose wait ran out).
template <int R>
struct LocalSmem {
    static constexpr int SLOTS = LocalWarps<R>::value * 32 * (kNS / R) * 4;
    static constexpr int FLAGS = ((LocalWarps<R>::value + 1) * 4 + 15) / 16 * 16;
    static constexpr int BYTES = SLOTS + FLAGS;
};

// Set by a block-local launch whose bounded wait ran out (read and cleared by
// take_local_error).
__device__ unsigned g_local_error;

// Block-local wait (lane 0 polls the shared flag, bounded in time) until the
// warp before has published the carry covering sub-chunk position `pos`.  A
// wait that runs out raises the device error word and the block's abort
// word; every other waiter of the block then gives up at once.
__device__ __forceinline__ bool local_wait(volatile unsigned *flag, volatile unsigned *abort_word, int lane,
                                           unsigned pos) {
    unsigned ok = 1;
    if (lane == 0) {
        if (*flag != pos) {
            unsigned long long t0, t;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
            unsigned ns = 32;
            while (*flag != pos) {
                asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
                if (*abort_word != 0u) {
                    ok = 0;
                    break;
                }
                if (t - t0 > 2000000000ull) {
                    atomicOr(&g_local_error, 1u);
                    *abort_word = 1u;
                    ok = 0;
                    break;
                }
                __nanosleep(ns);
                if (ns < 1024) ns <<= 1;
            }
        }
        __threadfence_block();  // the slot's contents are read after the flag
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Block-local publish: every lane has written its part of the slot.
__device__ __forceinline__ void local_publish(volatile unsigned *flag, int lane, unsigned pos) {
    __syncwarp();
    if (lane == 0) {
        __threadfence_block();
        *flag = pos;
    }
}

template <typename T, int R, bool SP, bool GATE, bool CONV, bool LOCAL, bool CL, bool UNR>
__global__ void __launch_bounds__(PairLaunch<R, LOCAL>::kWorkers * 32, PairLaunch<R, LOCAL>::kMinBlocks)
scan_fwd_pairs_kernel(const Params p) {
    using W = PairSmem<T, R>;
    static_assert(!(CL && CONV), "the fused convolution reads the dense layout");
    static_assert(!UNR || R == 2 || (!CONV && !CL), "the unrolled form of four lanes: dense layout, no fused conv1d");
    constexpr int kWorkers = PairLaunch<R, LOCAL>::kWorkers;
    constexpr bool ACC = sizeof(T) == 4;
    using Dk = Decay<ACC>;
    // a lane's states as pairs: fp32 (packed x2 arithmetic) for bf16
    // activations, fp64 for fp32 ones (Decay's note says why)
    using HV = typename std::conditional<ACC, double2, float2>::type;
    auto hv = [](float a, float b) {
        HV r;
        r.x = a;
        r.y = b;
        return r;
    };
    constexpr int kTC = W::kTC, V = W::V, CPR = W::CPR, CW = W::CW;
    constexpr int S = kNS / R;   // states per lane
    constexpr int OWN = 8 / R;   // outputs per lane per block of 8 timesteps
    // blocks of 8 timesteps in flight (the fused conv1d's prologue, and the
    // register cap of 12 warps with four lanes, leave room for two)
    constexpr int kBlkUnroll = UNR ? ((CONV || R == 4) ? 2 : kTC / 8) : 1;
    constexpr int PT = kTC / R;  // prologue timesteps per lane
    // Channel-last staging (CL: (batch, L, dim) activations, (batch, L, N) B
    // and C).  A stage then holds, per activation tensor, kTC rows of one
    // timestep's CW channels (CH 16-byte chunks; chunk c of row t sits at
    // slot c ^ swz(t), so the 8 lanes of a quarter-warp that read one chunk
    // each from consecutive rows hit distinct banks), then B and C as kTC
    // rows of kNS states.  The prologue lane takes one timestep's channels
    // (LPT lanes per timestep) instead of one channel's timesteps; the scan
    // is unchanged, so results are bit-equal to the dense layout's.
    constexpr int CH = CW * (int)sizeof(T) / 16;   // 16-byte chunks per activation row
    constexpr int CROW = CH * 16;
    constexpr int BCH = kNS * (int)sizeof(T) / 16;  // chunks per B / C row
    constexpr int BROW = BCH * 16;
    constexpr int LPT = 32 / kTC;                   // prologue lanes per timestep
    constexpr int CL_ACT = 3 * kTC * CROW;          // B / C rows start here
    constexpr int CL_BIAS = W::STAGE - CW * 4;      // stage 0's tail: the group's biases (fp32)
    static_assert(!CL || (CL_ACT + 2 * kTC * BROW <= CL_BIAS && kTC * CROW <= W::OUTB), "channel-last stage");
    auto swz = [](int t) { return (t / (8 / CH)) & (CH - 1); };
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    unsigned char *base = smem + warp * W::BYTES;
    float *bc32 = reinterpret_cast<float *>(base + 2 * W::STAGE);
    unsigned char *ddu = base + 2 * W::STAGE + W::BC32;
    unsigned char *outt = ddu + W::DDU;

    const int64_t L = p.seqlen, Dm = p.dim;
    const int N = p.dstate;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B);
    const T *gC = static_cast<const T *>(p.C);
    T *gout = static_cast<T *>(p.out);

    // block-local carry slots and flags, after the warps' areas
    float *lslots = reinterpret_cast<float *>(smem + kWorkers * W::BYTES);
    volatile unsigned *lflags = reinterpret_cast<volatile unsigned *>(smem + kWorkers * W::BYTES + LocalSmem<R>::SLOTS);
    if (LOCAL) {  // slot flags, then the abort word
        for (int i = threadIdx.x; i <= kWorkers; i += blockDim.x) lflags[i] = 0u;
        __syncthreads();
    }

    const int sc = lane / R, sr = lane % R;    // scan: channel, state slice
    const int pc = lane % CW, ph = lane / CW;  // prologue: channel, timestep slice

    int cur_group = -1;
    float2 A2[S / 2];
    float bias_p = 0.f, D_s = 0.f;
    float cw[4] = {0.f, 0.f, 0.f, 0.f}, cb_p = 0.f;  // CONV: the prologue channel's conv taps and bias

    // This worker's share of the balanced split: head, whole groups, tail.
    // Piece: sub-chunks [sb, se) of group g, carried state in from sub-chunk
    // sb and out at se (or the final state when se is the group's end).
    long long n_workers, scope_groups;
    Range rg;
    int producer = warp - 1;  // LOCAL: the warp whose share ends where this one's starts
    if (LOCAL) {  // this block's whole groups [gb, ge), split among its warps
        const long long G = p.n_groups, nb = gridDim.x;
        const int gb = (int)((long long)blockIdx.x * G / nb);
        const int ge = (int)(((long long)blockIdx.x + 1) * G / nb);
        n_workers = kWorkers;
        scope_groups = ge - gb;
        rg = worker_range_of(scope_groups, p.subs_per_chain, gb, warp, n_workers);
        // with fewer sub-chunks than warps some shares are empty: skip them
        const long long T = scope_groups * (long long)p.subs_per_chain;
        while (producer > 0 && ((long long)producer + 1) * T / n_workers == (long long)producer * T / n_workers)
            --producer;
    } else {
        n_workers = (long long)gridDim.x * kWarps;
        scope_groups = p.n_groups;
        rg = worker_range(p, (long long)blockIdx.x * kWarps + warp, n_workers);
    }
    // Shares shorter than ~0.55 of a group: waiting for the piece before
    // would chain a group's pieces end to end (the group's full length); the
    // two-phase pieces below cost ~1.8x their length but all run at once.
    const bool two_phase = 20LL * scope_groups < 11LL * n_workers;
    const int has_head = rg.head.se > 0 ? 1 : 0;
    const int n_pieces = has_head + (rg.full_e - rg.full_b) + (rg.tail.se > 0 ? 1 : 0);
#pragma unroll 1
    for (int pi = 0; pi < n_pieces; ++pi) {
        int g, sb, se;
        if (pi < has_head) {
            g = rg.head.g; sb = 0; se = rg.head.se;
        } else if (pi - has_head < rg.full_e - rg.full_b) {
            g = rg.full_b + (pi - has_head); sb = 0; se = p.subs_per_chain;
        } else {
            g = rg.tail.g; sb = rg.tail.sb; se = rg.tail.se;
        }
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (int64_t)(g % p.groups_per_batch) * CW;
        const int nrows = (Dm - d0) < CW ? (int)(Dm - d0) : CW;
        const int64_t ds = d0 + sc, dp = d0 + pc;

        if (g != cur_group) {
            cur_group = g;
#pragma unroll
            for (int k = 0; k < S / 2; ++k) {
                const int n0 = S * sr + 2 * k, n1 = n0 + 1;
                const float a0 = (ds < Dm && n0 < N && MSCAN_WITHIN(p.x_A, p.A + ds * N + n0, 4, kSiteA))
                                     ? __ldg(p.A + ds * N + n0) : 0.f;
                const float a1 = (ds < Dm && n1 < N && MSCAN_WITHIN(p.x_A, p.A + ds * N + n1, 4, kSiteA))
                                     ? __ldg(p.A + ds * N + n1) : 0.f;
                A2[k] = make_float2(a0 * Dk::kScale, a1 * Dk::kScale);
            }
            bias_p = (dp < Dm && p.delta_bias && MSCAN_WITHIN(p.x_bias, p.delta_bias + dp, 4, kSiteBias))
                         ? __ldg(p.delta_bias + dp) : 0.f;
            if (CL && lane < CW) {  // the prologue lane of a timestep needs every channel's bias
                float *sbias = reinterpret_cast<float *>(base + CL_BIAS);
                sbias[lane] = (d0 + lane < Dm && p.delta_bias &&
                               MSCAN_WITHIN(p.x_bias, p.delta_bias + d0 + lane, 4, kSiteBias))
                                  ? __ldg(p.delta_bias + d0 + lane) : 0.f;
            }
            D_s = (ds < Dm && p.D && MSCAN_WITHIN(p.x_D, p.D + ds, 4, kSiteD)) ? __ldg(p.D + ds) : 0.f;
            if (CONV) {  // taps right-aligned to 4: a shorter kernel sees zeros before it
                const int K = p.conv_k;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    cw[j] = (dp < Dm && j >= 4 - K &&
                             MSCAN_WITHIN(p.x_conv_w, p.conv_w + dp * K + (j - (4 - K)), 4, kSiteConvW))
                                ? __ldg(p.conv_w + dp * K + (j - (4 - K))) : 0.f;
                cb_p = (dp < Dm && p.conv_b && MSCAN_WITHIN(p.x_conv_b, p.conv_b + dp, 4, kSiteConvB))
                           ? __ldg(p.conv_b + dp) : 0.f;
            }
        }

        // the carried state in (from the worker before) and out (to the one
        // after): the group's workspace slot, or this block's shared slots
        float *carry_in = LOCAL ? lslots + ((int64_t)(producer > 0 ? producer : 0) * 32 + lane) * S
                                : p.carry + ((int64_t)g * 32 + lane) * S;
        float *carry_out = LOCAL ? lslots + ((int64_t)warp * 32 + lane) * S : carry_in;
        auto load_carry = [&](HV (&hh)[S / 2]) {
#pragma unroll
            for (int k = 0; k < S / 4; ++k) {
                const float4 v = LOCAL ? reinterpret_cast<const float4 *>(carry_in)[k]
                                 : MSCAN_WITHIN(p.x_carry, reinterpret_cast<const float4 *>(carry_in) + k, 16, kSiteCarry)
                                       ? __ldcg(reinterpret_cast<const float4 *>(carry_in) + k)  // S/4 float4
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                hh[2 * k] = hv(v.x, v.y);
                hh[2 * k + 1] = hv(v.z, v.w);
            }
        };
        auto store_carry = [&](const HV (&hh)[S / 2]) {
#pragma unroll
            for (int k = 0; k < S / 4; ++k) {
                const float4 v = make_float4((float)hh[2 * k].x, (float)hh[2 * k].y, (float)hh[2 * k + 1].x,
                                             (float)hh[2 * k + 1].y);
                if (LOCAL) reinterpret_cast<float4 *>(carry_out)[k] = v;
                else if (MSCAN_WITHIN(p.x_carry, reinterpret_cast<float4 *>(carry_out) + k, 16, kSiteCarry))
                    __stcg(reinterpret_cast<float4 *>(carry_out) + k, v);
            }
        };
        auto wait_carry = [&](int pos) {
            if (LOCAL) return local_wait(lflags + (producer > 0 ? producer : 0), lflags + kWorkers, lane, (unsigned)pos);
            return wait_progress(p, lane, g, pos);
        };
        auto publish_carry = [&](int pos) {
            if (g == p.stall_group) return;  // test hook: the next piece's wait runs out
            if (LOCAL) local_publish(lflags + warp, lane, (unsigned)pos);
            else publish_progress(p, lane, g, pos);
        };

        const int64_t tb0 = (int64_t)sb * kTC;
        const int nsub = se - sb;
        const int64_t row0 = (b * Dm + d0) * L;
        const int64_t bc0 = b * (int64_t)N * L;

        // this lane's 16-byte copies: chunk cx of rows (lane + 32 i) / CPR
        constexpr int NX = (CW * CPR + 31) / 32, NB = 2 * kNS * CPR / 32;
        const int cx = lane % CPR;
        int64_t xoff[NX], boff[NB], uoff[NX], zoff[NX];
        bool xok[NX], bok[NB];
#pragma unroll
        for (int i = 0; i < NX; ++i) {
            const int r = (lane + 32 * i) / CPR;
            xok[i] = lane + 32 * i < CW * CPR && r < nrows;
            xoff[i] = row0 + r * L + cx * V;
            uoff[i] = CONV ? b * p.u_bstride + (d0 + r) * L + cx * V : xoff[i];
            zoff[i] = CONV ? b * p.z_bstride + (d0 + r) * L + cx * V : xoff[i];
        }
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            const int n = ((lane + 32 * i) % (kNS * CPR)) / CPR;
            bok[i] = n < N;
            boff[i] = bc0 + (int64_t)n * L + cx * V;
        }
        // channel-last copies: chunk q = lane + 32 i of the activation tile is
        // (row t = q / CH, chunk c = q % CH); of the B / C tile (which, t, c)
        constexpr int NXC = kTC * CH / 32 > 0 ? kTC * CH / 32 : 1, NBC = 2 * kTC * BCH / 32;
        static_assert(!CL || (NXC * 32 == kTC * CH && NBC * 32 == 2 * kTC * BCH), "channel-last copy split");
        int64_t cxoff[NXC], cboff[NBC];
        bool cxok[NXC], cbok[NBC];
        if (CL) {
#pragma unroll
            for (int i = 0; i < NXC; ++i) {
                const int q = lane + 32 * i, t = q / CH, c = q % CH;
                cxok[i] = d0 + c * V < Dm;
                cxoff[i] = (b * L + t) * Dm + d0 + c * V;
            }
#pragma unroll
            for (int i = 0; i < NBC; ++i) {
                const int q = lane + 32 * i, t = (q / BCH) % kTC, c = q % BCH;
                cbok[i] = c * V < N;
                cboff[i] = (b * L + t) * (int64_t)N + c * V;
            }
        }
        bool so_stage = false;  // state-only run: no z or C rows to stage
        auto issue = [&](int sub, int st) {
            if (CL) {
                unsigned char *sb0 = base + st * W::STAGE;
                const int64_t t0 = tb0 + (int64_t)sub * kTC;
#pragma unroll
                for (int i = 0; i < NXC; ++i) {
                    const int q = lane + 32 * i, t = q / CH, c = q % CH;
                    const bool ok = cxok[i] && t0 + t < L;
                    const int64_t off = ok ? cxoff[i] + t0 * Dm : 0;
                    unsigned char *dst = sb0 + t * CROW + ((c ^ swz(t)) * 16);
                    cp16(dst, gu + off, ok && MSCAN_WITHIN(p.x_u, gu + off, 16, kSiteU));
                    cp16(dst + kTC * CROW, gd + off, ok && MSCAN_WITHIN(p.x_delta, gd + off, 16, kSiteDelta));
                    if (GATE && !so_stage)
                        cp16(dst + 2 * kTC * CROW, gz + off, ok && MSCAN_WITHIN(p.x_z, gz + off, 16, kSiteZ));
                }
#pragma unroll
                for (int i = 0; i < NBC; ++i) {
                    const int q = lane + 32 * i, which = q / (kTC * BCH), t = (q / BCH) % kTC, c = q % BCH;
                    const bool ok = cbok[i] && t0 + t < L;
                    const int64_t off = ok ? cboff[i] + t0 * N : 0;
                    if (!(so_stage && which))
                        cp16(sb0 + CL_ACT + which * kTC * BROW + t * BROW + c * 16, (which ? gC : gB) + off,
                             ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, (which ? gC : gB) + off, 16, which ? kSiteC : kSiteB));
                }
                cp_commit();
                return;
            }
            unsigned char *sbuf = base + st * W::STAGE + cx * 16;
            const int64_t t0 = tb0 + (int64_t)sub * kTC;
            const bool tok = t0 + cx * V < L;
#pragma unroll
            for (int i = 0; i < NX; ++i) {
                const int r = (lane + 32 * i) / CPR;
                if (lane + 32 * i < CW * CPR) {
                    const bool ok = xok[i] && tok;
                    const int64_t off = ok ? xoff[i] + t0 : 0;
                    const T *su = gu + (ok ? uoff[i] + t0 : 0), *sz = gz + (ok ? zoff[i] + t0 : 0);
                    cp16(sbuf + (0 * CW + r) * W::ROWB, su, ok && MSCAN_WITHIN(p.x_u, su, 16, kSiteU));
                    cp16(sbuf + (1 * CW + r) * W::ROWB, gd + off, ok && MSCAN_WITHIN(p.x_delta, gd + off, 16, kSiteDelta));
                    if (GATE && !so_stage)
                        cp16(sbuf + (2 * CW + r) * W::ROWB, sz, ok && MSCAN_WITHIN(p.x_z, sz, 16, kSiteZ));
                }
            }
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int which = (lane + 32 * i) / (kNS * CPR);
                const int n = ((lane + 32 * i) % (kNS * CPR)) / CPR;
                const bool ok = bok[i] && tok;
                const int64_t off = ok ? boff[i] + t0 : 0;
                if (!(so_stage && which))
                    cp16(sbuf + (3 * CW + which * kNS + n) * W::ROWB, (which ? gC : gB) + off,
                         ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, (which ? gC : gB) + off, 16, which ? kSiteC : kSiteB));
            }
            cp_commit();
        };

        // The piece's sub-chunks.  State-only (SO) runs do the recurrence alone
        // -- no C rows, readout, gate or stores -- and sum delta into dsum;
        // full runs publish the carried state at the end when `publish_end`.
        auto run_subs = [&](const bool SO, HV (&h)[S / 2], double &dsum, bool publish_end) {
        so_stage = SO;
        issue(0, 0);
        if (CONV && ph == 0) {
            // the conv inputs before sub-chunk 0 (zeros before the sequence),
            // kept in the padding of the channel's x row of stage 0
            T *halo = reinterpret_cast<T *>(base + (0 * CW + pc) * W::ROWB + kTC * sizeof(T));
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                const int64_t t = tb0 - 3 + k;
                const T *src = gu + b * p.u_bstride + (d0 + pc) * L + t;
                halo[k] = (t >= 0 && pc < nrows && MSCAN_WITHIN(p.x_u, src, sizeof(T), kSiteHalo)) ? *src : T(0.f);
            }
        }
#pragma unroll 1
        for (int sub = 0; sub < nsub; ++sub) {
            const int st = sub & 1;
            if (sub + 1 < nsub) {
                issue(sub + 1, st ^ 1);
                cp_wait<1>();
            } else {
                cp_wait<0>();
            }
            __syncwarp();
            const unsigned char *sbuf = base + st * W::STAGE;
            const int64_t t0 = tb0 + (int64_t)sub * kTC;
            const int tvalid = (L - t0) < kTC ? (int)(L - t0) : kTC;
            // checkpoint for the backward pass: the state entering every 32nd step
            if (!SO && p.ckpt != nullptr && (t0 & 31) == 0 && ds < Dm &&
                MSCAN_WITHIN(p.x_ckpt,
                       p.ckpt + (((b * p.ckpt_gpb + (ds >> 5)) * p.ckpt_nsup + (t0 >> 5)) * 32 + (ds & 31)) * 16 + S * sr,
                       S * 4, kSiteCkpt)) {
                float *dst = p.ckpt + (((b * p.ckpt_gpb + (ds >> 5)) * p.ckpt_nsup + (t0 >> 5)) * 32 + (ds & 31)) * 16 +
                             S * sr;
#pragma unroll
                for (int k = 0; k < S / 4; ++k)
                    __stcg(reinterpret_cast<float4 *>(dst) + k,
                           make_float4((float)h[2 * k].x, (float)h[2 * k].y, (float)h[2 * k + 1].x,
                                       (float)h[2 * k + 1].y));
            }

            // ---- prologue (0), fused conv1d: this lane's PT inputs of its
            // channel and the 3 before them (from the row, or from the
            // padding where the previous sub-chunk left its last 3) become
            // u = silu(conv_b + sum_k w_k x), rounded to the activation type
            // and written over the inputs, so everything below reads u
            if (CONV) {
                unsigned char *urw = base + st * W::STAGE + (0 * CW + pc) * W::ROWB;
                float xs[PT + 3];
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    xs[k] = Elem<T>::to_f(ph == 0 ? reinterpret_cast<const T *>(urw + kTC * sizeof(T))[k]
                                                  : reinterpret_cast<const T *>(urw)[ph * PT - 3 + k]);
#pragma unroll
                for (int v = 0; v < PT; v += V)
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(urw + (ph * PT + v) * sizeof(T)), xs + 3 + v);
                __syncwarp();  // every lane holds its inputs before any u is written over them
                if (ph == R - 1) {  // the next sub-chunk's 3 inputs before it
                    T *nh = reinterpret_cast<T *>(base + (st ^ 1) * W::STAGE + (0 * CW + pc) * W::ROWB + kTC * sizeof(T));
#pragma unroll
                    for (int k = 0; k < 3; ++k) Elem<T>::store(nh + k, xs[PT + k]);
                }
#pragma unroll
                for (int v = 0; v < PT; v += V) {
                    float uo[V];
#pragma unroll
                    for (int e = 0; e < V; e += 2) {  // the conv1d kernel's arithmetic, pair for pair
                        float2 acc = f2(cb_p, cb_p);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            acc = __ffma2_rn(f2(cw[k], cw[k]), f2(xs[v + e + k], xs[v + e + 1 + k]), acc);
                        acc = silu2_f(acc);
                        uo[e] = acc.x;
                        uo[e + 1] = acc.y;
                    }
                    *reinterpret_cast<uint4 *>(urw + (ph * PT + v) * sizeof(T)) = Elem<T>::pack(uo);
                }
            }
            // ---- prologue (a): B and C to fp32 [t][n].  Lane (which, q, c)
            // reads states 4q .. 4q+3 of B (which 0) or C (which 1) in chunk c
            // and writes them back as one 16-byte [t][4q .. 4q+3] piece per
            // timestep
            if (CL) {  // B and C rows are [t][n] already: widen to fp32
#pragma unroll
                for (int i = 0; i < NBC; ++i) {
                    const int q = lane + 32 * i, which = q / (kTC * BCH), t = (q / BCH) % kTC, c = q % BCH;
                    if (SO && which) continue;
                    float f[V];
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(sbuf + CL_ACT + which * kTC * BROW + t * BROW + c * 16), f);
                    float *dst = bc32 + which * (W::BARR / 4) + (t / V) * (W::BLKB / 4) + (t % V) * kNS + c * V;
#pragma unroll
                    for (int k = 0; k < V; k += 4)
                        *reinterpret_cast<float4 *>(dst + k) = make_float4(f[k], f[k + 1], f[k + 2], f[k + 3]);
                }
            } else if (!SO || lane < 16) {  // C rows only feed the readout
                static_assert(CPR == 4, "four chunks of timesteps per sub-chunk");
                const int which = lane >> 4, q = (lane >> 2) & 3, c = lane & 3;
                float f[4][V];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(
                                        sbuf + (3 * CW + which * kNS + 4 * q + k) * W::ROWB + c * 16), f[k]);
                unsigned char *dst = reinterpret_cast<unsigned char *>(bc32) + which * W::BARR + c * W::BLKB + 16 * q;
#pragma unroll
                for (int e = 0; e < V; ++e)
                    *reinterpret_cast<float4 *>(dst + e * kNS * 4) = make_float4(f[0][e], f[1][e], f[2][e], f[3][e]);
            }
            // ---- prologue (b): per element, once: delta and delta*u, stored
            // duplicated as (delta, delta, delta*u, delta*u) so the scan reads
            // both packed operand pairs with one 16-byte load
            if (CL) {  // lane: timestep t, channel chunks h * CH / LPT ..
                const int t = lane / LPT, h = lane % LPT;
                const float *sbias = reinterpret_cast<const float *>(base + CL_BIAS);
#pragma unroll
                for (int j = 0; j < CH / LPT; ++j) {
                    const int c = h * (CH / LPT) + j;
                    const unsigned char *src = sbuf + t * CROW + ((c ^ swz(t)) * 16);
                    float fu[V], fd[V], fb[V];
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(src), fu);
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(src + kTC * CROW), fd);
#pragma unroll
                    for (int e = 0; e < V; e += 4) {
                        const float4 b4 = *reinterpret_cast<const float4 *>(sbias + c * V + e);
                        fb[e] = b4.x; fb[e + 1] = b4.y; fb[e + 2] = b4.z; fb[e + 3] = b4.w;
                    }
#pragma unroll
                    for (int e = 0; e < V; e += 2) {  // channel pairs on the packed x2 instructions
                        const int ch = c * V + e;
                        float2 x = __fadd2_rn(f2(fd[e], fd[e + 1]), f2(fb[e], fb[e + 1]));
                        if (SP) x = Dk::softplus2(x);
                        if (t >= tvalid) x = f2(0.f, 0.f);  // past the end: Abar = 1, no input
                        const float2 xu = __fmul2_rn(x, f2(fu[e], fu[e + 1]));
                        *reinterpret_cast<float4 *>(ddu + ch * W::QUADB + t * 16) = make_float4(x.x, x.x, xu.x, xu.x);
                        *reinterpret_cast<float4 *>(ddu + (ch + 1) * W::QUADB + t * 16) =
                            make_float4(x.y, x.y, xu.y, xu.y);
                    }
                }
            }
#pragma unroll
            for (int v = 0; v < (CL ? 0 : PT); v += V) {
                const int tt = ph * PT + v;
                float fu[V], fd[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(sbuf + (0 * CW + pc) * W::ROWB + tt * sizeof(T)), fu);
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(sbuf + (1 * CW + pc) * W::ROWB + tt * sizeof(T)), fd);
                float4 *dd = reinterpret_cast<float4 *>(ddu + pc * W::QUADB + tt * 16);
#pragma unroll
                for (int e = 0; e < V; e += 2) {  // element pairs on the packed x2 instructions
                    float2 x = __fadd2_rn(f2(fd[e], fd[e + 1]), f2(bias_p, bias_p));
                    if (SP) x = Dk::softplus2(x);
                    if (tvalid < kTC) {  // past the end: Abar = 1, no input
                        x.x = (tt + e < tvalid) ? x.x : 0.f;
                        x.y = (tt + e + 1 < tvalid) ? x.y : 0.f;
                    }
                    const float2 xu = __fmul2_rn(x, f2(fu[e], fu[e + 1]));
                    dd[e] = make_float4(x.x, x.x, xu.x, xu.x);
                    dd[e + 1] = make_float4(x.y, x.y, xu.y, xu.y);
                }
            }
            __syncwarp();
            if (CONV && !SO && p.u_out) {  // the u it formed, for a backward pass
                T *gu_out = static_cast<T *>(p.u_out);
#pragma unroll
                for (int i = lane; i < CW * CPR; i += 32) {
                    const int r = i / CPR, c = i % CPR;
                    const int64_t t = t0 + c * V;
                    if (r < nrows && t < L && MSCAN_WITHIN(p.x_u_out, gu_out + row0 + r * L + t, 16, kSiteUOut))
                        stg16_stream(gu_out + row0 + r * L + t, *reinterpret_cast<const uint4 *>(sbuf + (0 * CW + r) * W::ROWB + c * 16));
                }
            }

            // ---- scan: lane (sc, sr), blocks of 8 timesteps
            {
                const unsigned char *drow = ddu + sc * W::QUADB;
                const unsigned char *urow = sbuf + (0 * CW + sc) * W::ROWB;
                const unsigned char *zrow = sbuf + (2 * CW + sc) * W::ROWB;
                unsigned char *orow = outt + sc * W::ROWB;
                const float *sB0 = bc32 + S * sr;
                // UNR: the sub-chunk's blocks unrolled, so one block's readout,
                // combine and epilogue overlap the next one's decays (Mamba-2.8B
                // layer 527 -> 510 us, same results).  Launched only where no
                // piece is two-phase: with warps running state-only and full
                // pieces side by side it is slower (long context 6.5 -> 6.8 ms
                // block-local, 5.8 -> 6.7 ms device-wide); four lanes per
                // channel would spill.
#pragma unroll kBlkUnroll
                for (int tb = 0; tb < kTC; tb += 8) {
                    const float *sB = sB0 + (tb / V) * (W::BLKB / 4);
                    const float *sC = sB + W::BARR / 4;
                    float4 dq[8];  // (delta, delta, delta*u, delta*u) per timestep
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dq[e] = *reinterpret_cast<const float4 *>(drow + (tb + e) * 16);
                    if (SO) {
                        float s8 = 0.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) s8 += dq[e].x;
                        dsum += (double)s8;
                    }
                    float2 y2[8];  // readout partial sums: packed fp32 pairs, or
                    double yd[8];  // fp64 with fp32 activations
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        y2[e] = make_float2(0.f, 0.f);
                        yd[e] = 0.0;
                    }
                    // timestep-major: every timestep advances all of the lane's
                    // state pairs, so the compiler interleaves S / 2 independent
                    // chains (1.5 % faster than state-major, same operations)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
#pragma unroll
                        for (int q = 0; q < S / 4; ++q) {
                            const int to = (e / V) * (W::BLKB / 4) + (e % V) * kNS + 4 * q;
                            const float4 bb = *reinterpret_cast<const float4 *>(sB + to);
                            const float2 dl2 = make_float2(dq[e].x, dq[e].y);
                            const float2 du2 = make_float2(dq[e].z, dq[e].w);
                            const float2 x0 = __fmul2_rn(dl2, A2[2 * q]);
                            const float2 x1 = __fmul2_rn(dl2, A2[2 * q + 1]);
                            const float2 bu0 = __fmul2_rn(du2, make_float2(bb.x, bb.y));
                            const float2 bu1 = __fmul2_rn(du2, make_float2(bb.z, bb.w));
                            if constexpr (ACC) {
                                h[2 * q].x = Dk::step(x0.x, h[2 * q].x, bu0.x);
                                h[2 * q].y = Dk::step(x0.y, h[2 * q].y, bu0.y);
                                h[2 * q + 1].x = Dk::step(x1.x, h[2 * q + 1].x, bu1.x);
                                h[2 * q + 1].y = Dk::step(x1.y, h[2 * q + 1].y, bu1.y);
                                if (!SO) {
                                    const float4 cc = *reinterpret_cast<const float4 *>(sC + to);
                                    yd[e] = fma((double)cc.x, h[2 * q].x, yd[e]);
                                    yd[e] = fma((double)cc.y, h[2 * q].y, yd[e]);
                                    yd[e] = fma((double)cc.z, h[2 * q + 1].x, yd[e]);
                                    yd[e] = fma((double)cc.w, h[2 * q + 1].y, yd[e]);
                                }
                            } else {
                                const float2 a0 = make_float2(ex2_mufu(x0.x), ex2_mufu(x0.y));
                                // state-only runs lean harder on the MUFU (no readout or
                                // gate work beside it): one decay pair in eight goes
                                // to the FMA-pipe exp2 there
                                float2 a1;
                                if (SO && q == S / 4 - 1 && (e & 1) == 0) a1 = ex2_poly2(x1);
                                else a1 = make_float2(ex2_mufu(x1.x), ex2_mufu(x1.y));
                                h[2 * q] = __ffma2_rn(a0, h[2 * q], bu0);
                                h[2 * q + 1] = __ffma2_rn(a1, h[2 * q + 1], bu1);
                                if (!SO) {
                                    const float4 cc = *reinterpret_cast<const float4 *>(sC + to);
                                    y2[e] = __ffma2_rn(make_float2(cc.x, cc.y), h[2 * q], y2[e]);
                                    y2[e] = __ffma2_rn(make_float2(cc.z, cc.w), h[2 * q + 1], y2[e]);
                                }
                            }
                        }
                    }
                    if (SO) continue;
                    // combine the R slices, transposed: lane sr ends with the
                    // complete outputs of timesteps tb + OWN sr .. + OWN - 1
                    float yv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) yv[e] = ACC ? (float)yd[e] : y2[e].x + y2[e].y;
                    LaneReduce<R / 2, 8>::run(yv, sr);
                    // epilogue of this lane's outputs: out = (y + D u) * silu(z),
                    // u and z read from the staged raw rows
                    const int te = tb + OWN * sr;
                    float fu[OWN], fz[OWN], o[OWN];
                    // channel-last: rows te .. share one swizzle when its period
                    // is a multiple of OWN rows (te is a multiple of OWN)
                    constexpr bool kOneSlot = (8 / CH) % OWN == 0;
                    const int slot0 = (sc / V) ^ swz(te);
                    if (CL) {  // channel sc of rows te ..
#pragma unroll
                        for (int i = 0; i < OWN; ++i) {
                            const int slot = kOneSlot ? slot0 : (sc / V) ^ swz(te + i);
                            const unsigned char *src = sbuf + (te + i) * CROW + slot * 16 + (sc % V) * (int)sizeof(T);
                            fu[i] = Elem<T>::to_f(*reinterpret_cast<const T *>(src));
                            if (GATE) fz[i] = Elem<T>::to_f(*reinterpret_cast<const T *>(src + 2 * kTC * CROW));
                        }
                    } else {
                        load_small<T, OWN>(urow + te * sizeof(T), fu);
                        if (GATE) load_small<T, OWN>(zrow + te * sizeof(T), fz);
                    }
#pragma unroll
                    for (int i = 0; i < OWN; i += 2) {
                        const float2 uu = f2(fu[i], fu[i + 1]);
                        const float2 yy = __ffma2_rn(f2(D_s, D_s), uu, f2(yv[i], yv[i + 1]));
                        const float2 oo = GATE ? __fmul2_rn(yy, silu2_f(f2(fz[i], fz[i + 1]))) : yy;
                        o[i] = oo.x;
                        o[i + 1] = oo.y;
                    }
                    if (CL) {
#pragma unroll
                        for (int i = 0; i < OWN; ++i) {
                            const int slot = kOneSlot ? slot0 : (sc / V) ^ swz(te + i);
                            Elem<T>::store(reinterpret_cast<T *>(outt + (te + i) * CROW + slot * 16 + (sc % V) * (int)sizeof(T)),
                                           o[i]);
                        }
                    } else if (OWN == 4) {
                        store4<T>(orow + te * sizeof(T), o);
                    } else {
                        store2<T>(orow + te * sizeof(T), o);
                    }
                }
            }
            __syncwarp();
            if (SO) continue;
            // the piece's last sub-chunk leaves the carried state: publish it
            // before this tile's stores, so the release waits on less
            if (publish_end && sub + 1 == nsub && se < p.subs_per_chain) {
                store_carry(h);
                publish_carry(se);
            }
            // ---- coalesced store of the output tile
            if (CL) {
#pragma unroll
                for (int i = 0; i < NXC; ++i) {
                    const int q = lane + 32 * i, t = q / CH, c = q % CH;
                    if (cxok[i] && t0 + t < L && MSCAN_WITHIN(p.x_out, gout + cxoff[i] + t0 * Dm, 16, kSiteOut))
                        stg16_stream(gout + cxoff[i] + t0 * Dm,
                                     *reinterpret_cast<const uint4 *>(outt + t * CROW + ((c ^ swz(t)) * 16)));
                }
            }
#pragma unroll
            for (int i = lane; i < (CL ? 0 : CW * CPR); i += 32) {
                const int r = i / CPR, c = i % CPR;
                const int64_t t = t0 + c * V;
                if (r < nrows && t < L && MSCAN_WITHIN(p.x_out, gout + row0 + r * L + t, 16, kSiteOut))
                    stg16_stream(gout + row0 + r * L + t,
                                 *reinterpret_cast<const uint4 *>(outt + r * W::ROWB + c * 16));
            }
            __syncwarp();
        }
        };

        // the state before sub-chunk 0: the initial state, or zeros
        auto load_h0 = [&](HV (&hh)[S / 2]) {
#pragma unroll
            for (int k = 0; k < S / 2; ++k) {
                const int n0 = S * sr + 2 * k;
                const float *src = p.h0 + (b * Dm + ds) * N;
                hh[k] = (p.h0 && ds < Dm)
                            ? hv((n0 < N && MSCAN_WITHIN(p.x_h0, src + n0, 4, kSiteH0)) ? __ldcg(src + n0) : 0.f,
                                 (n0 + 1 < N && MSCAN_WITHIN(p.x_h0, src + n0 + 1, 4, kSiteH0)) ? __ldcg(src + n0 + 1) : 0.f)
                                          : hv(0.f, 0.f);
            }
        };
        HV h[S / 2];
#pragma unroll
        for (int k = 0; k < S / 2; ++k) h[k] = hv(0.f, 0.f);
        double dsum = 0.0;
        if ((two_phase && se < p.subs_per_chain) || p.state_only) {
            // The piece ends inside its group and other workers' pieces of the
            // group wait for its end state.  Get that state first with a
            // state-only run from a zero start, while the worker before it is
            // still busy; then, with that worker's carry h_in (none when the
            // piece starts the group): end = exp(A sum(delta)) h_in + local
            // end, published at once.  The pieces of a group thus finish their
            // waits one after the other in a few steps instead of running one
            // after the other; the output run follows from h_in.  A launch for
            // the final state alone (state_only) takes this path for every
            // piece and stops after the end state.
            run_subs(true, h, dsum, false);
            HV hin[S / 2];
            if (sb > 0) {
                if (!wait_carry(sb)) return;
                load_carry(hin);
            } else {
                load_h0(hin);
            }
            HV hend[S / 2];
#pragma unroll
            for (int k = 0; k < S / 2; ++k) {
                // exp(A sum(delta)): fp64 for fp32 activations, else one ex2 each
                if constexpr (ACC) {
                    hend[k].x = fma(exp((double)A2[k].x * dsum), hin[k].x, h[k].x);
                    hend[k].y = fma(exp((double)A2[k].y * dsum), hin[k].y, h[k].y);
                } else {
                    const float2 decay = f2(ex2_mufu((float)((double)A2[k].x * dsum)),
                                            ex2_mufu((float)((double)A2[k].y * dsum)));
                    hend[k] = __ffma2_rn(decay, hin[k], h[k]);
                }
                h[k] = p.state_only ? hend[k] : hin[k];
            }
            if (se < p.subs_per_chain) {
                store_carry(hend);
                publish_carry(se);
            }
            if (!p.state_only) run_subs(false, h, dsum, false);
        } else {
            if (sb > 0) {
                if (!wait_carry(sb)) return;
                load_carry(h);
            } else {
                load_h0(h);
            }
            run_subs(false, h, dsum, true);
        }

        if (se == p.subs_per_chain && p.last_state != nullptr && ds < Dm) {
            float *ls = p.last_state + (b * Dm + ds) * N;
#pragma unroll
            for (int k = 0; k < S / 2; ++k) {
                const int n0 = S * sr + 2 * k;
                if (n0 < N && MSCAN_WITHIN(p.x_last, ls + n0, 4, kSiteLastState)) ls[n0] = (float)h[k].x;
                if (n0 + 1 < N && MSCAN_WITHIN(p.x_last, ls + n0 + 1, 4, kSiteLastState)) ls[n0 + 1] = (float)h[k].y;
            }
        }
    }
}

template <typename T, int R, bool SP, bool GATE, bool CONV, bool LOCAL, bool CL = false, bool UNR = false>
cudaError_t launch_t(const Params &kp, int sm_count, cudaStream_t st) {
    using PL = PairLaunch<R, LOCAL>;
    const int smem = PL::kWorkers * PairSmem<T, R>::BYTES + (LOCAL ? LocalSmem<R>::BYTES : 0);
    auto kern = scan_fwd_pairs_kernel<T, R, SP, GATE, CONV, LOCAL, CL, UNR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    static const int per_sm = [&] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, PL::kWorkers * 32, smem) != cudaSuccess) n = 0;
        return n < PL::kMinBlocks ? n : PL::kMinBlocks;
    }();
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(PL::kWorkers * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (LOCAL) {
        // independent blocks, one per SM, each with at least one whole group
        const int grid = kp.n_groups < sm_count ? kp.n_groups : sm_count;
        cfg.gridDim = dim3((unsigned)grid);
        cfg.numAttrs = 0;
    } else {
        // a worker may wait on the one before it: launch them all resident at once
        cfg.gridDim = dim3((unsigned)(sm_count * per_sm));
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, kp);
}

// Whether any worker of the launch gets a share short enough for two-phase
// pieces (the kernel's own test: 20 groups < 11 workers in its scope) -- in
// the block-local form, the block with the fewest whole groups.
template <int R, bool LOCAL>
bool has_two_phase(const Params &kp, int sm_count) {
    using PL = PairLaunch<R, LOCAL>;
    const long long G = kp.n_groups;
    if (LOCAL) {
        const long long nb = G < sm_count ? G : sm_count;
        return 20LL * (G / nb) < 11LL * PL::kWorkers;
    }
    return 20LL * G < 11LL * (long long)sm_count * PL::kMinBlocks * PL::kWorkers;
}

template <int R, bool LOCAL>
cudaError_t launch_r(const Params &kp, int act, int sm_count, cudaStream_t st) {
    const bool gate = kp.z != nullptr;
    using BF = __nv_bfloat16;
    if (kp.channels_last) {  // block-local form only, no fused convolution
        if (!LOCAL || kp.conv_w) return cudaErrorInvalidValue;
        // unrolled (with the gate: without it the channel-last form would spill)
        if (act == kBF16 && R == 2 && gate && !kp.state_only && !has_two_phase<R, LOCAL>(kp, sm_count))
            return kp.softplus ? launch_t<BF, 2, true, true, false, true, true, true>(kp, sm_count, st)
                               : launch_t<BF, 2, false, true, false, true, true, true>(kp, sm_count, st);
        if (act == kBF16) {
            if (kp.softplus) return gate ? launch_t<BF, R, true, true, false, true, true>(kp, sm_count, st)
                                         : launch_t<BF, R, true, false, false, true, true>(kp, sm_count, st);
            return gate ? launch_t<BF, R, false, true, false, true, true>(kp, sm_count, st)
                        : launch_t<BF, R, false, false, false, true, true>(kp, sm_count, st);
        }
        if (kp.softplus) return gate ? launch_t<float, R, true, true, false, true, true>(kp, sm_count, st)
                                     : launch_t<float, R, true, false, false, true, true>(kp, sm_count, st);
        return gate ? launch_t<float, R, false, true, false, true, true>(kp, sm_count, st)
                    : launch_t<float, R, false, false, false, true, true>(kp, sm_count, st);
    }
    if (kp.conv_w) {  // fused conv1d prologue: softplus on (checked by the caller)
        if (act == kBF16 && R == 2 && !has_two_phase<R, LOCAL>(kp, sm_count))
            return gate ? launch_t<BF, 2, true, true, true, LOCAL, false, true>(kp, sm_count, st)
                        : launch_t<BF, 2, true, false, true, LOCAL, false, true>(kp, sm_count, st);
        if (act == kBF16) return gate ? launch_t<BF, R, true, true, true, LOCAL>(kp, sm_count, st)
                                      : launch_t<BF, R, true, false, true, LOCAL>(kp, sm_count, st);
        return gate ? launch_t<float, R, true, true, true, LOCAL>(kp, sm_count, st)
                    : launch_t<float, R, true, false, true, LOCAL>(kp, sm_count, st);
    }
    if (act == kBF16) {
        // the unrolled form (four lanes: with the gate only, else it would spill)
        if (!kp.state_only && (R == 2 || gate) && !has_two_phase<R, LOCAL>(kp, sm_count)) {
            if (gate)
                return kp.softplus ? launch_t<BF, R, true, true, false, LOCAL, false, true>(kp, sm_count, st)
                                   : launch_t<BF, R, false, true, false, LOCAL, false, true>(kp, sm_count, st);
            if constexpr (R == 2)
                return kp.softplus ? launch_t<BF, 2, true, false, false, LOCAL, false, true>(kp, sm_count, st)
                                   : launch_t<BF, 2, false, false, false, LOCAL, false, true>(kp, sm_count, st);
        }
        if (kp.softplus) return gate ? launch_t<BF, R, true, true, false, LOCAL>(kp, sm_count, st)
                                     : launch_t<BF, R, true, false, false, LOCAL>(kp, sm_count, st);
        return gate ? launch_t<BF, R, false, true, false, LOCAL>(kp, sm_count, st)
                    : launch_t<BF, R, false, false, false, LOCAL>(kp, sm_count, st);
    }
    if (kp.softplus) return gate ? launch_t<float, R, true, true, false, LOCAL>(kp, sm_count, st)
                                 : launch_t<float, R, true, false, false, LOCAL>(kp, sm_count, st);
    return gate ? launch_t<float, R, false, true, false, LOCAL>(kp, sm_count, st)
                : launch_t<float, R, false, false, false, LOCAL>(kp, sm_count, st);
}

}  // namespace

int persistent_split_sub_chunk(int lanes, int act) {
    (void)lanes;
    return act == kBF16 ? PairSmem<__nv_bfloat16, 2>::kTC : PairSmem<float, 2>::kTC;
}

int persistent_split_blocks_per_sm(int lanes) {
    return lanes == 4 ? LanesOccupancy<4>::kBlocks : LanesOccupancy<2>::kBlocks;
}

cudaError_t launch_persistent_split(const Params &kp, int lanes, int act, int sm_count, cudaStream_t st) {
    if (lanes == 4) return launch_r<4, false>(kp, act, sm_count, st);
    return launch_r<2, false>(kp, act, sm_count, st);
}

int local_split_warps(int lanes) { return lanes == 4 ? LocalWarps<4>::value : LocalWarps<2>::value; }

cudaError_t launch_local_split(const Params &kp, int lanes, int act, int sm_count, cudaStream_t st) {
    if (lanes == 4) return launch_r<4, true>(kp, act, sm_count, st);
    return launch_r<2, true>(kp, act, sm_count, st);
}

MSCAN_BOUNDS_TAKE(pairs_bounds_take)

int take_local_error(unsigned *flag) {
    unsigned v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_local_error, sizeof(v)) != cudaSuccess) return -1;
    if (v != 0 && cudaMemcpyToSymbol(g_local_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
    *flag = v;
    return 0;
}

}  // namespace mscan
