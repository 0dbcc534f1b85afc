// scan_fwd_persistent.cu -- the selective-scan (S6) forward pass as a
// persistent, dynamically balanced kernel for sm_100a.
//
// Same result as scan_fwd.cu (one fused pass: softplus(delta + bias), the
// zero-order-hold decay exp(delta A), the diagonal recurrence, the C readout,
// the D skip and the silu(z) gate -- "Mamba SSM concept and implementation in
// Keras and TensorFlow", recurrent form and selective_scan / MambaBlock; fused
// without materialising (batch, L, dim, N) in HBM as in the Mamba paper,
// Appendix E.5), organised for throughput on B200:
//
// * One thread owns one channel and all of its (<= 16) states, so the
//   readout C.h needs no cross-lane sum and each element's softplus / gate is
//   computed exactly once, by the thread that uses it.
// * Each warp is an independent worker (its own shared-memory region, only
//   warp-level synchronisation).  Work units are (group of 32 channels of one
//   batch row, chunk of TU timesteps).  A unit needs the state its
//   predecessor chunk ended with; that carry goes through global memory.
// * Units are handed out by a ready queue: the first chunk of every group is
//   ready at launch, and finishing chunk j of a group enqueues chunk j+1.  A
//   worker always takes the oldest ready unit, so all SM sub-partitions stay
//   busy until the queue drains, whatever the number of groups relative to
//   the 4 x 148 sub-partitions -- the imbalance a static one-block-per-group
//   launch suffers when the group count is not a multiple of the SM count.
// * Inside a unit, sub-chunks of TC timesteps are double-buffered: raw
//   u / delta / z rows and the per-batch-row B / C rows are copied global ->
//   shared with 16-byte cp.async while the previous sub-chunk is computed;
//   B and C are widened to fp32 once per sub-chunk and read as warp-wide
//   broadcasts; outputs are packed to the activation type in a shared tile
//   and stored with coalesced 16-byte stores.
// * The state update runs on pairs of states with the packed fp32 x2
//   instructions (FMUL2 / FFMA2), halving FP32 issue slots; the 16 ex2 per
//   element go to the MUFU, which bounds the kernel.
// * Every wait on another worker is bounded: on timeout the worker sets the
//   error word in the workspace header and leaves; nothing spins forever.
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
using PParams = persist::Params;

template <typename T>
struct WarpSmem {
    static constexpr int kTC = 128 / (int)sizeof(T);       // timesteps per sub-chunk: 128-byte rows
    static constexpr int V = 16 / (int)sizeof(T);        // elements per 16 bytes
    static constexpr int ROWB = kTC * (int)sizeof(T) + 16;  // padded raw row (bytes)
    static constexpr int RAW_ROWS = 3 * 32 + 2 * 16;       // u, delta, z, B, C rows
    static constexpr int STAGE = RAW_ROWS * ROWB;
    static constexpr int BC32 = 2 * kTC * kNS * 4;         // fp32 B and C, [t][n]
    static constexpr int OUTB = 32 * ROWB;                 // packed output tile
    static constexpr int BYTES = 2 * STAGE + BC32 + OUTB;
};

template <typename T, bool SP, bool GATE>
__global__ void __launch_bounds__(kWarps * 32, 1)
scan_fwd_persistent_kernel(const PParams p) {
    using W = WarpSmem<T>;
    constexpr int V = W::V;
    constexpr int kTC = W::kTC;
    constexpr int CPR = kTC / V;  // 16-byte chunks per row per sub-chunk
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    unsigned char *base = smem + warp * W::BYTES;
    unsigned char *stage_base = base;                       // 2 stages
    float *bc32 = reinterpret_cast<float *>(base + 2 * W::STAGE);  // B: [t][16], then C
    unsigned char *outt = base + 2 * W::STAGE + W::BC32;

    const int64_t L = p.seqlen, Dm = p.dim;
    const int N = p.dstate;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B);
    const T *gC = static_cast<const T *>(p.C);
    T *gout = static_cast<T *>(p.out);
    int cur_group = -1;
    float2 A2[kNS / 2];
    float bias = 0.f, Dd = 0.f;

#pragma unroll 1
    while (true) {
        // ---- take the next ready unit
        const unsigned unit = pop_unit(p, lane);
        if (unit == kUnitDone || unit == kUnitAbort) break;
        const int g = (int)(unit % (unsigned)p.n_groups);
        const int j = (int)(unit / (unsigned)p.n_groups);
        const int64_t b = g / p.groups_per_batch;
        const int64_t d0 = (int64_t)(g % p.groups_per_batch) * 32;
        const int64_t d = d0 + lane;
        const bool dvalid = d < Dm;
        const int nrows = (Dm - d0) < 32 ? (int)(Dm - d0) : 32;  // valid channel rows

        if (g != cur_group) {
            cur_group = g;
#pragma unroll
            for (int k = 0; k < kNS / 2; ++k) {
                const int n0 = 2 * k, n1 = 2 * k + 1;
                const float a0 = (dvalid && n0 < N) ? __ldg(p.A + d * N + n0) : 0.f;
                const float a1 = (dvalid && n1 < N) ? __ldg(p.A + d * N + n1) : 0.f;
                A2[k] = make_float2(a0 * kLog2e, a1 * kLog2e);
            }
            bias = (dvalid && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.f;
            Dd = (dvalid && p.D) ? __ldg(p.D + d) : 0.f;
        }

        // ---- carried state
        float2 h[kNS / 2];
        float *carry = p.carry + ((int64_t)g * 32 + lane) * kNS;
        if (j == 0) {
#pragma unroll
            for (int k = 0; k < kNS / 2; ++k) h[k] = make_float2(0.f, 0.f);
        } else {
#pragma unroll
            for (int k = 0; k < kNS / 4; ++k) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(carry) + k);
                h[2 * k] = make_float2(v.x, v.y);
                h[2 * k + 1] = make_float2(v.z, v.w);
            }
        }

        const int64_t tb0 = (int64_t)j * p.chunk_len;
        const int64_t tb1 = (tb0 + p.chunk_len) < L ? (tb0 + p.chunk_len) : L;
        const int nsub = (int)((tb1 - tb0 + kTC - 1) / kTC);
        const int64_t row0 = (b * Dm + d0) * L;  // element offset of this group's first row
        const int64_t bc0 = b * (int64_t)N * L;

        auto issue = [&](int sub, int st) {
            unsigned char *sb = stage_base + st * W::STAGE;
            const int64_t t0 = tb0 + (int64_t)sub * kTC;
            // u, delta, z: 32 rows x CPR chunks each
#pragma unroll
            for (int i = lane; i < 32 * CPR; i += 32) {
                const int r = i / CPR, c = i % CPR;
                const int64_t t = t0 + c * V;
                const bool ok = (r < nrows) && (t < L);
                const int64_t off = ok ? row0 + r * L + t : 0;
                cp16(sb + (0 * 32 + r) * W::ROWB + c * 16, gu + off, ok);
                cp16(sb + (1 * 32 + r) * W::ROWB + c * 16, gd + off, ok);
                if (GATE) cp16(sb + (2 * 32 + r) * W::ROWB + c * 16, gz + off, ok);
            }
            // B, C: 16 rows x CPR chunks each
#pragma unroll
            for (int i = lane; i < 2 * kNS * CPR; i += 32) {
                const int which = i / (kNS * CPR), rem = i % (kNS * CPR);
                const int n = rem / CPR, c = rem % CPR;
                const int64_t t = t0 + c * V;
                const bool ok = (n < N) && (t < L);
                const int64_t off = ok ? bc0 + (int64_t)n * L + t : 0;
                cp16(sb + (96 + which * 16 + n) * W::ROWB + c * 16, (which ? gC : gB) + off, ok);
            }
            cp_commit();
        };

        issue(0, 0);
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
            const unsigned char *sb = stage_base + st * W::STAGE;
            const int64_t t0 = tb0 + (int64_t)sub * kTC;
            const int tvalid = (L - t0) < kTC ? (int)(L - t0) : kTC;

            // widen B and C to fp32, transposed to [t][n] for broadcast reads
#pragma unroll
            for (int i = lane; i < 2 * kNS * CPR; i += 32) {
                const int which = i / (kNS * CPR), rem = i % (kNS * CPR);
                const int n = rem / CPR, c = rem % CPR;
                float f[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(sb + (96 + which * 16 + n) * W::ROWB + c * 16), f);
                float *dst = bc32 + which * kTC * kNS;
#pragma unroll
                for (int e = 0; e < V; ++e) dst[(c * V + e) * kNS + n] = f[e];
            }
            __syncwarp();

            const unsigned char *ru = sb + (0 * 32 + lane) * W::ROWB;
            const unsigned char *rd = sb + (1 * 32 + lane) * W::ROWB;
            const unsigned char *rz = sb + (2 * 32 + lane) * W::ROWB;
            unsigned char *ro = outt + lane * W::ROWB;
            const float *sBt = bc32;
            const float *sCt = bc32 + kTC * kNS;
            // Per-element values of one vector of V timesteps.  The vector
            // loop is software-pipelined: the next vector's values (smem
            // loads, softplus, gate) are computed while the current
            // vector's states update.  Reads one vector past the sub-chunk
            // land in the row padding and are never used; timesteps past
            // the end have delta = 0 (Abar = 1, no input) and are not stored.
            struct Pre { float dl[V], du[V], gg[V], sk[V]; };
            auto pre = [&](int tv, Pre &P) {
                float fu[V], fd[V], fz[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(ru + tv * sizeof(T)), fu);
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rd + tv * sizeof(T)), fd);
                if (GATE) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rz + tv * sizeof(T)), fz);
#pragma unroll
                for (int e = 0; e < V; e += 2) {  // element pairs on the packed x2 instructions
                    float2 x = __fadd2_rn(f2(fd[e], fd[e + 1]), f2(bias, bias));
                    if (SP) x = softplus2_f(x);
                    P.dl[e] = (tv + e < tvalid) ? x.x : 0.f;
                    P.dl[e + 1] = (tv + e + 1 < tvalid) ? x.y : 0.f;
                    const float2 uu = f2(fu[e], fu[e + 1]);
                    const float2 xu = __fmul2_rn(f2(P.dl[e], P.dl[e + 1]), uu);
                    P.du[e] = xu.x; P.du[e + 1] = xu.y;
                    const float2 gg = GATE ? silu2_f(f2(fz[e], fz[e + 1])) : f2(1.f, 1.f);
                    P.gg[e] = gg.x; P.gg[e + 1] = gg.y;
                    const float2 sk = __fmul2_rn(f2(Dd, Dd), uu);
                    P.sk[e] = sk.x; P.sk[e + 1] = sk.y;
                }
            };
            Pre cur, nxt;
            pre(0, cur);
#pragma unroll 2
            for (int tv = 0; tv < kTC; tv += V) {
                pre(tv + V, nxt);
                // states: state pairs outer, timesteps inner.  Per pair the
                // recurrence is a short FFMA2 chain through the V timesteps;
                // the exponentials depend only on delta and can all be issued
                // ahead; the V readout sums are independent accumulators.
                float2 y2[V];
#pragma unroll
                for (int e = 0; e < V; ++e) y2[e] = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) {
#pragma unroll
                    for (int e = 0; e < V; ++e) {
                        const int t = tv + e;
                        const float4 bb = *reinterpret_cast<const float4 *>(sBt + t * kNS + 4 * q);
                        const float4 cc = *reinterpret_cast<const float4 *>(sCt + t * kNS + 4 * q);
                        const float2 dl2 = make_float2(cur.dl[e], cur.dl[e]);
                        const float2 du2 = make_float2(cur.du[e], cur.du[e]);
                        const float2 x0 = __fmul2_rn(dl2, A2[2 * q]);
                        const float2 x1 = __fmul2_rn(dl2, A2[2 * q + 1]);
                        const float2 a0 = make_float2(ex2_mufu(x0.x), ex2_mufu(x0.y));
                        const float2 a1 = make_float2(ex2_mufu(x1.x), ex2_mufu(x1.y));
                        const float2 bu0 = __fmul2_rn(du2, make_float2(bb.x, bb.y));
                        const float2 bu1 = __fmul2_rn(du2, make_float2(bb.z, bb.w));
                        h[2 * q] = __ffma2_rn(a0, h[2 * q], bu0);
                        h[2 * q + 1] = __ffma2_rn(a1, h[2 * q + 1], bu1);
                        y2[e] = __ffma2_rn(make_float2(cc.x, cc.y), h[2 * q], y2[e]);
                        y2[e] = __ffma2_rn(make_float2(cc.z, cc.w), h[2 * q + 1], y2[e]);
                    }
                }
                float fo[V];
#pragma unroll
                for (int e = 0; e < V; ++e) fo[e] = (y2[e].x + y2[e].y + cur.sk[e]) * cur.gg[e];
                *reinterpret_cast<uint4 *>(ro + tv * sizeof(T)) = Elem<T>::pack(fo);
                cur = nxt;
            }
            __syncwarp();
            // the last sub-chunk's state is final: publish the successor unit
            // before this tile's stores, so the release waits on less
            if (sub + 1 == nsub && j + 1 < p.n_chunks) {
#pragma unroll
                for (int k = 0; k < kNS / 4; ++k)
                    __stcg(reinterpret_cast<float4 *>(carry) + k,
                           make_float4(h[2 * k].x, h[2 * k].y, h[2 * k + 1].x, h[2 * k + 1].y));
                push_unit(p, lane, (unsigned)((j + 1) * p.n_groups + g));
            }
            // coalesced store of the packed tile
#pragma unroll
            for (int i = lane; i < 32 * CPR; i += 32) {
                const int r = i / CPR, c = i % CPR;
                const int64_t t = t0 + c * V;
                if (r < nrows && t < L)
                    stg16_stream(gout + row0 + r * L + t,
                                 *reinterpret_cast<const uint4 *>(outt + r * W::ROWB + c * 16));
            }
            __syncwarp();
        }

        if (j + 1 == p.n_chunks && p.last_state != nullptr && dvalid) {
            float *ls = p.last_state + (b * Dm + d) * N;
#pragma unroll
            for (int k = 0; k < kNS / 2; ++k) {
                if (2 * k < N) ls[2 * k] = h[k].x;
                if (2 * k + 1 < N) ls[2 * k + 1] = h[k].y;
            }
        }
    }
}

}  // namespace

template <typename T, bool SP, bool GATE>
static cudaError_t launch_t(const persist::Params &kp, int grid, cudaStream_t st) {
    const int smem = kWarps * WarpSmem<T>::BYTES;
    auto kern = scan_fwd_persistent_kernel<T, SP, GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarps * 32, smem, st>>>(kp);
    return cudaGetLastError();
}

int persistent_lanes1_sub_chunk(int act) {
    return act == kBF16 ? WarpSmem<__nv_bfloat16>::kTC : WarpSmem<float>::kTC;
}

int persistent_lanes1_blocks_per_sm() { return 1; }

cudaError_t launch_persistent_lanes1(const persist::Params &kp, int act, int grid, cudaStream_t st) {
    const bool gate = kp.z != nullptr;
    if (act == kBF16) {
        if (kp.softplus) return gate ? launch_t<__nv_bfloat16, true, true>(kp, grid, st)
                                     : launch_t<__nv_bfloat16, true, false>(kp, grid, st);
        return gate ? launch_t<__nv_bfloat16, false, true>(kp, grid, st)
                    : launch_t<__nv_bfloat16, false, false>(kp, grid, st);
    }
    if (kp.softplus) return gate ? launch_t<float, true, true>(kp, grid, st)
                                 : launch_t<float, true, false>(kp, grid, st);
    return gate ? launch_t<float, false, true>(kp, grid, st) : launch_t<float, false, false>(kp, grid, st);
}

}  // namespace mscan
