// scan_bwd.cu -- backward pass of the selective scan (S6): the gradients of
// the forward in scan_fwd*.cu with respect to every input, given dL/dout and
// (optionally) dL/dlast_state.  Reverse-mode differentiation of the
// recurrence h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t,
// y_t = C_t h_t + D u_t, out_t = y_t silu(z_t) (training the layer
// back-propagates through the scan; the Mamba paper's hardware-aware
// algorithm, Section 3.3, recomputes the states in the backward pass rather
// than storing them).  With g = dL/dh_t carried backwards and, per step,
// g' = g + dy C_t (the adjoint of h_t once the step's readout is in):
//   dy = dout silu(z);  dz = dout y silu'(z);  dD += dy u
//   dC[n,t] += dy h_t[n];  dB[n,t] += g'[n] delta u
//   S_B = sum_n g'[n] B[n,t];  S_A = sum_n g'[n] Abar h_{t-1}[n] A[n]
//   du = dy D + delta S_B;  ddelta = S_A + u S_B;  dA[n] += g'[n] Abar h_{t-1}[n] delta
//   g[n] <- Abar g'[n]   (the adjoint of h_{t-1})
//   ddelta_raw = ddelta sigmoid(delta_raw + bias) (softplus);  dbias += ddelta_raw
// and, when the forward started from a given state h0, dh0 = g after t = 0.
//
// Design.  A block of four warps takes a group of 32 channels of one batch
// row; in a warp, lane 4 c + r takes channel c (of 8) and states 4 r .. 4 r + 3.
//   * States every kSup = 32 timesteps (the checkpoints) come from the forward
//     (mamba_scan_fwd_ckpt writes them) or from a first sweep of this kernel.
//   * The sequence is then walked backwards one 32-step super-segment at a
//     time.  Its inputs are staged once for the block (16-byte cp.async, the
//     next super-segment's copies issued as soon as this one's are
//     converted); per element, delta = softplus(raw + bias), sigmoid(raw +
//     bias), dy = dout silu(z) and the gate factor dout sigmoid(z) (1 + z (1 -
//     sigmoid(z))) are formed once into shared memory, B and C widened once.
//   * From the segment's checkpoint the states are recomputed over the 32
//     steps, leaving one sub-checkpoint every kSub = 4 steps (per-group
//     workspace, L2-resident); then each 4-step window, last first, is
//     recomputed once more into registers -- states and decays -- and walked
//     in reverse from them, so the reverse step evaluates no exponential.
//   * Sums over a channel's states (C h, S_A, S_B) are kept per step of the
//     4-step window and summed over the channel's 4 lanes at its end,
//     transposed: lane r then holds step r's totals and forms that step's
//     du, ddelta_raw, dz and its dD and dbias terms.  dB and dC,
//     sums over every channel of a batch row, are summed over a warp's 8
//     channels by a transposed shuffle reduction, over the block's warps in
//     shared memory, and added with one atomic add per (state, step) and
//     block into one of kRep copies (group % kRep: the blocks of a batch row
//     walk the sequence in step and would otherwise all queue on the same
//     addresses); a last kernel adds the copies.  dB / dC are therefore not
//     bitwise reproducible from run to run (the atomics' order varies).  dA,
//     dD and dbias are summed per group in registers, one atomic add each at
//     the end.
//   * du, ddelta_raw and dz of a super-segment are staged in shared memory and
//     written as whole 16-byte pieces of each row.
// fp32 activations keep states and adjoints in fp64 with the accurate decays
// of device_math.cuh (Decay<true>), bf16 ones fp32 with one ex2 per decay.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "bounds.cuh"
#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kNS = 16;                  // padded states per channel (dstate <= 16)
constexpr int kSPL = 4;                  // states per lane
constexpr int kCPW = 8;                  // channels per warp
constexpr int kSup = 32;                 // timesteps between checkpoints (one staged super-segment)
constexpr int kSub = 4;                  // timesteps recomputed into registers at a time
constexpr int kNSub = kSup / kSub;       // sub-checkpoints per super-segment
constexpr int kRep = 8;                  // copies of dB / dC the blocks add into (group % kRep)
constexpr int kCkCh = 32;                // channels per checkpoint group (the forward's layout)
// a window's steps are shared out one per lane of a channel for the per-step sums
static_assert(kSub == kNS / kSPL, "one window step per lane of a channel");

// per-channel fp32 values of a super-segment: one 16-byte record per (step,
// channel) -- (delta, u, dy, gate factor) -- read with one load, and the
// sigmoid of the raw step, [t][channel]

// Row pitches are padded so that the accesses below are free of bank
// conflicts: raw / output rows by 16 bytes (rows read or written 16 bytes at
// a time by lanes of different rows, or element-wise by lanes of 8 rows).
// The per-channel arrays are written by 32 lanes of one step (contiguous)
// and read by lanes of 8 channels of one step (broadcast within a channel).
// A block: WARPS warps = 8 WARPS channels of one batch row (4 or 6 warps,
// chosen per shape so that the blocks spread evenly over the SMs).
template <typename T, int WARPS>
struct BwdSmem {
    static constexpr int kCh = WARPS * kCPW;                  // channels per block
    static constexpr int kRawRows = 4 * kCh + 2 * kNS;        // u, delta_raw, dout, z rows; B, C rows
    static constexpr int V = 16 / (int)sizeof(T);            // elements per 16-byte copy
    static constexpr int CPR = kSup / V;                      // copies per staged row
    static constexpr int RP = kSup + V;                       // raw / output row pitch (elements)
    static constexpr int RAW = kRawRows * RP * (int)sizeof(T);
    static constexpr int SX = kSup * kCh * 16 + kSup * kCh * 4;  // records [t][c], sigmoid [t][c]
    static constexpr int BC = kSup * 2 * kNS * 4;             // [t][B 0..15, C 16..31] fp32
    static constexpr int RED = 2 * kSub * WARPS * 32 * 4;     // two buffers of [step][warp][slot]
    static constexpr int OUT = 3 * kCh * RP * (int)sizeof(T); // du, ddelta_raw, dz [q][c][t]
    static constexpr int BYTES = (RAW + 15) / 16 * 16 + SX + BC + RED + OUT;
};

struct BwdParams {
    const void *u, *delta, *B, *C, *z, *dout;
    const float *A, *D, *delta_bias, *dlast, *h0;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *dbias, *dh0;
    float *ckpt;        // [batch * ckpt_g32][n_sup][32 channels][16 states]: the state entering each super-segment
    int ckpt_g32;       // ceil(dim / 32)
    float *rep;         // [kRep][2 (dB, dC)][batch][16][L] fp32, zeroed: the atomics' targets
    void *subck;        // [group][kNSub][threads][4 states] (state type): sub-checkpoints
    int ckpt_given;     // the checkpoints were written by the forward: no sweep
    int vec;            // rows 16-byte aligned and L a whole number of 16-byte copies
    int64_t batch, dim, seqlen;
    int dstate, softplus;
    int groups_per_batch, n_groups, n_sup;
    // byte ranges of the pointer arguments and workspace parts, for the
    // bounds-checked build (indexed by the fetch's row kind: u, delta, dout,
    // z, then B, C)
    MSCAN_EXTENTS(x_in[6], x_A, x_D, x_bias, x_dlast, x_h0, x_dout3[3], x_dA, x_dB, x_dC, x_dD, x_dbias, x_dh0,
                  x_ckpt, x_subck, x_rep)
};

__device__ __forceinline__ void cp16_async(void *smem, const void *gmem, bool pred) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(sa), "l"(gmem), "r"(pred ? 16 : 0) : "memory");
}

// Sum v[] over the 8 lanes that share lane & 3, transposed: afterwards v[0]
// of lane 4 c + r holds the total of the lanes' original v[c].  Round K (lane
// bit 16, 8, 4) halves the live values; the lane with bit K set keeps the
// upper half.
template <int K, int CNT>
struct ChannelTranspose {
    __device__ __forceinline__ static void run(float (&v)[8], int lane) {
        constexpr int HALF = CNT / 2;
        const bool upper = (lane & K) != 0;
        float recv[HALF], keep[HALF];
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
            const float send = upper ? v[i] : v[i + HALF];
            keep[i] = upper ? v[i + HALF] : v[i];
            recv[i] = __shfl_xor_sync(0xffffffffu, send, K);
        }
        // the sums two at a time on the packed x2 add
#pragma unroll
        for (int i = 0; i + 1 < HALF; i += 2) {
            const float2 s2 = __fadd2_rn(f2(keep[i], keep[i + 1]), f2(recv[i], recv[i + 1]));
            v[i] = s2.x;
            v[i + 1] = s2.y;
        }
        if (HALF & 1) v[HALF - 1] = keep[HALF - 1] + recv[HALF - 1];
        ChannelTranspose<K / 2, HALF>::run(v, lane);
    }
};
template <int CNT>
struct ChannelTranspose<2, CNT> {
    __device__ __forceinline__ static void run(float (&)[8], int) {}
};

// Sum part[w][q] over the 4 lanes of a channel (lane bits 0 and 1),
// transposed: afterwards part[0][q] of lane r holds the total of the lanes'
// original part[r][q].  Round K = 2 keeps steps 2, 3 in the lanes with bit 1
// set and 0, 1 in the others; round K = 1 keeps the odd or even one.
template <typename X>
struct QuadTranspose {
    __device__ __forceinline__ static void run(X (&part)[4][3], int lane) {
        const bool up2 = (lane & 2) != 0, up1 = (lane & 1) != 0;
        X keep[2][3], recv[2][3];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const X send = up2 ? part[i][q] : part[i + 2][q];
                keep[i][q] = up2 ? part[i + 2][q] : part[i][q];
                recv[i][q] = __shfl_xor_sync(0xffffffffu, send, 2);
            }
        }
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            if constexpr (std::is_same<X, float>::value) {  // steps 0 and 1 on one packed x2 add
                const float2 s2 = __fadd2_rn(f2(keep[0][q], keep[1][q]), f2(recv[0][q], recv[1][q]));
                part[0][q] = s2.x;
                part[1][q] = s2.y;
            } else {
                part[0][q] = keep[0][q] + recv[0][q];
                part[1][q] = keep[1][q] + recv[1][q];
            }
        }
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            const X send = up1 ? part[0][q] : part[1][q];
            const X keep1 = up1 ? part[1][q] : part[0][q];
            part[0][q] = keep1 + __shfl_xor_sync(0xffffffffu, send, 1);
        }
    }
};

// A lane's 4 states of a sub-checkpoint: one 16-byte access (fp32 states)
// or two (fp64); the slot is 16-byte aligned.
__device__ __forceinline__ void store4(float *q, const float (&h)[4]) {
    *reinterpret_cast<float4 *>(q) = make_float4(h[0], h[1], h[2], h[3]);
}
__device__ __forceinline__ void store4(double *q, const double (&h)[4]) {
    reinterpret_cast<double2 *>(q)[0] = make_double2(h[0], h[1]);
    reinterpret_cast<double2 *>(q)[1] = make_double2(h[2], h[3]);
}
__device__ __forceinline__ void load4(const float *q, float (&h)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(q);
    h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
}
__device__ __forceinline__ void load4(const double *q, double (&h)[4]) {
    const double2 a = reinterpret_cast<const double2 *>(q)[0], b = reinterpret_cast<const double2 *>(q)[1];
    h[0] = a.x; h[1] = a.y; h[2] = b.x; h[3] = b.y;
}

template <typename X>
__device__ __forceinline__ X quad_sum(X x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// 1 / (1 + e^-x): the MUFU form for bf16 activations, CUDA's full-precision
// expf and division for fp32 ones.
template <bool ACC>
__device__ __forceinline__ float sigmoid(float x) {
    if (ACC) return 1.f / (1.f + expf(-x));
    return __fdividef(1.f, 1.f + __expf(-x));
}

// Blocks per SM that shared memory allows ([fp32 activations][6 warps]; 228
// KiB per SM, 1 KiB of it reserved per block): bf16 48 KiB (4 warps) or
// 68.75 KiB (6); fp32 64 KiB or 91.75 KiB.  The register cap follows from it.
constexpr int kBwdBlocksPerSM[2][2] = {{4, 3}, {3, 2}};

template <typename T, bool SP, bool GATE, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, kBwdBlocksPerSM[sizeof(T) == 4][WARPS == 6])
scan_bwd_kernel(const BwdParams p) {
    constexpr bool ACC = sizeof(T) == 4;
    using Dk = Decay<ACC>;
    using HS = typename Dk::H;  // states and adjoints: fp64 for fp32 activations
    using SM = BwdSmem<T, WARPS>;
    constexpr int kWarpsBwd = WARPS, kCh = SM::kCh, kRawRows = SM::kRawRows;
    constexpr int V = SM::V, CPR = SM::CPR, RP = SM::RP;
    extern __shared__ __align__(16) unsigned char bwd_smem[];
    T *raw = reinterpret_cast<T *>(bwd_smem);                              // [kRawRows][RP]
    float4 *srec = reinterpret_cast<float4 *>(bwd_smem + (SM::RAW + 15) / 16 * 16);  // [t][c]
    float *ssig = reinterpret_cast<float *>(srec + kSup * kCh);           // [t][c]
    float *sbc = ssig + kSup * kCh;                                        // [t][32]
    float *red = sbc + kSup * 2 * kNS;                                     // [2][step][warp][slot]
    T *outs = reinterpret_cast<T *>(red + 2 * kSub * kWarpsBwd * 32);      // [3][c][RP]

    const int tid = threadIdx.x, lane = tid & 31, wib = tid >> 5;
    const int c = lane >> 2, r = lane & 3;
    const int cb = wib * kCPW + c;  // this lane's channel within the block
    const int64_t L = p.seqlen, Dm = p.dim;
    const int N = p.dstate;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B);
    const T *gC = static_cast<const T *>(p.C);
    const T *go = static_cast<const T *>(p.dout);
    T *gdst[3] = {static_cast<T *>(p.du), static_cast<T *>(p.ddelta), static_cast<T *>(p.dz)};

    for (int64_t grp = blockIdx.x; grp < p.n_groups; grp += gridDim.x) {
        const int64_t b = grp / p.groups_per_batch;
        const int64_t d0 = (grp % p.groups_per_batch) * kCh;
        const int64_t dc = d0 + cb;
        const bool valid = dc < Dm;
        float A2[kSPL], Ar[kSPL];
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int n = kSPL * r + i;
            Ar[i] = (valid && n < N && MSCAN_WITHIN(p.x_A, p.A + dc * N + n, 4, kSiteA)) ? __ldg(p.A + dc * N + n) : 0.f;
            A2[i] = Ar[i] * Dk::kScale;
        }
        const float Dd = (valid && p.D && MSCAN_WITHIN(p.x_D, p.D + dc, 4, kSiteD)) ? __ldg(p.D + dc) : 0.f;
        // this lane's checkpoints (the forward's layout: 32-channel groups): + s * 32 * 16
        float *ck = p.ckpt + ((b * p.ckpt_g32 + dc / kCkCh) * (int64_t)p.n_sup) * kCkCh * kNS + (dc % kCkCh) * kNS +
                    kSPL * r;
        HS *sub = static_cast<HS *>(p.subck) + (grp * kNSub * (kWarpsBwd * 32) + tid) * kSPL;  // + j * 128 * 4

        // ---- staging of super-segment s: the raw rows to shared memory
        // (16-byte cp.async, element copies for unaligned or ragged rows).
        // Thread -> (row, copy): rows of u, delta_raw, dout, z (kCh each, the
        // block's channels), then 16 B and 16 C rows.
        auto fetch = [&](int s, bool full) {
            const int64_t t0 = (int64_t)s * kSup;
            const int tn = (L - t0) < kSup ? (int)(L - t0) : kSup;
            for (int i = tid; i < kRawRows * CPR; i += kWarpsBwd * 32) {
                const int row = i / CPR, cp = i % CPR;
                const int q = row < 4 * kCh ? row / kCh : 4, rr = row < 4 * kCh ? row % kCh : row - 4 * kCh;
                if (!full && (q == 2 || q == 3 || (q == 4 && rr >= kNS))) continue;  // sweep: u, delta, B
                if (!GATE && q == 3) continue;
                const T *src;
                bool ok;
                if (q < 4) {
                    src = (q == 0 ? gu : q == 1 ? gd : q == 2 ? go : gz) + (b * Dm + d0 + rr) * L;
                    ok = d0 + rr < Dm;
                } else {
                    src = (rr < kNS ? gB : gC) + (b * N + (rr & 15)) * L;
                    ok = (rr & 15) < N;
                }
                T *dst = raw + row * RP + cp * V;
#ifdef MSCAN_BOUNDS_CHECK
                const int kind = q < 4 ? q : (rr < kNS ? 4 : 5);
                const int site = kind == 0 ? kSiteU : kind == 1 ? kSiteDelta : kind == 2 ? kSiteOut
                               : kind == 3 ? kSiteZ : kind == 4 ? kSiteB : kSiteC;
#endif
                if (p.vec) {
                    const bool in = ok && cp * V < tn && MSCAN_WITHIN(p.x_in[kind], src + t0 + cp * V, 16, site);
                    cp16_async(dst, in ? src + t0 + cp * V : src, in);
                } else {
#pragma unroll
                    for (int e = 0; e < V; ++e)
                        dst[e] = (ok && cp * V + e < tn && MSCAN_WITHIN(p.x_in[kind], src + t0 + cp * V + e, sizeof(T), site))
                                     ? src[t0 + cp * V + e] : T(0.f);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        // ---- per-element values of the staged super-segment, once for the
        // block: thread -> (channel tid % kCh, 16-byte piece of V steps), the
        // rows read 16 bytes at a time; B / C widened to [t][n].  Past the end
        // of the sequence delta = 0 (Abar = 1, no input) and the staged u,
        // dout, B, C are zero, so a step there leaves every state and adjoint
        // as it was: the loops below always run whole windows.
        auto convert = [&](int s, bool full) {
            const int64_t t0 = (int64_t)s * kSup;
            const int tn = (L - t0) < kSup ? (int)(L - t0) : kSup;
            const int cc = tid % kCh;
            const float bias = (d0 + cc < Dm && p.delta_bias && MSCAN_WITHIN(p.x_bias, p.delta_bias + d0 + cc, 4, kSiteBias))
                                   ? __ldg(p.delta_bias + d0 + cc) : 0.f;
            for (int piece = tid / kCh; piece < CPR; piece += (kWarpsBwd * 32) / kCh) {
                float fu[V], fd[V], fo[V], fz[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + cc * RP + piece * V), fu);
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + (kCh + cc) * RP + piece * V), fd);
                if (full) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + (2 * kCh + cc) * RP + piece * V), fo);
                if (full && GATE)
                    Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + (3 * kCh + cc) * RP + piece * V), fz);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    const int t = piece * V + e;
                    const float x = fd[e] + bias;
                    const float dl = t >= tn ? 0.f : SP ? Dk::softplus(x) : x;
                    float dy = 0.f, gzf = 0.f;
                    if (full) {
                        dy = fo[e];
                        if (GATE) {
                            const float sg = sigmoid<ACC>(fz[e]);
                            dy = fo[e] * fz[e] * sg;                          // dout silu(z)
                            gzf = fo[e] * sg * fmaf(fz[e], 1.f - sg, 1.f);    // dz = y * this
                        }
                        // zero past the end: those padding steps add nothing to dbias
                        ssig[t * kCh + cc] = t >= tn ? 0.f : SP ? sigmoid<ACC>(x) : 1.f;
                    }
                    srec[t * kCh + cc] = make_float4(dl, fu[e], dy, gzf);
                }
            }
            {  // B and C rows (after the channels' rows): row tid % 32, 16-byte piece
                const int row = tid & 31;
                if (full || row < kNS) {
                    for (int piece = tid >> 5; piece < CPR; piece += kWarpsBwd) {
                        float f[V];
                        Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + (4 * kCh + row) * RP + piece * V), f);
#pragma unroll
                        for (int e = 0; e < V; ++e) sbc[(piece * V + e) * 2 * kNS + row] = f[e];
                    }
                }
            }
        };
        // one forward step of this lane's states at step t of the staged segment
        auto step = [&](HS (&h)[kSPL], int t) {
            const float2 rec = *reinterpret_cast<const float2 *>(srec + t * kCh + cb);
            const float dl = rec.x;
            const float du = dl * rec.y;
            const float4 bb = *reinterpret_cast<const float4 *>(sbc + t * 2 * kNS + kSPL * r);
            const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
            if constexpr (ACC) {
#pragma unroll
                for (int i = 0; i < kSPL; ++i) h[i] = Dk::step(dl * A2[i], h[i], du * bv[i]);
            } else {  // state pairs on the packed x2 instructions (the same roundings)
#pragma unroll
                for (int k = 0; k < kSPL / 2; ++k) {
                    const float2 x = __fmul2_rn(f2(dl, dl), f2(A2[2 * k], A2[2 * k + 1]));
                    const float2 hn = __ffma2_rn(f2(ex2_mufu(x.x), ex2_mufu(x.y)), f2(h[2 * k], h[2 * k + 1]),
                                                 __fmul2_rn(f2(du, du), f2(bv[2 * k], bv[2 * k + 1])));
                    h[2 * k] = hn.x;
                    h[2 * k + 1] = hn.y;
                }
            }
        };
        auto seg_len = [&](int s) {
            const int64_t t0 = (int64_t)s * kSup;
            return (L - t0) < kSup ? (int)(L - t0) : kSup;
        };

        // ---- sweep (no checkpoints from the forward): the state entering
        // every super-segment, from h0 (or zeros)
        if (!p.ckpt_given) {
            HS h[kSPL];
#pragma unroll
            for (int i = 0; i < kSPL; ++i) {
                const int n = kSPL * r + i;
                h[i] = (valid && p.h0 && n < N && MSCAN_WITHIN(p.x_h0, p.h0 + (b * Dm + dc) * N + n, 4, kSiteH0))
                           ? (HS)__ldg(p.h0 + (b * Dm + dc) * N + n) : (HS)0.f;
            }
            fetch(0, false);
            for (int s = 0; s < p.n_sup; ++s) {
                if (valid && MSCAN_WITHIN(p.x_ckpt, ck + (int64_t)s * kCkCh * kNS, 16, kSiteCkpt))
                    __stcg(reinterpret_cast<float4 *>(ck + (int64_t)s * kCkCh * kNS),
                           make_float4((float)h[0], (float)h[1], (float)h[2], (float)h[3]));
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                __syncthreads();  // the raw rows have landed
                convert(s, false);
                __syncthreads();  // converted; the raw buffer is free
                if (s + 1 < p.n_sup) fetch(s + 1, false);
                const int nwin = (seg_len(s) + kSub - 1) / kSub;
                for (int j = 0; j < nwin; ++j) {
#pragma unroll
                    for (int w = 0; w < kSub; ++w) step(h, j * kSub + w);
                }
                __syncthreads();  // sx / sbc consumed
            }
        }

        // ---- reverse sweep, one super-segment at a time from the end
        HS g[kSPL], dA_acc[kSPL];
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int n = kSPL * r + i;
            g[i] = (valid && p.dlast && n < N && MSCAN_WITHIN(p.x_dlast, p.dlast + (b * Dm + dc) * N + n, 4, kSiteLastState))
                       ? (HS)p.dlast[(b * Dm + dc) * N + n] : (HS)0.f;
            dA_acc[i] = 0.f;
        }
        HS dD_acc = 0.f, dbias_acc = 0.f;
        // this lane's slot of the warp's channel-summed dB / dC: lanes c < 4
        // hold dB of state 4 r + c, lanes c >= 4 dC of state 4 r + c - 4
        const int kslot = (c < 4 ? 0 : 16) + kSPL * r + (c & 3);
        int rbuf = 0;  // which red buffer the next window uses
        fetch(p.n_sup - 1, true);
        for (int s = p.n_sup - 1; s >= 0; --s) {
            const int64_t t0 = (int64_t)s * kSup;
            const int tn = seg_len(s);
            // the segment's checkpoint, loaded before the staging work that
            // hides its latency (channels past dim have no checkpoint of the
            // forward's: zeros)
            const float4 ckv = (valid && MSCAN_WITHIN(p.x_ckpt, ck + (int64_t)s * kCkCh * kNS, 16, kSiteCkpt))
                                   ? __ldcg(reinterpret_cast<const float4 *>(ck + (int64_t)s * kCkCh * kNS))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            __syncthreads();  // raw landed; sx, sbc, outs of the previous segment consumed
            convert(s, true);
            __syncthreads();  // converted; the raw buffer is free
            if (s > 0) fetch(s - 1, true);
            // recompute the segment from its checkpoint, one sub-checkpoint every kSub steps
            {
                HS h[kSPL] = {(HS)ckv.x, (HS)ckv.y, (HS)ckv.z, (HS)ckv.w};
                for (int j = 0; j * kSub < tn; ++j) {
                    if (MSCAN_WITHIN(p.x_subck, sub + j * (kWarpsBwd * 32) * kSPL, kSPL * sizeof(HS), kSiteCarry))
                        store4(sub + j * (kWarpsBwd * 32) * kSPL, h);
#pragma unroll
                    for (int w = 0; w < kSub; ++w) step(h, j * kSub + w);
                }
            }
            // windows of kSub steps, last first: states and decays into
            // registers, then the reverse steps from them.  A window's
            // sub-checkpoint (this thread's own store, in L2) is loaded one
            // window ahead.
            HS hnext[kSPL] = {};
            auto load_sub = [&](int j) {
                if (MSCAN_WITHIN(p.x_subck, sub + j * (kWarpsBwd * 32) * kSPL, kSPL * sizeof(HS), kSiteCarry)) {
                    load4(sub + j * (kWarpsBwd * 32) * kSPL, hnext);
                } else {
#pragma unroll
                    for (int i = 0; i < kSPL; ++i) hnext[i] = (HS)0.f;
                }
            };
            load_sub((tn - 1) / kSub);
            for (int j = (tn - 1) / kSub; j >= 0; --j) {
                const int tb = j * kSub;
                HS hin[kSPL], hs[kSub][kSPL];
                // the decays: Abar (bf16 activations), or Abar - 1 (from the
                // near-zero polynomial, else the exponential) with fp32
                // activations, so the adjoint decays with the state's accuracy
                float ab[kSub][kSPL];
#pragma unroll
                for (int i = 0; i < kSPL; ++i) hin[i] = hnext[i];
                if (j > 0) load_sub(j - 1);
#pragma unroll
                for (int w = 0; w < kSub; ++w) {
                    {
                        const int t = tb + w;
                        const float2 rec = *reinterpret_cast<const float2 *>(srec + t * kCh + cb);
                        const float dl = rec.x;
                        const float du = dl * rec.y;
                        const float4 bb = *reinterpret_cast<const float4 *>(sbc + t * 2 * kNS + kSPL * r);
                        const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
                        if constexpr (ACC) {
#pragma unroll
                            for (int i = 0; i < kSPL; ++i) {
                                const HS prev = w == 0 ? hin[i] : hs[w - 1][i];
                                const float x = dl * A2[i];
                                ab[w][i] = Dk::near_one(x) ? expm1_poly(x) : __expf(x) - 1.f;
                                hs[w][i] = Dk::step(x, prev, du * bv[i]);
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < kSPL / 2; ++k) {
                                const float2 prev = w == 0 ? f2(hin[2 * k], hin[2 * k + 1])
                                                           : f2(hs[w - 1][2 * k], hs[w - 1][2 * k + 1]);
                                const float2 x = __fmul2_rn(f2(dl, dl), f2(A2[2 * k], A2[2 * k + 1]));
                                const float2 a = f2(ex2_mufu(x.x), ex2_mufu(x.y));
                                const float2 hn =
                                    __ffma2_rn(a, prev, __fmul2_rn(f2(du, du), f2(bv[2 * k], bv[2 * k + 1])));
                                ab[w][2 * k] = a.x;
                                ab[w][2 * k + 1] = a.y;
                                hs[w][2 * k] = hn.x;
                                hs[w][2 * k + 1] = hn.y;
                            }
                        }
                    }
                }
                float *rb = red + rbuf * (kSub * kWarpsBwd * 32);
                HS part[kSub][3];  // per step: this lane's share of C h, S_A, S_B
#pragma unroll
                for (int w = kSub - 1; w >= 0; --w) {
                    const int t = tb + w;
                    const float4 rec = srec[t * kCh + cb];
                    const float dl = rec.x, ut = rec.y, dy = rec.z;
                    const float4 bb = *reinterpret_cast<const float4 *>(sbc + t * 2 * kNS + kSPL * r);
                    const float4 cq = *reinterpret_cast<const float4 *>(sbc + t * 2 * kNS + kNS + kSPL * r);
                    const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cq.x, cq.y, cq.z, cq.w};
                    HS yp = 0.f, sA = 0.f, sB = 0.f;
                    float v[8];  // dB (0-3) and dC (4-7) terms of this lane's states
                    const float dlu = dl * ut;
                    if constexpr (ACC) {
#pragma unroll
                        for (int i = 0; i < kSPL; ++i) {
                            const HS hc = hs[w][i];
                            const HS hp = w == 0 ? hin[i] : hs[w - 1][i];
                            yp = fma((HS)cv[i], hc, yp);
                            const HS gq = fma((HS)dy, (HS)cv[i], g[i]);   // g'
                            const HS gab = fma(gq, (HS)ab[w][i], gq);     // g' + (Abar - 1) g'
                            const HS gha = gab * hp;                      // g' Abar h_{t-1}
                            sA = fma(gha, (HS)Ar[i], sA);
                            sB = fma(gq, (HS)bv[i], sB);
                            dA_acc[i] = fma(gha, (HS)dl, dA_acc[i]);
                            v[i] = (float)gq * dlu;
                            v[4 + i] = dy * (float)hc;
                            g[i] = gab;
                        }
                    } else {  // state pairs on the packed x2 instructions
                        float2 yp2 = f2(0.f, 0.f), sA2 = f2(0.f, 0.f), sB2 = f2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < kSPL / 2; ++k) {
                            const int i0 = 2 * k, i1 = 2 * k + 1;
                            const float2 hc = f2(hs[w][i0], hs[w][i1]);
                            const float2 hp = w == 0 ? f2(hin[i0], hin[i1]) : f2(hs[w - 1][i0], hs[w - 1][i1]);
                            const float2 c2 = f2(cv[i0], cv[i1]);
                            yp2 = __ffma2_rn(c2, hc, yp2);
                            const float2 gq = __ffma2_rn(f2(dy, dy), c2, f2(g[i0], g[i1]));   // g'
                            const float2 gab = __fmul2_rn(gq, f2(ab[w][i0], ab[w][i1]));
                            const float2 gha = __fmul2_rn(gab, hp);                          // g' Abar h_{t-1}
                            sA2 = __ffma2_rn(gha, f2(Ar[i0], Ar[i1]), sA2);
                            sB2 = __ffma2_rn(gq, f2(bv[i0], bv[i1]), sB2);
                            const float2 da = __ffma2_rn(gha, f2(dl, dl), f2(dA_acc[i0], dA_acc[i1]));
                            const float2 vb = __fmul2_rn(gq, f2(dlu, dlu));
                            const float2 vc = __fmul2_rn(f2(dy, dy), hc);
                            dA_acc[i0] = da.x; dA_acc[i1] = da.y;
                            v[i0] = vb.x; v[i1] = vb.y;
                            v[4 + i0] = vc.x; v[4 + i1] = vc.y;
                            g[i0] = gab.x; g[i1] = gab.y;
                        }
                        yp = yp2.x + yp2.y;
                        sA = sA2.x + sA2.y;
                        sB = sB2.x + sB2.y;
                    }
                    ChannelTranspose<16, 8>::run(v, lane);
                    rb[(w * kWarpsBwd + wib) * 32 + kslot] = v[0];
                    part[w][0] = yp;
                    part[w][1] = sA;
                    part[w][2] = sB;
                }
                // the channel's sums over its states, transposed over the
                // window: lane r ends with the totals of step tb + r and
                // forms that step's outputs, dD and dbias terms
                QuadTranspose<HS>::run(part, lane);
                {
                    const int t = tb + r;
                    const float4 rec = srec[t * kCh + cb];
                    const float dl = rec.x, ut = rec.y, dy = rec.z;
                    const float y = (float)part[0][0] + Dd * ut;
                    const float SA = (float)part[0][1], SBs = (float)part[0][2];
                    const float ddelta = fmaf(ut, SBs, SA);
                    const float ddraw = ddelta * ssig[t * kCh + cb];
                    dbias_acc += (HS)ddraw;
                    dD_acc = fma((HS)dy, (HS)ut, dD_acc);
                    outs[(0 * kCh + cb) * RP + t] = T(fmaf(dy, Dd, dl * SBs));
                    outs[(1 * kCh + cb) * RP + t] = T(ddraw);
                    if (GATE) outs[(2 * kCh + cb) * RP + t] = T(y * rec.w);
                }
                __syncthreads();  // the window's dB / dC terms of every warp are in rb
                // dB / dC of the window: thread -> (step, slot), the warps summed in order
                {
                    const int w = tid >> 5, slot = tid & 31;
                    const int n = slot & 15;
                    if (w < kSub && tb + w < tn && n < N) {
                        float acc = 0.f;
#pragma unroll
                        for (int k = 0; k < kWarpsBwd; ++k) acc += rb[(w * kWarpsBwd + k) * 32 + slot];
                        float *dst = p.rep + (((grp % kRep) * 2 + (slot >> 4)) * p.batch + b) * (int64_t)kNS * L +
                                     (int64_t)n * L + t0 + tb + w;
                        if (MSCAN_WITHIN(p.x_rep, dst, 4, kSiteCarry)) atomicAdd(dst, acc);
                    }
                }
                rbuf ^= 1;  // the next window fills the other buffer while this one is read
            }
            __syncthreads();  // every output of the segment is staged
            // du, ddelta_raw, dz rows of the segment: thread -> (quantity, channel, copy)
            for (int i = tid; i < 3 * kCh * CPR; i += kWarpsBwd * 32) {
                const int q = i / (kCh * CPR), rem = i % (kCh * CPR);
                const int cc = rem / CPR, cp = rem % CPR;
                if (q == 2 && !GATE) continue;
                if (d0 + cc >= Dm) continue;
                T *dst = gdst[q] + (b * Dm + d0 + cc) * L + t0 + cp * V;
                const T *srcp = outs + (q * kCh + cc) * RP + cp * V;
                if (p.vec) {
                    if (cp * V < tn && MSCAN_WITHIN(p.x_dout3[q], dst, 16, kSiteOut))
                        *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(srcp);
                } else {
#pragma unroll
                    for (int e = 0; e < V; ++e)
                        if (cp * V + e < tn && MSCAN_WITHIN(p.x_dout3[q], dst + e, sizeof(T), kSiteOut)) dst[e] = srcp[e];
                }
            }
        }
        if (valid) {
#pragma unroll
            for (int i = 0; i < kSPL; ++i) {
                const int n = kSPL * r + i;
                if (n < N) {
                    if (MSCAN_WITHIN(p.x_dA, p.dA + dc * N + n, 4, kSiteA)) atomicAdd(p.dA + dc * N + n, (float)dA_acc[i]);
                    if (p.dh0 && MSCAN_WITHIN(p.x_dh0, p.dh0 + (b * Dm + dc) * N + n, 4, kSiteH0))
                        p.dh0[(b * Dm + dc) * N + n] = (float)g[i];  // dL/dh_{-1}
                }
            }
        }
        // each lane summed dD and dbias over its step of every window
        dD_acc = quad_sum(dD_acc);
        dbias_acc = quad_sum(dbias_acc);
        if (valid && r == 0) {
            if (p.dD && MSCAN_WITHIN(p.x_dD, p.dD + dc, 4, kSiteD)) atomicAdd(p.dD + dc, (float)dD_acc);
            if (p.dbias && MSCAN_WITHIN(p.x_dbias, p.dbias + dc, 4, kSiteBias)) atomicAdd(p.dbias + dc, (float)dbias_acc);
        }
        __syncthreads();  // before the next group reuses shared memory
    }
}

// dB / dC = the sum of the kRep copies, for states n < N: one thread per
// (B or C, batch row, state, 4 timesteps).
__global__ void __launch_bounds__(256) bwd_sum_copies_kernel(const BwdParams p) {
    const int64_t L = p.seqlen, N = p.dstate;
    const int64_t q4 = (L + 3) / 4;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * p.batch * N * q4) return;
    const int64_t tq = i % q4, rest = i / q4;
    const int64_t n = rest % N, wb = rest / N;  // wb = which * batch + b
    const int64_t which = wb / p.batch, b = wb % p.batch;
    float *dst = (which ? p.dC : p.dB) + (b * N + n) * L;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int64_t t = tq * 4 + e;
        if (t >= L) break;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < kRep; ++k) {
            const float *q = p.rep + ((k * 2 + which) * p.batch + b) * (int64_t)kNS * L + n * L + t;
            acc += MSCAN_WITHIN(p.x_rep, q, 4, kSiteCarry) ? __ldcg(q) : 0.f;
        }
        if (MSCAN_WITHIN(which ? p.x_dC : p.x_dB, dst + t, 4, which ? kSiteC : kSiteB)) dst[t] = acc;
    }
}

template <typename T, bool SP, bool GATE, int WARPS>
cudaError_t launch_w(const BwdParams &p, int sm_count, cudaStream_t st) {
    static_assert((BwdSmem<T, WARPS>::BYTES + 1024) * kBwdBlocksPerSM[sizeof(T) == 4][WARPS == 6] <= 228 * 1024,
                  "the blocks per SM of the launch bounds fit in shared memory");
    auto kern = scan_bwd_kernel<T, SP, GATE, WARPS>;
    const int smem = BwdSmem<T, WARPS>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, WARPS * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sm_count * per_sm;  // one block per channel group, grid-strided
    if (grid > p.n_groups) grid = p.n_groups;
    kern<<<(unsigned)grid, WARPS * 32, smem, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t items = 2 * p.batch * p.dstate * ((p.seqlen + 3) / 4);
    const int64_t blocks = (items + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    bwd_sum_copies_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename T, bool SP, bool GATE>
cudaError_t launch_t(const BwdParams &p, int warps, int sm_count, cudaStream_t st) {
    return warps == 6 ? launch_w<T, SP, GATE, 6>(p, sm_count, st) : launch_w<T, SP, GATE, 4>(p, sm_count, st);
}

template <typename T>
cudaError_t launch_typed(const BwdParams &p, int warps, int sm_count, cudaStream_t st) {
    const bool gate = p.z != nullptr;
    if (p.softplus)
        return gate ? launch_t<T, true, true>(p, warps, sm_count, st) : launch_t<T, true, false>(p, warps, sm_count, st);
    return gate ? launch_t<T, false, true>(p, warps, sm_count, st) : launch_t<T, false, false>(p, warps, sm_count, st);
}

// Warps per block.  A channel group's adjoint runs through the sequence in
// order, so the groups are the units of work and the SM that holds the most
// of them sets the time: of the block sizes whose blocks are all resident at
// once (kBwdBlocksPerSM per SM), pick the one whose busiest SM carries the
// fewest warps.  Mamba-2.8B layer: 640 groups of 32 channels do not fit (592
// resident); 428 of 48 do (3 per SM: 18 warps).
int bwd_warps(int64_t batch, int64_t dim, int act, int sm_count) {
    const int f32 = act == kBF16 ? 0 : 1;
    const int64_t g4 = batch * ((dim + 31) / 32), g6 = batch * ((dim + 47) / 48);
    const bool fit4 = g4 <= (int64_t)sm_count * kBwdBlocksPerSM[f32][0];
    const bool fit6 = g6 <= (int64_t)sm_count * kBwdBlocksPerSM[f32][1];
    if (fit4 && fit6) {
        const int64_t load4 = 4 * ((g4 + sm_count - 1) / sm_count), load6 = 6 * ((g6 + sm_count - 1) / sm_count);
        return load6 < load4 ? 6 : 4;
    }
    return fit6 ? 6 : 4;
}

}  // namespace

int64_t scan_bwd_ckpt_floats(int64_t batch, int64_t dim, int64_t seqlen) {
    const int64_t groups = batch * ((dim + kCkCh - 1) / kCkCh);
    return groups * ((seqlen + kSup - 1) / kSup) * kCkCh * kNS;
}

int scan_bwd_ckpt_interval() { return kSup; }

namespace {
struct BwdLayout {
    size_t ck, sub, rep, bytes;  // offsets of the checkpoints, sub-checkpoints, dB / dC copies
};
BwdLayout bwd_layout(int64_t batch, int64_t dim, int64_t seqlen) {
    // threads over all groups, for either block size (4 warps: 32 channels per group, 6: 48)
    const int64_t t4 = ((dim + 31) / 32) * 128, t6 = ((dim + 47) / 48) * 192;
    const int64_t threads = batch * (t4 > t6 ? t4 : t6);
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    BwdLayout l;
    l.ck = 0;
    l.sub = up((size_t)scan_bwd_ckpt_floats(batch, dim, seqlen) * 4);
    // sub-checkpoints: per group, kNSub x (its threads) x 4 states of up to 8 bytes
    l.rep = l.sub + up((size_t)(threads * kNSub * kSPL) * 8);
    l.bytes = l.rep + (size_t)(kRep * 2 * batch * kNS * seqlen) * 4;
    return l;
}
}  // namespace

MSCAN_BOUNDS_TAKE(bwd_bounds_take)

size_t scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen) {
    return bwd_layout(batch, dim, seqlen).bytes;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs &a, void *workspace, const float *ckpt, int sm_count,
                            cudaStream_t st) {
    BwdParams p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z; p.dout = a.dout;
    p.A = a.A; p.D = a.D; p.delta_bias = a.delta_bias; p.dlast = a.dlast; p.h0 = a.h0;
    p.du = a.du; p.ddelta = a.ddelta; p.dz = a.dz;
    p.dA = a.dA; p.dB = a.dB; p.dC = a.dC; p.dD = a.dD; p.dbias = a.ddelta_bias; p.dh0 = a.dh0;
    const BwdLayout l = bwd_layout(a.batch, a.dim, a.seqlen);
    unsigned char *w = static_cast<unsigned char *>(workspace);
    p.ckpt = ckpt ? const_cast<float *>(ckpt) : reinterpret_cast<float *>(w + l.ck);
    p.ckpt_given = ckpt ? 1 : 0;
    p.subck = w + l.sub;
    p.rep = reinterpret_cast<float *>(w + l.rep);
    {
        const int es = a.act == kBF16 ? 2 : 4, V = 16 / es;
        auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
        p.vec = (a.seqlen % V == 0) && al(a.u) && al(a.delta) && al(a.z) && al(a.dout) && al(a.B) && al(a.C) &&
                al(a.du) && al(a.ddelta) && al(a.dz);
    }
    p.batch = a.batch; p.dim = a.dim; p.seqlen = a.seqlen; p.dstate = a.dstate; p.softplus = a.softplus;
    const int warps = bwd_warps(a.batch, a.dim, a.act, sm_count);
    const int ch = warps * kCPW;
    p.groups_per_batch = (int)((a.dim + ch - 1) / ch);
    p.ckpt_g32 = (int)((a.dim + kCkCh - 1) / kCkCh);
    p.n_groups = (int)(a.batch * p.groups_per_batch);
    p.n_sup = (int)((a.seqlen + kSup - 1) / kSup);
#ifdef MSCAN_BOUNDS_CHECK
    {  // byte ranges (bounds-checked build)
        const unsigned long long es = a.act == kBF16 ? 2 : 4;
        const unsigned long long x = (unsigned long long)(a.batch * a.dim * a.seqlen) * es;
        const unsigned long long bc = (unsigned long long)(a.batch * a.dstate * a.seqlen) * es;
        const unsigned long long stb = (unsigned long long)(a.batch * a.dim * a.dstate) * 4;
        const unsigned long long ob = x > (unsigned long long)g_out_extent_shrink ? x - g_out_extent_shrink : 0;
        p.x_in[0] = extent_of(a.u, x);
        p.x_in[1] = extent_of(a.delta, x);
        p.x_in[2] = extent_of(a.dout, x);
        p.x_in[3] = extent_of(a.z, x);
        p.x_in[4] = extent_of(a.B, bc);
        p.x_in[5] = extent_of(a.C, bc);
        p.x_A = extent_of(a.A, (unsigned long long)(a.dim * a.dstate) * 4);
        p.x_D = extent_of(a.D, (unsigned long long)a.dim * 4);
        p.x_bias = extent_of(a.delta_bias, (unsigned long long)a.dim * 4);
        p.x_dlast = extent_of(a.dlast, stb);
        p.x_h0 = extent_of(a.h0, stb);
        p.x_dout3[0] = extent_of(a.du, ob);
        p.x_dout3[1] = extent_of(a.ddelta, ob);
        p.x_dout3[2] = extent_of(a.dz, ob);
        p.x_dA = extent_of(a.dA, (unsigned long long)(a.dim * a.dstate) * 4);
        p.x_dB = extent_of(a.dB, (unsigned long long)(a.batch * a.dstate * a.seqlen) * 4);
        p.x_dC = extent_of(a.dC, (unsigned long long)(a.batch * a.dstate * a.seqlen) * 4);
        p.x_dD = extent_of(a.dD, (unsigned long long)a.dim * 4);
        p.x_dbias = extent_of(a.ddelta_bias, (unsigned long long)a.dim * 4);
        p.x_dh0 = extent_of(a.dh0, stb);
        p.x_ckpt = extent_of(p.ckpt, (unsigned long long)scan_bwd_ckpt_floats(a.batch, a.dim, a.seqlen) * 4);
        p.x_subck = extent_of(p.subck, l.rep - l.sub);
        p.x_rep = extent_of(p.rep, l.bytes - l.rep);
    }
#endif
    // every sum over channels, time or batch rows accumulates into zeroed outputs
    cudaError_t e = cudaMemsetAsync(a.dA, 0, (size_t)(a.dim * a.dstate) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.rep, 0, l.bytes - l.rep, st);
    if (e == cudaSuccess && a.dD) e = cudaMemsetAsync(a.dD, 0, (size_t)a.dim * 4, st);
    if (e == cudaSuccess && a.ddelta_bias) e = cudaMemsetAsync(a.ddelta_bias, 0, (size_t)a.dim * 4, st);
    if (e != cudaSuccess) return e;
    return a.act == kBF16 ? launch_typed<__nv_bfloat16>(p, warps, sm_count, st)
                          : launch_typed<float>(p, warps, sm_count, st);
}

}  // namespace mscan
