// scan_bwd.cu -- backward pass of the selective scan (S6): the gradients of
// the forward in scan_fwd*.cu with respect to every input, given dL/dout and
// (optionally) dL/dlast_state.  Reverse-mode differentiation of the
// recurrence h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t,
// y_t = C_t h_t + D u_t, out_t = y_t silu(z_t) (training the layer
// back-propagates through the scan; the Mamba paper's hardware-aware
// algorithm, Section 3.3, recomputes the states in the backward pass rather
// than storing them).  With g = dL/dh_t carried backwards:
//   dy = dout silu(z);  dz = dout y silu'(z);  dD += dy u;  du = dy D
//   dC[n,t] += dy h_t[n];  g[n] += dy C[n,t]
//   ddelta += g[n] (h_{t-1}[n] Abar A[n] + B[n,t] u);  dA[n] += g[n] h_{t-1}[n] Abar delta
//   dB[n,t] += g[n] delta u;  du += g[n] delta B[n,t];  g[n] *= Abar
//   ddelta_raw = ddelta sigmoid(delta_raw + bias) (softplus);  dbias += ddelta_raw
// and, when the forward started from a given state h0, dh0 = g after t = 0.
//
// Design.  A block of four warps takes a group of 32 channels of one batch
// row through the whole sequence, twice: forward, storing the state every
// kSeg timesteps in the workspace (the checkpoints), then backward segment
// by segment from the end: each segment's inputs are staged once for the
// block in shared memory (B and C widened to fp32 [t][n] for broadcast
// reads; u, delta, sigmoid, z and dout per channel), its states recomputed
// from the checkpoint into shared memory and consumed in reverse.  Four
// lanes share a channel, four states each, so a group is four warps and
// each SM sub-partition holds several -- the reverse sweep is a long chain of
// dependent steps, and the warps hide each other's latency.  Per-channel
// sums over states (the readout, ddelta, du) are shuffles among a channel's
// lanes.  dB and dC are sums over all channels of a batch row: each warp sums
// its 8 channels with a transposed shuffle reduction, the block adds its
// warps in a fixed order and stores the group's partial sum; a second kernel
// adds the groups of each batch row in a fixed order.  dA, dD and dbias are
// summed over a group's whole sequence in registers and added once per
// group with atomics.  fp32 activations take the accurate decay, softplus and
// sigmoid (Decay<true> of device_math.cuh: the state and the adjoint advance
// by (Abar - 1) x + b, Abar - 1 on the FMA pipe), bf16 ones one ex2 per decay.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kNS = 16;       // padded states per channel (dstate <= 16)
constexpr int kSeg = 8;       // timesteps between checkpoints
constexpr int kWarpsBwd = 4;  // warps per block

struct BwdParams {
    const void *u, *delta, *B, *C, *z, *dout;
    const float *A, *D, *delta_bias, *dlast, *h0;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *dbias, *dh0;
    float *ckpt;  // workspace: n_groups x n_segs x 32 lanes x kNS checkpointed states
    float *part;  // workspace: n_groups x seqlen x 32 partial dB (lanes 0-15) / dC (16-31) sums
    int vec;      // rows 16-byte aligned and a whole number of 16-byte chunks
    int64_t batch, dim, seqlen;
    int dstate, softplus;
    int groups_per_batch, n_groups, n_segs;
};

// Lane layout.  A block of kWarpsBwd warps owns one group of 32 channels of
// one batch row; in a warp, lane = 4 c + r takes channel c (of the warp's 8)
// and states 4 r .. 4 r + 3.  Sums over a channel's states are shuffles
// among its 4 lanes; sums over channels (dB, dC) are shuffles among the 8
// lanes with the same r, then shared memory across the block's warps.
constexpr int kCPW = 8;  // channels per warp
constexpr int kSPL = 4;  // states per lane

// Shared memory per block (floats): per warp the recomputed states after
// each step of the segment [step][lane][4 states]; the segment's B and C rows
// widened to fp32 [t][state] (C 16 floats after B's end, so the widening
// stores are free of bank conflicts); per warp the channels' per-timestep
// values [quantity][t][channel]; per warp the dB / dC partial sums [t][32].
enum { X_U, X_DL, X_SIG, X_Z, X_DOUT, X_SGZ, X_N };  // X_SIG: sigmoid(delta_raw + bias), X_SGZ: sigmoid(z)
constexpr int kHistW = (kSeg + 1) * 32 * kSPL;
constexpr int kBC = 2 * kSeg * kNS + 16;
constexpr int kXW = X_N * kSeg * kCPW;
constexpr int kRedW = kSeg * 32;
constexpr int kOutW = 3 * kSeg * kCPW;  // per warp: du, ddelta_raw, dz [q][t][channel]
// raw rows in flight, per stage: 32 B / C rows and 32 x 4 (channel, quantity)
// rows of kSeg elements, sized for fp32 (bf16 uses half)
constexpr int kRawRows = 32 + kWarpsBwd * 32;
constexpr int kRawStage = kRawRows * kSeg;  // elements of T per stage (room reserved as floats)
constexpr int kBlockFloats = kWarpsBwd * (kHistW + kXW + kRedW + kOutW) + kBC + 2 * kRawStage;

__device__ __forceinline__ void cp16_async(void *smem, const void *gmem, bool pred) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(sa), "l"(gmem), "r"(pred ? 16 : 0) : "memory");
}

// Sum v[] over the 8 lanes that share lane & 3, transposed: afterwards
// v[0] of lane 4 c + r holds the total of the lanes' original v[c].  Round K
// (lane bit 16, 8, 4) halves the live values; the lane with bit K set keeps
// the upper half.
template <int K, int CNT>
struct ChannelTranspose {
    __device__ __forceinline__ static void run(float (&v)[8], int lane) {
        constexpr int HALF = CNT / 2;
        const bool upper = (lane & K) != 0;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
            const float send = upper ? v[i] : v[i + HALF];
            const float keep = upper ? v[i + HALF] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, K);
        }
        ChannelTranspose<K / 2, HALF>::run(v, lane);
    }
};
template <int CNT>
struct ChannelTranspose<2, CNT> {
    __device__ __forceinline__ static void run(float (&)[8], int) {}
};

// 1 / (1 + e^-x): the MUFU form for bf16 activations, CUDA's full-precision
// expf and division for fp32 ones.
template <bool ACC>
__device__ __forceinline__ float sigmoid(float x) {
    if (ACC) return 1.f / (1.f + expf(-x));
    return __fdividef(1.f, 1.f + __expf(-x));
}

__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

template <typename T, bool SP, bool GATE>
__global__ void __launch_bounds__(kWarpsBwd * 32, 5) scan_bwd_kernel(const BwdParams p) {
    constexpr bool ACC = sizeof(T) == 4;
    using Dk = Decay<ACC>;
    extern __shared__ __align__(16) float bwd_smem[];
    const int tid = threadIdx.x, lane = tid & 31, wib = tid >> 5;
    const int c = lane >> 2, r = lane & 3;
    float4 *hist = reinterpret_cast<float4 *>(bwd_smem + wib * kHistW);       // [kSeg + 1][32]
    float *sB = bwd_smem + kWarpsBwd * kHistW;                                 // [t][n]
    float *sC = sB + kSeg * kNS + 16;                                          // [t][n]
    float *sxAll = sB + kBC;                                                   // [warp][q][t][c]
    float *redAll = sxAll + kWarpsBwd * kXW;                                   // [warp][t][32]
    float *sx = sxAll + wib * kXW;
    float *red = redAll + wib * kRedW;
    float *so = redAll + kWarpsBwd * kRedW + wib * kOutW;                      // [q][t][c]
    T *rawBase = reinterpret_cast<T *>(redAll + kWarpsBwd * (kRedW + kOutW));  // [2][kRawRows][kSeg]
    const int64_t L = p.seqlen;
    const int N = p.dstate;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B);
    const T *gC = static_cast<const T *>(p.C);
    const T *go = static_cast<const T *>(p.dout);
    T *gdu = static_cast<T *>(p.du);
    T *gdd = static_cast<T *>(p.ddelta);
    T *gdz = static_cast<T *>(p.dz);
    const bool vec = p.vec != 0;

    for (int64_t grp = blockIdx.x; grp < p.n_groups; grp += gridDim.x) {
        const int64_t b = grp / p.groups_per_batch;
        const int64_t d0 = (grp % p.groups_per_batch) * 32;
        const int64_t dc = d0 + wib * kCPW + c;  // this lane's channel
        const bool valid = dc < p.dim;
        const int64_t row = (b * p.dim + (valid ? dc : 0)) * L;
        float A2[kSPL], Ar[kSPL];
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int n = kSPL * r + i;
            Ar[i] = (valid && n < N) ? __ldg(p.A + dc * N + n) : 0.f;
            A2[i] = Ar[i] * Dk::kScale;
        }
        const float bias = (valid && p.delta_bias) ? __ldg(p.delta_bias + dc) : 0.f;
        const float Dd = (valid && p.D) ? __ldg(p.D + dc) : 0.f;
        // checkpoints: [group][segment][32 channels][16 states]; this lane's 4 states
        float *ck = p.ckpt + grp * (int64_t)p.n_segs * 32 * kNS + (wib * kCPW + c) * kNS + kSPL * r;

        // Staging of segment [t0, t0 + tn) for the whole block, in two halves.
        // fetch: the raw rows go to a double-buffered shared area with 16-byte
        // cp.async (element copies when rows are not 16-byte aligned), issued
        // one segment ahead so the copies overlap the current segment's work:
        // threads 0-31 copy a B (0-15) or C (16-31) row, every thread one
        // (channel, quantity) row -- 0 u, 1 delta, 2 dout, 3 z.  convert: each
        // thread, once its own copies have landed, widens its rows to fp32:
        // B / C into [t][n], u / delta (softplus, sigmoid) / dout / z into
        // each warp's sx[q][t][c].
        const int fch = tid & 31, fq = tid >> 5;
        const int64_t fd = d0 + fch;
        const bool fok = fd < p.dim;
        const T *fsrc = (fq == 0 ? gu : fq == 1 ? gd : fq == 2 ? go : gz) + (b * p.dim + (fok ? fd : 0)) * L;
        const float fbias = (fok && p.delta_bias) ? __ldg(p.delta_bias + fd) : 0.f;
        const int bwhich = tid >> 4, bn = tid & 15;
        const T *bsrc = (bwhich ? gC : gB) + (b * N + (bn < N ? bn : 0)) * L;
        auto fetch = [&](int64_t t0, int tn, bool full, int buf) {
            T *raw = rawBase + buf * kRawStage;
            auto copy_row = [&](T *dst, const T *src, bool ok) {
                if (vec) {
                    constexpr int V = 16 / (int)sizeof(T);
#pragma unroll
                    for (int q = 0; q < kSeg / V; ++q) {
                        const bool in = ok && q * V < tn;
                        cp16_async(dst + q * V, in ? src + q * V : src, in);
                    }
                } else {
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) dst[s] = (ok && s < tn) ? src[s] : T(0.f);
                }
            };
            if (tid < 32) copy_row(raw + tid * kSeg, bsrc + t0, bn < N && (full || bwhich == 0));
            if (fq < (full ? (GATE ? 4 : 3) : 2)) copy_row(raw + (32 + tid) * kSeg, fsrc + t0, fok);
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        auto convert = [&](bool full, int buf) {
            asm volatile("cp.async.wait_group 0;" ::: "memory");  // this thread's copies
            const T *raw = rawBase + buf * kRawStage;
            float f[kSeg];
            if (tid < 32) {
                const T *row = raw + tid * kSeg;
#pragma unroll
                for (int s = 0; s < kSeg; ++s) f[s] = Elem<T>::to_f(row[s]);
                float *dst = (bwhich ? sC : sB) + bn;
#pragma unroll
                for (int s = 0; s < kSeg; ++s) dst[s * kNS] = f[s];
            }
            if (fq < (full ? (GATE ? 4 : 3) : 2)) {
                const T *row = raw + (32 + tid) * kSeg;
#pragma unroll
                for (int s = 0; s < kSeg; ++s) f[s] = Elem<T>::to_f(row[s]);
                float *dst = sxAll + (fch >> 3) * kXW + (fch & 7);
                if (fq == 1) {
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) {
                        const float x = f[s] + fbias;
                        dst[(X_DL * kSeg + s) * kCPW] = SP ? Dk::softplus(x) : x;
                        if (full) dst[(X_SIG * kSeg + s) * kCPW] = SP ? sigmoid<ACC>(x) : 1.f;
                    }
                } else {
                    const int X = fq == 0 ? X_U : fq == 2 ? X_DOUT : X_Z;
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) dst[(X * kSeg + s) * kCPW] = f[s];
                    if (fq == 3) {
#pragma unroll
                        for (int s = 0; s < kSeg; ++s) dst[(X_SGZ * kSeg + s) * kCPW] = sigmoid<ACC>(f[s]);
                    }
                }
            }
        };
        // h <- the states after `tn` steps of the staged segment; into hist[1..] when asked
        auto advance = [&](float (&h)[kSPL], int tn, bool keep) {
#pragma unroll
            for (int s = 0; s < kSeg; ++s) {
                if (s >= tn) break;
                const float dl = sx[(X_DL * kSeg + s) * kCPW + c];
                const float du = dl * sx[(X_U * kSeg + s) * kCPW + c];
                const float4 bb = *reinterpret_cast<const float4 *>(sB + s * kNS + kSPL * r);
                const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int i = 0; i < kSPL; ++i) h[i] = Dk::step(dl * A2[i], h[i], du * bv[i]);
                if (keep) hist[(s + 1) * 32 + lane] = make_float4(h[0], h[1], h[2], h[3]);
            }
        };

        // ---- forward from h0 (or zeros): checkpoints every kSeg timesteps (state before the segment)
        float h[kSPL];
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int n = kSPL * r + i;
            h[i] = (valid && p.h0 && n < N) ? __ldg(p.h0 + (b * p.dim + dc) * N + n) : 0.f;
        }
        auto seg_len = [&](int seg) {
            const int64_t t0 = (int64_t)seg * kSeg;
            return (L - t0) < kSeg ? (int)(L - t0) : kSeg;
        };
        fetch(0, seg_len(0), false, 0);
        for (int seg = 0; seg < p.n_segs; ++seg) {
            __stcg(reinterpret_cast<float4 *>(ck + (int64_t)seg * 32 * kNS), make_float4(h[0], h[1], h[2], h[3]));
            __syncthreads();  // the previous segment's staging is consumed
            convert(false, seg & 1);
            if (seg + 1 < p.n_segs) fetch((int64_t)(seg + 1) * kSeg, seg_len(seg + 1), false, (seg + 1) & 1);
            __syncthreads();
            advance(h, seg_len(seg), false);
        }

        // ---- reverse sweep, segment by segment from the end
        float g[kSPL], dA_acc[kSPL];
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int n = kSPL * r + i;
            g[i] = (valid && p.dlast && n < N) ? p.dlast[(b * p.dim + dc) * N + n] : 0.f;
            dA_acc[i] = 0.f;
        }
        float dD_acc = 0.f, dbias_acc = 0.f;
        // this lane's slot of the warp's channel-summed dB / dC: lanes c < 4
        // hold dB of state 4 r + c, lanes c >= 4 dC of state 4 r + c - 4
        const int kslot = (c < 4 ? 0 : 16) + kSPL * r + (c & 3);
        fetch((int64_t)(p.n_segs - 1) * kSeg, seg_len(p.n_segs - 1), true, (p.n_segs - 1) & 1);
        for (int seg = p.n_segs - 1; seg >= 0; --seg) {
            const int64_t t0 = (int64_t)seg * kSeg;
            const int tn = seg_len(seg);
            __syncthreads();  // staging, hist and red of the previous segment are consumed
            convert(true, seg & 1);
            if (seg > 0) fetch(t0 - kSeg, seg_len(seg - 1), true, (seg - 1) & 1);
            {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(ck + (int64_t)seg * 32 * kNS));
                h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
            }
            __syncthreads();
            hist[lane] = make_float4(h[0], h[1], h[2], h[3]);
            advance(h, tn, true);
            __syncwarp();
            float4 hc4 = make_float4(h[0], h[1], h[2], h[3]);  // the state after the segment's last step
#pragma unroll
            for (int s = kSeg - 1; s >= 0; --s) {
                if (s >= tn) continue;
                const float dl = sx[(X_DL * kSeg + s) * kCPW + c];
                const float ut = sx[(X_U * kSeg + s) * kCPW + c];
                const float dout = sx[(X_DOUT * kSeg + s) * kCPW + c];
                const float4 hp4 = hist[s * 32 + lane];
                const float4 bb = *reinterpret_cast<const float4 *>(sB + s * kNS + kSPL * r);
                const float4 cc = *reinterpret_cast<const float4 *>(sC + s * kNS + kSPL * r);
                const float hcur[4] = {hc4.x, hc4.y, hc4.z, hc4.w}, hp[4] = {hp4.x, hp4.y, hp4.z, hp4.w};
                const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
                float yp = 0.f;
#pragma unroll
                for (int i = 0; i < kSPL; ++i) yp = fmaf(cv[i], hcur[i], yp);
                const float y = fmaf(Dd, ut, quad_sum(yp));
                float dy = dout;
                if (GATE) {
                    const float zt = sx[(X_Z * kSeg + s) * kCPW + c];
                    const float sg = sx[(X_SGZ * kSeg + s) * kCPW + c];
                    if (r == 0) so[(2 * kSeg + s) * kCPW + c] = dout * y * sg * fmaf(zt, 1.f - sg, 1.f);
                    dy = dout * zt * sg;
                }
                dD_acc = fmaf(dy, ut, dD_acc);
                float dut_p = 0.f, ddelta_p = 0.f;
                float v[8];  // dB (0-3) and dC (4-7) terms of this lane's states
#pragma unroll
                for (int i = 0; i < kSPL; ++i) {
                    v[4 + i] = dy * hcur[i];
                    g[i] = fmaf(dy, cv[i], g[i]);
                    const float xa = dl * A2[i];
                    const float ab = Dk::abar(xa);
                    const float gha = g[i] * hp[i] * ab;
                    ddelta_p = fmaf(gha, Ar[i], fmaf(g[i], bv[i] * ut, ddelta_p));
                    dA_acc[i] = fmaf(gha, dl, dA_acc[i]);
                    v[i] = g[i] * dl * ut;
                    dut_p = fmaf(g[i] * dl, bv[i], dut_p);
                    g[i] = ACC ? Dk::scale(xa, g[i]) : g[i] * ab;
                }
                ChannelTranspose<16, 8>::run(v, lane);
                red[s * 32 + kslot] = v[0];
                const float ddelta = quad_sum(ddelta_p);
                const float ddraw = ddelta * sx[(X_SIG * kSeg + s) * kCPW + c];
                dbias_acc += ddraw;
                const float dut = fmaf(dy, Dd, quad_sum(dut_p));
                if (r == 0) {
                    so[(0 * kSeg + s) * kCPW + c] = dut;
                    so[(1 * kSeg + s) * kCPW + c] = ddraw;
                }
                hc4 = hp4;
            }
            // this channel's rows of the segment: lane r = 0 du, 1 ddelta_raw,
            // 2 dz, 16 bytes at a time where possible
            __syncwarp();
            if (valid && r < (GATE ? 3 : 2)) {
                constexpr int V = 16 / (int)sizeof(T);
                T *dst = (r == 0 ? gdu : r == 1 ? gdd : gdz) + row + t0;
                float f[kSeg];
#pragma unroll
                for (int s = 0; s < kSeg; ++s) f[s] = so[(r * kSeg + s) * kCPW + c];
#pragma unroll
                for (int q = 0; q < kSeg / V; ++q) {
                    if (vec && (q + 1) * V <= tn) {
                        *reinterpret_cast<uint4 *>(dst + q * V) = Elem<T>::pack(f + q * V);
                    } else {
#pragma unroll
                        for (int e = 0; e < V; ++e)
                            if (q * V + e < tn) Elem<T>::store(dst + q * V + e, f[q * V + e]);
                    }
                }
            }
            // the block's dB / dC partial sums: the warps' sums added in warp order
            __syncthreads();
            float *part = p.part + (grp * L + t0) * 32;
            for (int idx = tid; idx < tn * 32; idx += kWarpsBwd * 32) {
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < kWarpsBwd; ++w) acc += redAll[w * kRedW + idx];
                __stcg(part + idx, acc);
            }
        }
        if (valid) {
#pragma unroll
            for (int i = 0; i < kSPL; ++i) {
                const int n = kSPL * r + i;
                if (n < N) {
                    atomicAdd(p.dA + dc * N + n, dA_acc[i]);
                    if (p.dh0) p.dh0[(b * p.dim + dc) * N + n] = g[i];  // dL/dh_{-1}
                }
            }
            if (r == 0) {
                if (p.dD) atomicAdd(p.dD + dc, dD_acc);
                if (p.dbias) atomicAdd(p.dbias + dc, dbias_acc);
            }
        }
        __syncthreads();  // before the next group reuses shared memory
    }
}

// dB[b,n,t] / dC[b,n,t] = sum over the groups of batch row b of their
// partial sums part[g][t][n] / part[g][t][16 + n]: one block per (b, 32
// timesteps) tile, the groups summed in registers, the tile transposed
// through shared memory so that both the reads and the writes are coalesced.
__global__ void __launch_bounds__(256) bwd_reduce_bc_kernel(const BwdParams p) {
    __shared__ float tile[32][33];
    const int64_t tiles_per_b = (p.seqlen + 31) / 32;
    const int64_t b = blockIdx.x / tiles_per_b;
    const int64_t t0 = (blockIdx.x % tiles_per_b) * 32;
    const int tx = threadIdx.x & 31, ty0 = threadIdx.x >> 5;  // 8 rows per pass
    const int N = p.dstate;
    for (int ty = ty0; ty < 32; ty += 8) {
        const int64_t t = t0 + ty;
        float acc = 0.f;
        if (t < p.seqlen) {
            const float *src = p.part + ((b * p.groups_per_batch) * p.seqlen + t) * 32 + tx;
            for (int gi = 0; gi < p.groups_per_batch; ++gi) acc += __ldcg(src + (int64_t)gi * p.seqlen * 32);
        }
        tile[ty][tx] = acc;
    }
    __syncthreads();
    for (int k = ty0; k < 32; k += 8) {  // k: (B or C, state) pair; tx: timestep in the tile
        const int n = k & 15;
        const int64_t t = t0 + tx;
        if (n < N && t < p.seqlen) (k < 16 ? p.dB : p.dC)[(b * N + n) * p.seqlen + t] = tile[tx][k];
    }
}

template <typename T, bool SP, bool GATE>
cudaError_t launch_t(const BwdParams &p, int sm_count, cudaStream_t st) {
    auto kern = scan_bwd_kernel<T, SP, GATE>;
    const int smem = kBlockFloats * 4;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpsBwd * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sm_count * per_sm;  // one block per channel group, grid-strided
    if (grid > p.n_groups) grid = p.n_groups;
    kern<<<(unsigned)grid, kWarpsBwd * 32, smem, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t blocks = p.batch * ((p.seqlen + 31) / 32);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    bwd_reduce_bc_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const BwdParams &p, int sm_count, cudaStream_t st) {
    const bool gate = p.z != nullptr;
    if (p.softplus) return gate ? launch_t<T, true, true>(p, sm_count, st) : launch_t<T, true, false>(p, sm_count, st);
    return gate ? launch_t<T, false, true>(p, sm_count, st) : launch_t<T, false, false>(p, sm_count, st);
}

}  // namespace

size_t scan_bwd_workspace_bytes(int64_t batch, int64_t dim, int64_t seqlen) {
    const int64_t groups = batch * ((dim + 31) / 32);
    const int64_t segs = (seqlen + kSeg - 1) / kSeg;
    return (size_t)(groups * segs * 32 * kNS) * 4 + (size_t)(groups * seqlen * 32) * 4;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs &a, void *workspace, int sm_count, cudaStream_t st) {
    BwdParams p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z; p.dout = a.dout;
    p.A = a.A; p.D = a.D; p.delta_bias = a.delta_bias; p.dlast = a.dlast; p.h0 = a.h0;
    p.du = a.du; p.ddelta = a.ddelta; p.dz = a.dz;
    p.dA = a.dA; p.dB = a.dB; p.dC = a.dC; p.dD = a.dD; p.dbias = a.ddelta_bias; p.dh0 = a.dh0;
    p.ckpt = static_cast<float *>(workspace);
    p.part = p.ckpt + (size_t)((a.batch * ((a.dim + 31) / 32)) * ((a.seqlen + kSeg - 1) / kSeg)) * 32 * kNS;
    {
        const int es = a.act == kBF16 ? 2 : 4, V = 16 / es;
        auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
        p.vec = (a.seqlen % V == 0) && al(a.u) && al(a.delta) && al(a.z) && al(a.dout) && al(a.B) && al(a.C) &&
                al(a.du) && al(a.ddelta) && al(a.dz);
    }
    p.batch = a.batch; p.dim = a.dim; p.seqlen = a.seqlen; p.dstate = a.dstate; p.softplus = a.softplus;
    p.groups_per_batch = (int)((a.dim + 31) / 32);
    p.n_groups = (int)(a.batch * p.groups_per_batch);
    p.n_segs = (int)((a.seqlen + kSeg - 1) / kSeg);
    // the sums over channels and time accumulate into zeroed outputs
    cudaError_t e = cudaMemsetAsync(a.dA, 0, (size_t)(a.dim * a.dstate) * 4, st);
    if (e == cudaSuccess && a.dD) e = cudaMemsetAsync(a.dD, 0, (size_t)a.dim * 4, st);
    if (e == cudaSuccess && a.ddelta_bias) e = cudaMemsetAsync(a.ddelta_bias, 0, (size_t)a.dim * 4, st);
    if (e != cudaSuccess) return e;
    return a.act == kBF16 ? launch_typed<__nv_bfloat16>(p, sm_count, st) : launch_typed<float>(p, sm_count, st);
}

}  // namespace mscan
