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
// Design.  One lane per channel with all (<= 16) states in registers; a warp
// takes a group of 32 channels of one batch row through the whole sequence,
// twice: forward, storing the state every kSeg timesteps in the workspace
// (the checkpoints), then backward segment by segment from the end: each
// segment's inputs are staged in shared memory (B and C widened to fp32
// [t][n] for broadcast reads, the lane's own u, delta, sigmoid, z and dout),
// its states recomputed from the checkpoint into shared memory and consumed
// in reverse.  dB and dC are sums over all channels of a batch row: each warp
// sums its 32 channels with a transposed shuffle reduction that leaves lane l
// the total for one (B or C, state) pair and stores it as the group's partial
// sum; a second kernel adds the groups of each batch row in a fixed order.
// dA, dD and dbias are summed over a group's whole sequence in registers and
// added once per group with atomics.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kNS = 16;       // states per lane (dstate <= 16)
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

// Sum v[i] over the 32 lanes, transposed: afterwards v[0] of lane l holds the
// warp total of the lanes' original v[l].
template <int K, int CNT>
struct WarpTranspose {
    __device__ __forceinline__ static void run(float (&v)[32], int lane) {
        constexpr int HALF = CNT / 2;
        const bool upper = (lane & K) != 0;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
            const float send = upper ? v[i] : v[i + HALF];
            const float keep = upper ? v[i + HALF] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, K);
        }
        WarpTranspose<K / 2, HALF>::run(v, lane);
    }
};
template <int CNT>
struct WarpTranspose<0, CNT> {
    __device__ __forceinline__ static void run(float (&)[32], int) {}
};

// Per-warp shared memory (floats): recomputed states [step][state][lane],
// the segment's B and C rows widened to fp32 [t][state] (C 16 floats after
// B's end, so the widening stores are free of bank conflicts), and this
// lane's per-timestep values [quantity][t][lane].
constexpr int kHist = (kSeg + 1) * kNS * 32;
constexpr int kBC = 2 * kSeg * kNS + 16;
enum { X_U, X_DL, X_SIG, X_Z, X_DOUT, X_N };
constexpr int kX = X_N * kSeg * 32;
constexpr int kWarpFloats = kHist + kBC + kX;

template <typename T>
__device__ __forceinline__ void load_row16(const T *src, int tn, float (&f)[kSeg]) {
    constexpr int V = 16 / (int)sizeof(T);
#pragma unroll
    for (int c = 0; c < kSeg / V; ++c) {
        if (c * V < tn) Elem<T>::unpack(ldg16(src + c * V), f + c * V);
        else {
#pragma unroll
            for (int e = 0; e < V; ++e) f[c * V + e] = 0.f;
        }
    }
}

template <typename T, bool SP, bool GATE>
__global__ void __launch_bounds__(kWarpsBwd * 32) scan_bwd_kernel(const BwdParams p) {
    extern __shared__ __align__(16) float bwd_smem[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    float *wsm = bwd_smem + wib * kWarpFloats;
    float(*hist)[kNS][32] = reinterpret_cast<float(*)[kNS][32]>(wsm);
    float *sB = wsm + kHist;                   // [t][n]
    float *sC = sB + kSeg * kNS + 16;          // [t][n]
    float(*sx)[kSeg][32] = reinterpret_cast<float(*)[kSeg][32]>(wsm + kHist + kBC);
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
    const int64_t total_warps = (int64_t)gridDim.x * kWarpsBwd;
    const bool vec = p.vec != 0;  // 16-byte row loads (aligned rows, whole chunks)

    for (int64_t grp = (int64_t)blockIdx.x * kWarpsBwd + wib; grp < p.n_groups; grp += total_warps) {
        const int64_t b = grp / p.groups_per_batch;
        const int64_t dc = (grp % p.groups_per_batch) * 32 + lane;
        const bool valid = dc < p.dim;
        const int64_t row = (b * p.dim + (valid ? dc : 0)) * L;  // this lane's channel row
        float A2[kNS], Ar[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) {
            Ar[n] = (valid && n < N) ? __ldg(p.A + dc * N + n) : 0.f;
            A2[n] = Ar[n] * kLog2e;
        }
        const float bias = (valid && p.delta_bias) ? __ldg(p.delta_bias + dc) : 0.f;
        const float Dd = (valid && p.D) ? __ldg(p.D + dc) : 0.f;
        float *ck = p.ckpt + grp * (int64_t)p.n_segs * 32 * kNS + lane * kNS;

        // Stage segment [t0, t0 + tn): B (and C) widened into [t][n]; this
        // lane's u, delta (after softplus), sigmoid(delta_raw) and, for the
        // backward, z and dout, into sx[.][t][lane].
        auto stage = [&](int64_t t0, int tn, bool full) {
            __syncwarp();
            {
                const int which = lane >> 4, n = lane & 15;  // lanes 0-15: B, 16-31: C
                float f[kSeg];
                if (n < N && (full || which == 0)) {
                    const T *src = (which ? gC : gB) + (b * N + n) * L + t0;
                    if (vec) load_row16<T>(src, tn, f);
                    else {
#pragma unroll
                        for (int s = 0; s < kSeg; ++s) f[s] = s < tn ? Elem<T>::load(src + s) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) f[s] = 0.f;
                }
                float *dst = (which ? sC : sB) + n;
#pragma unroll
                for (int s = 0; s < kSeg; ++s) dst[s * kNS] = f[s];
            }
            float fu[kSeg], fd[kSeg];
            const bool ok = valid;
            auto load_own = [&](const T *base, float (&f)[kSeg]) {
                if (ok && vec) load_row16<T>(base + row + t0, tn, f);
                else {
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) f[s] = (ok && s < tn) ? Elem<T>::load(base + row + t0 + s) : 0.f;
                }
            };
            load_own(gu, fu);
            load_own(gd, fd);
#pragma unroll
            for (int s = 0; s < kSeg; ++s) {
                const float x = fd[s] + bias;
                sx[X_U][s][lane] = fu[s];
                sx[X_DL][s][lane] = SP ? softplus_f(x) : x;
                if (full) sx[X_SIG][s][lane] = SP ? __fdividef(1.f, 1.f + __expf(-x)) : 1.f;
            }
            if (full) {
                load_own(go, fu);
#pragma unroll
                for (int s = 0; s < kSeg; ++s) sx[X_DOUT][s][lane] = fu[s];
                if (GATE) {
                    load_own(gz, fu);
#pragma unroll
                    for (int s = 0; s < kSeg; ++s) sx[X_Z][s][lane] = fu[s];
                }
            }
            __syncwarp();
        };
        // h <- the states after `tn` steps of the staged segment; into hist[1..] when asked
        auto advance = [&](float (&h)[kNS], int tn, bool keep) {
            for (int s = 0; s < tn; ++s) {
                const float dl = sx[X_DL][s][lane];
                const float du = dl * sx[X_U][s][lane];
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) {
                    const float4 bb = *reinterpret_cast<const float4 *>(sB + s * kNS + 4 * q);
                    const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = 4 * q + i;
                        h[n] = fmaf(ex2_mufu(dl * A2[n]), h[n], du * bv[i]);
                        if (keep) hist[s + 1][n][lane] = h[n];
                    }
                }
            }
        };

        // ---- forward from h0 (or zeros): checkpoints every kSeg timesteps (state before the segment)
        float h[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) h[n] = (valid && p.h0 && n < N) ? __ldg(p.h0 + (b * p.dim + dc) * N + n) : 0.f;
        for (int seg = 0; seg < p.n_segs; ++seg) {
            const int64_t t0 = (int64_t)seg * kSeg;
            const int tn = (L - t0) < kSeg ? (int)(L - t0) : kSeg;
            float4 *dst = reinterpret_cast<float4 *>(ck + seg * 32 * kNS);
#pragma unroll
            for (int q = 0; q < kNS / 4; ++q) __stcg(dst + q, make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
            stage(t0, tn, false);
            advance(h, tn, false);
        }

        // ---- backward, segment by segment from the end
        float g[kNS], dA_acc[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) {
            g[n] = (valid && p.dlast && n < N) ? p.dlast[(b * p.dim + dc) * N + n] : 0.f;
            dA_acc[n] = 0.f;
        }
        float dD_acc = 0.f, dbias_acc = 0.f;
        float *part = p.part + grp * L * 32 + lane;  // this lane's (B or C, state) partial sums
        for (int seg = p.n_segs - 1; seg >= 0; --seg) {
            const int64_t t0 = (int64_t)seg * kSeg;
            const int tn = (L - t0) < kSeg ? (int)(L - t0) : kSeg;
            stage(t0, tn, true);
            const float4 *src = reinterpret_cast<const float4 *>(ck + seg * 32 * kNS);
#pragma unroll
            for (int q = 0; q < kNS / 4; ++q) {
                const float4 v = __ldcg(src + q);
                h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int n = 0; n < kNS; ++n) hist[0][n][lane] = h[n];
            advance(h, tn, true);
            float o_du[kSeg], o_dd[kSeg], o_dz[kSeg];
#pragma unroll
            for (int s = 0; s < kSeg; ++s) { o_du[s] = 0.f; o_dd[s] = 0.f; o_dz[s] = 0.f; }
#pragma unroll
            for (int s = kSeg - 1; s >= 0; --s) {
                if (s >= tn) continue;
                const float dl = sx[X_DL][s][lane];
                const float ut = sx[X_U][s][lane];
                const float dout = sx[X_DOUT][s][lane];
                float y = Dd * ut;
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) {
                    const float4 cc = *reinterpret_cast<const float4 *>(sC + s * kNS + 4 * q);
                    y = fmaf(cc.x, hist[s + 1][4 * q][lane], y);
                    y = fmaf(cc.y, hist[s + 1][4 * q + 1][lane], y);
                    y = fmaf(cc.z, hist[s + 1][4 * q + 2][lane], y);
                    y = fmaf(cc.w, hist[s + 1][4 * q + 3][lane], y);
                }
                float dy = dout;
                if (GATE) {
                    const float zt = sx[X_Z][s][lane];
                    const float sg = __fdividef(1.f, 1.f + __expf(-zt));
                    o_dz[s] = dout * y * sg * fmaf(zt, 1.f - sg, 1.f);
                    dy = dout * zt * sg;
                }
                dD_acc = fmaf(dy, ut, dD_acc);
                float dut = dy * Dd, ddelta = 0.f;
                float v[32];  // this lane's dB (states 0-15) and dC (16-31) terms
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) {
                    const float4 bb = *reinterpret_cast<const float4 *>(sB + s * kNS + 4 * q);
                    const float4 cc = *reinterpret_cast<const float4 *>(sC + s * kNS + 4 * q);
                    const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, cv[4] = {cc.x, cc.y, cc.z, cc.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = 4 * q + i;
                        const float hcur = hist[s + 1][n][lane], hp = hist[s][n][lane];
                        v[16 + n] = dy * hcur;
                        g[n] = fmaf(dy, cv[i], g[n]);
                        const float ab = ex2_mufu(dl * A2[n]);
                        const float gha = g[n] * hp * ab;
                        ddelta = fmaf(gha, Ar[n], fmaf(g[n], bv[i] * ut, ddelta));
                        dA_acc[n] = fmaf(gha, dl, dA_acc[n]);
                        v[n] = g[n] * dl * ut;
                        dut = fmaf(g[n] * dl, bv[i], dut);
                        g[n] *= ab;
                    }
                }
                WarpTranspose<16, 32>::run(v, lane);
                __stcg(part + (t0 + s) * 32, v[0]);
                const float ddraw = ddelta * sx[X_SIG][s][lane];
                dbias_acc += ddraw;
                o_du[s] = dut;
                o_dd[s] = ddraw;
            }
            // this lane's row of the segment, 16 bytes at a time where possible
            if (valid) {
                constexpr int V = 16 / (int)sizeof(T);
#pragma unroll
                for (int c = 0; c < kSeg / V; ++c) {
                    if (vec && (c + 1) * V <= tn) {
                        *reinterpret_cast<uint4 *>(gdu + row + t0 + c * V) = Elem<T>::pack(o_du + c * V);
                        *reinterpret_cast<uint4 *>(gdd + row + t0 + c * V) = Elem<T>::pack(o_dd + c * V);
                        if (GATE) *reinterpret_cast<uint4 *>(gdz + row + t0 + c * V) = Elem<T>::pack(o_dz + c * V);
                    } else {
#pragma unroll
                        for (int e = 0; e < V; ++e) {
                            const int s = c * V + e;
                            if (s < tn) {
                                Elem<T>::store(gdu + row + t0 + s, o_du[s]);
                                Elem<T>::store(gdd + row + t0 + s, o_dd[s]);
                                if (GATE) Elem<T>::store(gdz + row + t0 + s, o_dz[s]);
                            }
                        }
                    }
                }
            }
        }
        if (valid) {
#pragma unroll
            for (int n = 0; n < kNS; ++n) {
                if (n < N) atomicAdd(p.dA + dc * N + n, dA_acc[n]);
                if (n < N && p.dh0) p.dh0[(b * p.dim + dc) * N + n] = g[n];  // dL/dh_{-1}
            }
            if (p.dD) atomicAdd(p.dD + dc, dD_acc);
            if (p.dbias) atomicAdd(p.dbias + dc, dbias_acc);
        }
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
    const int smem = kWarpsBwd * kWarpFloats * 4;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpsBwd * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sm_count * per_sm;
    const int64_t need = (p.n_groups + kWarpsBwd - 1) / kWarpsBwd;
    if (grid > need) grid = need;
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
