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
//
// Design.  One lane per channel with all (<= 16) states in registers; a warp
// takes a group of 32 channels of one batch row through the whole sequence,
// twice: forward, storing the state every kSeg timesteps in the workspace
// (the checkpoints), then backward segment by segment from the end: each
// segment's states are recomputed from its checkpoint into shared memory and
// consumed in reverse.  dB and dC are sums over all channels of a batch row:
// each warp sums its 32 channels with a transposed shuffle reduction that
// leaves lane l the total for one (B or C, state) pair, and adds it to global
// memory with one reduction per lane and timestep.  dA, dD and dbias are
// summed over a group's whole sequence in registers and added once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kNS = 16;       // states per lane (dstate <= 16)
constexpr int kSeg = 16;      // timesteps between checkpoints
constexpr int kWarpsBwd = 2;  // warps per block

struct BwdParams {
    const void *u, *delta, *B, *C, *z, *dout;
    const float *A, *D, *delta_bias, *dlast;
    void *du, *ddelta, *dz;
    float *dA, *dB, *dC, *dD, *dbias;
    float *ckpt;  // workspace: n_groups x n_segs x 32 lanes x kNS
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

template <typename T, bool SP, bool GATE>
__global__ void __launch_bounds__(kWarpsBwd * 32) scan_bwd_kernel(const BwdParams p) {
    extern __shared__ float bwd_smem[];  // per warp: [step][state][lane] recomputed states
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    float(*hist)[kNS][32] = reinterpret_cast<float(*)[kNS][32]>(bwd_smem + wib * (kSeg + 1) * kNS * 32);
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

    for (int64_t grp = (int64_t)blockIdx.x * kWarpsBwd + wib; grp < p.n_groups; grp += total_warps) {
        const int64_t b = grp / p.groups_per_batch;
        const int64_t dc = (grp % p.groups_per_batch) * 32 + lane;
        const bool valid = dc < p.dim;
        const int64_t row = (b * p.dim + (valid ? dc : 0)) * L;  // this lane's channel row
        const T *Bb = gB + b * (int64_t)N * L;
        const T *Cb = gC + b * (int64_t)N * L;
        float A2[kNS], Ar[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) {
            Ar[n] = (valid && n < N) ? __ldg(p.A + dc * N + n) : 0.f;
            A2[n] = Ar[n] * kLog2e;
        }
        const float bias = (valid && p.delta_bias) ? __ldg(p.delta_bias + dc) : 0.f;
        const float Dd = (valid && p.D) ? __ldg(p.D + dc) : 0.f;
        float *ck = p.ckpt + grp * (int64_t)p.n_segs * 32 * kNS + lane * kNS;

        auto delta_at = [&](int64_t t) {
            float x = (valid ? Elem<T>::load(gd + row + t) : 0.f) + bias;
            return SP ? softplus_f(x) : x;
        };
        auto bval = [&](const T *base, int n, int64_t t) { return n < N ? Elem<T>::load(base + (int64_t)n * L + t) : 0.f; };

        // ---- forward: checkpoints every kSeg timesteps (state before the segment)
        float h[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) h[n] = 0.f;
        for (int64_t t = 0; t < L; ++t) {
            if (t % kSeg == 0) {
                float4 *dst = reinterpret_cast<float4 *>(ck + (t / kSeg) * 32 * kNS);
#pragma unroll
                for (int q = 0; q < kNS / 4; ++q) __stcg(dst + q, make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
            }
            const float dl = delta_at(t);
            const float du = dl * (valid ? Elem<T>::load(gu + row + t) : 0.f);
#pragma unroll
            for (int n = 0; n < kNS; ++n) h[n] = fmaf(ex2_mufu(dl * A2[n]), h[n], du * bval(Bb, n, t));
        }

        // ---- backward, segment by segment from the end
        float g[kNS], dA_acc[kNS];
#pragma unroll
        for (int n = 0; n < kNS; ++n) {
            g[n] = (valid && p.dlast && n < N) ? p.dlast[(b * p.dim + dc) * N + n] : 0.f;
            dA_acc[n] = 0.f;
        }
        float dD_acc = 0.f, dbias_acc = 0.f;
        for (int seg = p.n_segs - 1; seg >= 0; --seg) {
            const int64_t t0 = (int64_t)seg * kSeg;
            const int tn = (L - t0) < kSeg ? (int)(L - t0) : kSeg;
            // recompute the segment's states: hist[s] = h_{t0 - 1 + s}
            const float4 *src = reinterpret_cast<const float4 *>(ck + seg * 32 * kNS);
#pragma unroll
            for (int q = 0; q < kNS / 4; ++q) {
                const float4 v = __ldcg(src + q);
                h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int n = 0; n < kNS; ++n) hist[0][n][lane] = h[n];
            for (int s = 0; s < tn; ++s) {
                const int64_t t = t0 + s;
                const float dl = delta_at(t);
                const float du = dl * (valid ? Elem<T>::load(gu + row + t) : 0.f);
#pragma unroll
                for (int n = 0; n < kNS; ++n) {
                    h[n] = fmaf(ex2_mufu(dl * A2[n]), h[n], du * bval(Bb, n, t));
                    hist[s + 1][n][lane] = h[n];
                }
            }
            for (int s = tn - 1; s >= 0; --s) {
                const int64_t t = t0 + s;
                const float draw = (valid ? Elem<T>::load(gd + row + t) : 0.f) + bias;
                const float dl = SP ? softplus_f(draw) : draw;
                const float ut = valid ? Elem<T>::load(gu + row + t) : 0.f;
                const float dout = valid ? Elem<T>::load(go + row + t) : 0.f;
                float y = Dd * ut;
#pragma unroll
                for (int n = 0; n < kNS; ++n) y = fmaf(bval(Cb, n, t), hist[s + 1][n][lane], y);
                float dy = dout;
                if (GATE) {
                    const float zt = valid ? Elem<T>::load(gz + row + t) : 0.f;
                    const float sg = __fdividef(1.f, 1.f + __expf(-zt));
                    if (valid) Elem<T>::store(gdz + row + t, dout * y * sg * fmaf(zt, 1.f - sg, 1.f));
                    dy = dout * zt * sg;
                }
                dD_acc = fmaf(dy, ut, dD_acc);
                float dut = dy * Dd, ddelta = 0.f;
                float v[32];  // this lane's dB (states 0-15) and dC (16-31) terms
#pragma unroll
                for (int n = 0; n < kNS; ++n) {
                    const float bn = bval(Bb, n, t);
                    const float hcur = hist[s + 1][n][lane], hp = hist[s][n][lane];
                    v[16 + n] = dy * hcur;
                    g[n] = fmaf(dy, bval(Cb, n, t), g[n]);
                    const float ab = ex2_mufu(dl * A2[n]);
                    const float gha = g[n] * hp * ab;
                    ddelta = fmaf(gha, Ar[n], fmaf(g[n], bn * ut, ddelta));
                    dA_acc[n] = fmaf(gha, dl, dA_acc[n]);
                    v[n] = g[n] * dl * ut;
                    dut = fmaf(g[n] * dl, bn, dut);
                    g[n] *= ab;
                }
                WarpTranspose<16, 32>::run(v, lane);
                const int n_red = lane & 15;
                if (n_red < N) atomicAdd((lane < 16 ? p.dB : p.dC) + (b * N + n_red) * L + t, v[0]);
                const float ddraw = SP ? ddelta * __fdividef(1.f, 1.f + __expf(-draw)) : ddelta;
                dbias_acc += ddraw;
                if (valid) {
                    Elem<T>::store(gdu + row + t, dut);
                    Elem<T>::store(gdd + row + t, ddraw);
                }
            }
        }
        if (valid) {
#pragma unroll
            for (int n = 0; n < kNS; ++n)
                if (n < N) atomicAdd(p.dA + dc * N + n, dA_acc[n]);
            if (p.dD) atomicAdd(p.dD + dc, dD_acc);
            if (p.dbias) atomicAdd(p.dbias + dc, dbias_acc);
        }
    }
}

template <typename T, bool SP, bool GATE>
cudaError_t launch_t(const BwdParams &p, int sm_count, cudaStream_t st) {
    auto kern = scan_bwd_kernel<T, SP, GATE>;
    const int smem = kWarpsBwd * (kSeg + 1) * kNS * 32 * 4;
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
    return (size_t)(groups * segs * 32 * kNS) * 4;
}

cudaError_t launch_scan_bwd(const ScanBwdArgs &a, void *workspace, int sm_count, cudaStream_t st) {
    BwdParams p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z; p.dout = a.dout;
    p.A = a.A; p.D = a.D; p.delta_bias = a.delta_bias; p.dlast = a.dlast;
    p.du = a.du; p.ddelta = a.ddelta; p.dz = a.dz;
    p.dA = a.dA; p.dB = a.dB; p.dC = a.dC; p.dD = a.dD; p.dbias = a.ddelta_bias;
    p.ckpt = static_cast<float *>(workspace);
    p.batch = a.batch; p.dim = a.dim; p.seqlen = a.seqlen; p.dstate = a.dstate; p.softplus = a.softplus;
    p.groups_per_batch = (int)((a.dim + 31) / 32);
    p.n_groups = (int)(a.batch * p.groups_per_batch);
    p.n_segs = (int)((a.seqlen + kSeg - 1) / kSeg);
    // the sums over channels and time accumulate into zeroed outputs
    const size_t nBC = (size_t)(a.batch * a.dstate * a.seqlen) * 4;
    cudaError_t e = cudaMemsetAsync(a.dB, 0, nBC, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dC, 0, nBC, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dA, 0, (size_t)(a.dim * a.dstate) * 4, st);
    if (e == cudaSuccess && a.dD) e = cudaMemsetAsync(a.dD, 0, (size_t)a.dim * 4, st);
    if (e == cudaSuccess && a.ddelta_bias) e = cudaMemsetAsync(a.ddelta_bias, 0, (size_t)a.dim * 4, st);
    if (e != cudaSuccess) return e;
    return a.act == kBF16 ? launch_typed<__nv_bfloat16>(p, sm_count, st) : launch_typed<float>(p, sm_count, st);
}

}  // namespace mscan
