// scan_fwd.cu -- fused selective-scan (S6) forward kernel for sm_100a.
//
// What one launch computes (per batch row b and channel d, time in order):
//   delta = softplus(delta_raw + bias[d]);  Abar = exp(delta * A[d,n])
//   h[n]  = Abar * h[n] + (delta * u) * B[b,n,t];   y = sum_n C[b,n,t] h[n]
//   out   = (y + D[d] u) * silu(z)
// following the recurrent form and the selective_scan / MambaBlock listings
// of "Mamba SSM concept and implementation in Keras and TensorFlow", fused so
// that nothing of size (batch, L, dim, N) ever reaches HBM (Mamba paper,
// Appendix E.5).
//
// Work decomposition
//   * A block owns one batch row and CG = THREADS / R consecutive channels and
//     walks the whole sequence in chunks of TC timesteps, carrying the state
//     h in registers from chunk to chunk (no inter-block communication).
//   * Each channel's NP (padded) states are split over R consecutive lanes of
//     one warp, S = NP / R states per thread.  R trades balance against
//     overhead: more lanes per channel give more warps to spread over the 592
//     SM sub-partitions but need a cross-lane sum of the readout.
//   * Raw u / delta / z / B / C tiles are copied global -> shared with 16-byte
//     cp.async into a double buffer, so the next chunk's loads overlap this
//     chunk's scan.  B and C tiles are staged once per block and shared by all
//     CG channels (they are per batch row, not per channel).
//   * Prologue (one thread per 16-byte vector): delta = softplus(raw + bias)
//     and delta*u are computed once per element into fp32 shared memory.
//   * Scan: per thread, per state, per timestep: one ex2 (MUFU), one FMUL
//     (delta*u*B), one FFMA (state), one FFMA (readout).  fp32 activations
//     take the accurate decay of device_math.cuh (Decay<true>: the state
//     advances by (Abar - 1) h + b with Abar - 1 on the FMA pipe).  Partial readouts of
//     the R lanes are summed with a transposed butterfly (log2 R shuffle
//     rounds) so each lane ends up owning complete outputs.
//   * Epilogue (one thread per 16-byte vector): out = (y + D u) silu(z),
//     rounded to the activation type and stored with 16-byte stores.
//
// Layouts.  Every sequence tensor has its own (batch, channel or state, time)
// element strides.  The kernel comes in two orientations: time-contiguous
// (CL = false: u / delta / z / out rows of consecutive timesteps, the dense
// (batch, dim, L) layout among them) and channel-contiguous (CL = true: the
// (batch, L, dim) layout of a sequence model's activations, possibly a slice
// of a wider projection output).  Both stage a tile in the orientation it
// has in memory -- [channel][time] or [time][channel] -- so the copies stay
// 16-byte and coalesced, and read it transposed on chip.  B and C are staged
// as [state][time] or [time][state] the same way, independently.  Tensors
// that fit neither vector form take element copies with any strides.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.cuh"
#include "device_math.cuh"
#include "internal.h"

namespace mscan {

struct KParams {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    float *last_state;
    const float *h0;
    ScanStrides st;    // element strides of u, delta, z, out, B, C
    int64_t dim, seqlen;
    int64_t n_groups;  // channel groups per batch row
    int dstate;
    int softplus;
    int vec;           // u / delta / z / out: 16-byte vectors along the kernel's contiguous axis
    int bc_mode;       // B / C: 0 element copies, 1 vectors along time, 2 vectors along states
    // byte ranges of the pointer arguments, for the bounds-checked build
    MSCAN_EXTENTS(x_u, x_delta, x_z, x_B, x_C, x_A, x_D, x_bias, x_out, x_last, x_h0)
};

// ------------------------------------------------------------ geometry
template <typename T, int NP, int R, int THREADS>
struct Geom {
    static constexpr int S = NP / R;
    static constexpr int CG = THREADS / R;
    static constexpr int V = 16 / (int)sizeof(T);
    static constexpr int RB = R > 4 ? R : 4;
    static constexpr size_t smem_for(int tc) {
        return (size_t)(2 * CG + 2 * NP) * (tc + 4) * 4 +
               (size_t)2 * (3 * CG + 2 * NP) * tc * sizeof(T);
    }
    static constexpr bool tc_ok(int tc) {
        return tc % (V * R) == 0 && tc % RB == 0;
    }
    // Largest chunk in {64, 32, 16, 8} that fits 56 KB (four blocks per SM),
    // else the smallest legal chunk.
    static constexpr int pick_tc() {
        return (tc_ok(64) && smem_for(64) <= 56 * 1024) ? 64
             : (tc_ok(32) && smem_for(32) <= 56 * 1024) ? 32
             : (tc_ok(16) && smem_for(16) <= 56 * 1024) ? 16
             : (tc_ok(8) && smem_for(8) <= 56 * 1024) ? 8
             : tc_ok(8) ? 8 : tc_ok(16) ? 16 : tc_ok(32) ? 32 : tc_ok(64) ? 64 : 128;
    }
    static constexpr int TC = pick_tc();
    static constexpr size_t SMEM = smem_for(TC);
};

// ------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool pred) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int nbytes = pred ? 16 : 0;  // 0 -> zero-fill, nothing read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(s), "l"(gmem), "r"(nbytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Sum v[] over the R lanes of a channel, transposed: afterwards lane r holds
// the complete sums for indices [r * RB / R, (r + 1) * RB / R) in v[0 ..].
// Round K (K = R/2, R/4, .., 1) halves the live values: the lane whose bit K
// is set keeps the upper half and sends the lower half to its partner.
template <int K, int CNT, int RB>
struct TransposeReduce {
    __device__ __forceinline__ static void run(float (&v)[RB], int r) {
        constexpr int HALF = CNT / 2;
        const bool upper = (r & K) != 0;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
            const float send = upper ? v[i] : v[i + HALF];
            const float keep = upper ? v[i + HALF] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, K);
        }
        TransposeReduce<K / 2, HALF, RB>::run(v, r);
    }
};
template <int CNT, int RB>
struct TransposeReduce<0, CNT, RB> {
    __device__ __forceinline__ static void run(float (&)[RB], int) {}
};

template <int R, int RB>
__device__ __forceinline__ void transpose_reduce(float (&v)[RB], int r) {
    TransposeReduce<R / 2, RB, RB>::run(v, r);
}

template <typename T, int NP, int R, int THREADS, bool CL>
__global__ void __launch_bounds__(THREADS)
scan_fwd_kernel(const KParams p) {
    using G = Geom<T, NP, R, THREADS>;
    using Dk = Decay<sizeof(T) == 4>;
    constexpr int S = G::S, CG = G::CG, V = G::V, RB = G::RB, TC = G::TC;
    constexpr int TCP = TC + 4;            // fp32 row pitch (16-byte multiple)
    constexpr int VPR = TC / V;            // 16-byte vectors per row per chunk
    constexpr int CH_VEC = CG * VPR;       // channel-tile vectors per tensor
    constexpr int BC_VEC = NP * VPR;       // B (or C) tile vectors
    constexpr int CVR = CG / V;            // channel-contiguous: vectors per timestep row
    constexpr int NVR = NP / V;            // state-contiguous B / C: vectors per timestep row

    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *sDelta = reinterpret_cast<float *>(smem_raw);  // delta, then y
    float *sDu = sDelta + CG * TCP;                       // delta * u
    float *sB = sDu + CG * TCP;
    float *sC = sB + NP * TCP;
    T *rawBase = reinterpret_cast<T *>(sC + NP * TCP);    // 2 stages
    constexpr int STAGE = (3 * CG + 2 * NP) * TC;         // elements per stage

    const int tid = threadIdx.x;
    const int64_t grp = blockIdx.x % p.n_groups;
    const int64_t b = blockIdx.x / p.n_groups;
    const int64_t d0 = grp * CG;
    const int64_t L = p.seqlen, Dm = p.dim;
    const int N = p.dstate;
    const bool has_z = p.z != nullptr;

    const T *__restrict__ gu = static_cast<const T *>(p.u);
    const T *__restrict__ gd = static_cast<const T *>(p.delta);
    const T *__restrict__ gz = static_cast<const T *>(p.z);
    const T *__restrict__ gB = static_cast<const T *>(p.B);
    const T *__restrict__ gC = static_cast<const T *>(p.C);
    T *__restrict__ gout = static_cast<T *>(p.out);
    const Stride3 su = p.st.u, sdl = p.st.delta, sz = p.st.z, so = p.st.out, sBs = p.st.B, sCs = p.st.C;

    // ---- scan identity: channel c, lane r, states r*S .. r*S+S-1
    const int c = tid / R, r = tid % R;
    const int64_t d = d0 + c;
    using HS = typename Dk::H;  // the state: fp64 for fp32 activations
    HS h[S];
    float A2[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int n = r * S + s;
        A2[s] = (d < Dm && n < N && MSCAN_WITHIN(p.x_A, p.A + d * N + n, 4, kSiteA)) ? __ldg(p.A + d * N + n) * Dk::kScale
                                                                               : 0.f;
        h[s] = (p.h0 && d < Dm && n < N && MSCAN_WITHIN(p.x_h0, p.h0 + (b * Dm + d) * N + n, 4, kSiteH0))
                   ? __ldcg(p.h0 + (b * Dm + d) * N + n) : 0.f;
    }

    // ---- copy one chunk's raw tiles into stage `st`: u / delta / z as
    // [channel][time] (CL = false) or [time][channel] (CL = true); B / C as
    // [state][time], or [time][state] when they are state-contiguous
    auto issue_loads = [&](int64_t t0, int st) {
        T *rU = rawBase + st * STAGE;
        T *rD = rU + CG * TC;
        T *rZ = rD + CG * TC;
        T *rB = rZ + CG * TC;
        T *rC = rB + NP * TC;
        if (p.vec) {
            if (!CL) {
                for (int vi = tid; vi < CH_VEC; vi += THREADS) {
                    const int pc = vi / VPR, tv = vi % VPR;
                    const int64_t t = t0 + tv * V, dd = d0 + pc;
                    const bool ok = (dd < Dm) && (t < L);
                    const T *pu = gu + (ok ? b * su.b + dd * su.d + t : 0), *pd = gd + (ok ? b * sdl.b + dd * sdl.d + t : 0);
                    cp_async16(rU + pc * TC + tv * V, pu, ok && MSCAN_WITHIN(p.x_u, pu, 16, kSiteU));
                    cp_async16(rD + pc * TC + tv * V, pd, ok && MSCAN_WITHIN(p.x_delta, pd, 16, kSiteDelta));
                    if (has_z) {
                        const T *pz = gz + (ok ? b * sz.b + dd * sz.d + t : 0);
                        cp_async16(rZ + pc * TC + tv * V, pz, ok && MSCAN_WITHIN(p.x_z, pz, 16, kSiteZ));
                    }
                }
            } else {
                for (int vi = tid; vi < TC * CVR; vi += THREADS) {
                    const int tt = vi / CVR, cv = vi % CVR;
                    const int64_t t = t0 + tt, dd = d0 + cv * V;
                    const bool ok = (dd < Dm) && (t < L);  // dim is a whole number of vectors
                    const T *pu = gu + (ok ? b * su.b + t * su.t + dd : 0), *pd = gd + (ok ? b * sdl.b + t * sdl.t + dd : 0);
                    cp_async16(rU + tt * CG + cv * V, pu, ok && MSCAN_WITHIN(p.x_u, pu, 16, kSiteU));
                    cp_async16(rD + tt * CG + cv * V, pd, ok && MSCAN_WITHIN(p.x_delta, pd, 16, kSiteDelta));
                    if (has_z) {
                        const T *pz = gz + (ok ? b * sz.b + t * sz.t + dd : 0);
                        cp_async16(rZ + tt * CG + cv * V, pz, ok && MSCAN_WITHIN(p.x_z, pz, 16, kSiteZ));
                    }
                }
            }
        } else {
            // any strides: element copies, zero outside the problem
            for (int e = tid; e < CG * TC; e += THREADS) {
                const int pc = CL ? e % CG : e / TC, tt = CL ? e / CG : e % TC;
                const int64_t t = t0 + tt, dd = d0 + pc;
                const bool ok = (dd < Dm) && (t < L);
                const T *pu = gu + b * su.b + dd * su.d + t * su.t, *pd = gd + b * sdl.b + dd * sdl.d + t * sdl.t;
                rU[e] = (ok && MSCAN_WITHIN(p.x_u, pu, sizeof(T), kSiteU)) ? *pu : T(0.f);
                rD[e] = (ok && MSCAN_WITHIN(p.x_delta, pd, sizeof(T), kSiteDelta)) ? *pd : T(0.f);
                if (has_z) {
                    const T *pz = gz + b * sz.b + dd * sz.d + t * sz.t;
                    rZ[e] = (ok && MSCAN_WITHIN(p.x_z, pz, sizeof(T), kSiteZ)) ? *pz : T(0.f);
                }
            }
        }
        if (p.bc_mode == 1) {
            for (int vi = tid; vi < 2 * BC_VEC; vi += THREADS) {
                const int which = vi / BC_VEC, rem = vi % BC_VEC;
                const int n = rem / VPR, tv = rem % VPR;
                const int64_t t = t0 + tv * V;
                const bool ok = (n < N) && (t < L);
                const Stride3 &sx = which ? sCs : sBs;
                const int64_t off = ok ? b * sx.b + n * sx.d + t : 0;
                const T *src = (which ? gC : gB) + off;
                cp_async16((which ? rC : rB) + n * TC + tv * V, src,
                           ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, src, 16, which ? kSiteC : kSiteB));
            }
        } else if (p.bc_mode == 2) {
            for (int vi = tid; vi < 2 * TC * NVR; vi += THREADS) {
                const int which = vi / (TC * NVR), rem = vi % (TC * NVR);
                const int tt = rem / NVR, n = (rem % NVR) * V;
                const int64_t t = t0 + tt;
                const bool ok = (n < N) && (t < L);  // dstate is a whole number of vectors
                const Stride3 &sx = which ? sCs : sBs;
                const int64_t off = ok ? b * sx.b + t * sx.t + n : 0;
                const T *src = (which ? gC : gB) + off;
                cp_async16((which ? rC : rB) + tt * NP + n, src,
                           ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, src, 16, which ? kSiteC : kSiteB));
            }
        } else {
            for (int e = tid; e < 2 * NP * TC; e += THREADS) {
                const int which = e / (NP * TC), rem = e % (NP * TC);
                const int n = rem / TC, tt = rem % TC;
                const int64_t t = t0 + tt;
                const bool ok = (n < N) && (t < L);
                const Stride3 &sx = which ? sCs : sBs;
                const T *src = (which ? gC : gB) + b * sx.b + n * sx.d + t * sx.t;
                (which ? rC : rB)[rem] =
                    (ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, src, sizeof(T), which ? kSiteC : kSiteB)) ? *src : T(0.f);
            }
        }
        cp_async_commit();  // an empty group when everything was copied by hand
    };

    issue_loads(0, 0);

    int stage = 0;
#pragma unroll 1
    for (int64_t t0 = 0; t0 < L; t0 += TC, stage ^= 1) {
        const T *rU = rawBase + stage * STAGE;
        const T *rD = rU + CG * TC;
        const T *rZ = rD + CG * TC;
        const T *rB = rZ + CG * TC;
        const T *rC = rB + NP * TC;
        const int tvalid = (L - t0) < TC ? (int)(L - t0) : TC;

        cp_async_wait_all();
        __syncthreads();  // raw stage ready; previous epilogue finished

        // ---- prologue: delta and delta*u for every element of the tile
        for (int vi = tid; vi < CH_VEC; vi += THREADS) {
            const int pc = CL ? vi % CG : vi / VPR, tv = CL ? vi / CG : vi % VPR;
            const int64_t dd = d0 + pc;
            const float bias = (dd < Dm && p.delta_bias && MSCAN_WITHIN(p.x_bias, p.delta_bias + dd, 4, kSiteBias))
                                   ? __ldg(p.delta_bias + dd) : 0.f;
            float fu[V], fd[V];
            if (!CL) {
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rD + pc * TC + tv * V), fd);
            } else {  // a column of the [time][channel] tile
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    fu[i] = Elem<T>::to_f(rU[(tv * V + i) * CG + pc]);
                    fd[i] = Elem<T>::to_f(rD[(tv * V + i) * CG + pc]);
                }
            }
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float dl = fd[i] + bias;
                if (p.softplus) dl = Dk::softplus(dl);
                if (tv * V + i >= tvalid) dl = 0.f;  // past the end: Abar = 1, no input
                fd[i] = dl;
                fu[i] = dl * fu[i];
            }
            float *dst = sDelta + pc * TCP + tv * V;
            float *dsu = sDu + pc * TCP + tv * V;
#pragma unroll
            for (int i = 0; i < V; i += 4) {
                *reinterpret_cast<float4 *>(dst + i) = make_float4(fd[i], fd[i + 1], fd[i + 2], fd[i + 3]);
                *reinterpret_cast<float4 *>(dsu + i) = make_float4(fu[i], fu[i + 1], fu[i + 2], fu[i + 3]);
            }
        }
        for (int vi = tid; vi < 2 * BC_VEC; vi += THREADS) {
            const int which = vi / BC_VEC, rem = vi % BC_VEC;
            const bool by_state = p.bc_mode == 2;
            const int n = by_state ? rem % NP : rem / VPR, tv = by_state ? rem / NP : rem % VPR;
            const T *raw = which ? rC : rB;
            float f[V];
            if (!by_state) {
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(raw + n * TC + tv * V), f);
            } else {  // a column of the [time][state] tile
#pragma unroll
                for (int i = 0; i < V; ++i) f[i] = Elem<T>::to_f(raw[(tv * V + i) * NP + n]);
            }
            float *dst = (which ? sC : sB) + n * TCP + tv * V;
#pragma unroll
            for (int i = 0; i < V; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
        }

        // next chunk's copies overlap this chunk's scan
        if (t0 + TC < L) issue_loads(t0 + TC, stage ^ 1);
        __syncthreads();

        // ---- scan: thread (c, r) advances its S states through the chunk
        {
            float *dRow = sDelta + c * TCP;
            const float *uRow = sDu + c * TCP;
#pragma unroll 1
            for (int tb = 0; tb < tvalid; tb += RB) {
                float yp[RB];
#pragma unroll
                for (int q = 0; q < RB; q += 4) {
                    const float4 dl = *reinterpret_cast<const float4 *>(dRow + tb + q);
                    const float4 du = *reinterpret_cast<const float4 *>(uRow + tb + q);
                    HS y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        const int n = r * S + s;
                        const float4 bb = *reinterpret_cast<const float4 *>(sB + n * TCP + tb + q);
                        const float4 cc = *reinterpret_cast<const float4 *>(sC + n * TCP + tb + q);
                        h[s] = Dk::step(dl.x * A2[s], h[s], du.x * bb.x); y0 = fma((HS)cc.x, h[s], y0);
                        h[s] = Dk::step(dl.y * A2[s], h[s], du.y * bb.y); y1 = fma((HS)cc.y, h[s], y1);
                        h[s] = Dk::step(dl.z * A2[s], h[s], du.z * bb.z); y2 = fma((HS)cc.z, h[s], y2);
                        h[s] = Dk::step(dl.w * A2[s], h[s], du.w * bb.w); y3 = fma((HS)cc.w, h[s], y3);
                    }
                    yp[q] = (float)y0; yp[q + 1] = (float)y1; yp[q + 2] = (float)y2; yp[q + 3] = (float)y3;
                }
                if (R > 1) transpose_reduce<R, RB>(yp, r);
                __syncwarp();  // every lane of the channel has read dRow[tb .. tb+RB)
                constexpr int OWN = RB / R;  // outputs owned per lane
                float *yo = dRow + tb + r * OWN;
                if (OWN == 1) {
                    yo[0] = yp[0];
                } else if (OWN == 2) {
                    *reinterpret_cast<float2 *>(yo) = make_float2(yp[0], yp[1]);
                } else {
                    *reinterpret_cast<float4 *>(yo) = make_float4(yp[0], yp[1], yp[2], yp[3]);
                }
            }
        }
        __syncthreads();

        // ---- epilogue: out = (y + D u) * silu(z)
        if (!CL) {
            for (int vi = tid; vi < CH_VEC; vi += THREADS) {
                const int pc = vi / VPR, tv = vi % VPR;
                const int64_t dd = d0 + pc;
                const int64_t t = t0 + tv * V;
                if (dd >= Dm || tv * V >= tvalid) continue;
                const float Dd = (p.D && MSCAN_WITHIN(p.x_D, p.D + dd, 4, kSiteD)) ? __ldg(p.D + dd) : 0.f;
                float fu[V], fz[V], y[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
                if (has_z) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rZ + pc * TC + tv * V), fz);
                const float *ys = sDelta + pc * TCP + tv * V;
#pragma unroll
                for (int i = 0; i < V; i += 4) {
                    const float4 q = *reinterpret_cast<const float4 *>(ys + i);
                    y[i] = q.x; y[i + 1] = q.y; y[i + 2] = q.z; y[i + 3] = q.w;
                }
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    float o = fmaf(Dd, fu[i], y[i]);
                    if (has_z) o *= silu_f(fz[i]);
                    y[i] = o;
                }
                T *dst = gout + b * so.b + dd * so.d + t * so.t;
                if (p.vec) {
                    if (MSCAN_WITHIN(p.x_out, dst, 16, kSiteOut)) stg16_stream(dst, Elem<T>::pack(y));
                } else {
#pragma unroll
                    for (int i = 0; i < V; ++i)
                        if (tv * V + i < tvalid && MSCAN_WITHIN(p.x_out, dst + i * so.t, sizeof(T), kSiteOut))
                            Elem<T>::store(dst + i * so.t, y[i]);
                }
            }
        } else {  // one thread per V channels of one timestep
            for (int vi = tid; vi < TC * CVR; vi += THREADS) {
                const int tt = vi / CVR, cv = vi % CVR;
                const int64_t dd = d0 + cv * V;
                const int64_t t = t0 + tt;
                if (dd >= Dm || tt >= tvalid) continue;
                float fu[V], fz[V], y[V];
                Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + tt * CG + cv * V), fu);
                if (has_z) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rZ + tt * CG + cv * V), fz);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const float Dd = (p.D && dd + i < Dm && MSCAN_WITHIN(p.x_D, p.D + dd + i, 4, kSiteD)) ? __ldg(p.D + dd + i)
                                                                                                : 0.f;
                    float o = fmaf(Dd, fu[i], sDelta[(cv * V + i) * TCP + tt]);
                    if (has_z) o *= silu_f(fz[i]);
                    y[i] = o;
                }
                T *dst = gout + b * so.b + t * so.t + dd * so.d;
                if (p.vec) {
                    if (MSCAN_WITHIN(p.x_out, dst, 16, kSiteOut)) stg16_stream(dst, Elem<T>::pack(y));
                } else {
#pragma unroll
                    for (int i = 0; i < V; ++i)
                        if (dd + i < Dm && MSCAN_WITHIN(p.x_out, dst + i * so.d, sizeof(T), kSiteOut))
                            Elem<T>::store(dst + i * so.d, y[i]);
                }
            }
        }
    }

    if (p.last_state != nullptr && d < Dm) {
        float *ls = p.last_state + (b * Dm + d) * N;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int n = r * S + s;
            if (n < N && MSCAN_WITHIN(p.x_last, ls + n, 4, kSiteLastState)) ls[n] = (float)h[s];
        }
    }
}

// ------------------------------------------------------------ dispatch
template <typename T, int NP, int R, int THREADS, bool CL>
static cudaError_t launch_impl(const KParams &kp, int64_t blocks, cudaStream_t st) {
    using G = Geom<T, NP, R, THREADS>;
    auto kern = scan_fwd_kernel<T, NP, R, THREADS, CL>;
    if (G::SMEM > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)G::SMEM);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)blocks, THREADS, G::SMEM, st>>>(kp);
    return cudaGetLastError();
}

template <typename T, int NP, int R, int THREADS>
static void geom_info(ScanPlan *pl) {
    using G = Geom<T, NP, R, THREADS>;
    pl->chunk = G::TC;
    pl->channels_per_block = G::CG;
    pl->smem_bytes = G::SMEM;
}

// Every (dtype, NP, R, THREADS) the library is built for.  R ranges over the
// divisors of NP with at most 16 states per thread and at most 16 lanes.
#define MSCAN_FOR_NP_R(X, T, TH) \
    X(T, 8, 1, TH) X(T, 8, 2, TH) X(T, 8, 4, TH) X(T, 8, 8, TH) \
    X(T, 16, 1, TH) X(T, 16, 2, TH) X(T, 16, 4, TH) X(T, 16, 8, TH) X(T, 16, 16, TH) \
    X(T, 32, 2, TH) X(T, 32, 4, TH) X(T, 32, 8, TH) X(T, 32, 16, TH) \
    X(T, 64, 4, TH) X(T, 64, 8, TH) X(T, 64, 16, TH)
#define MSCAN_FOR_ALL(X) \
    MSCAN_FOR_NP_R(X, float, 128) MSCAN_FOR_NP_R(X, float, 256) \
    MSCAN_FOR_NP_R(X, __nv_bfloat16, 128) MSCAN_FOR_NP_R(X, __nv_bfloat16, 256)

template <typename T> constexpr int act_of();
template <> constexpr int act_of<float>() { return kF32; }
template <> constexpr int act_of<__nv_bfloat16>() { return kBF16; }

static bool lookup_geom(int act, int np, int r, int th, ScanPlan *pl) {
#define X(T, NP_, R_, TH_) \
    if (act == act_of<T>() && np == NP_ && r == R_ && th == TH_) { geom_info<T, NP_, R_, TH_>(pl); return true; }
    MSCAN_FOR_ALL(X)
#undef X
    return false;
}

// How the static kernel reads and writes the sequence tensors: the
// orientation (channel-contiguous when u is), whether u / delta / z / out all
// allow 16-byte vectors along it, and the form of the B / C copies.
struct StaticLayout {
    ScanStrides st;
    bool cl;
    int vec, bc_mode;
};

static StaticLayout static_layout(const ScanArgs &a) {
    StaticLayout r;
    const int64_t Dm = a.dim, L = a.seqlen, N = a.dstate;
    if (a.strides) {
        r.st = *a.strides;
    } else {
        r.st.u = r.st.delta = r.st.z = r.st.out = Stride3{Dm * L, L, 1};
        r.st.B = r.st.C = Stride3{N * L, L, 1};
    }
    const int64_t V = a.act == kBF16 ? 8 : 4;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    r.cl = r.st.u.d == 1 && r.st.u.t != 1 && L > 1;
    auto x_ok = [&](const void *q, const Stride3 &s) {
        if (q == nullptr) return true;
        if (!al(q) || s.b % V != 0) return false;
        return r.cl ? (s.d == 1 && s.t % V == 0) : (s.t == 1 && s.d % V == 0);
    };
    const bool len_ok = r.cl ? Dm % V == 0 : L % V == 0;
    r.vec = len_ok && x_ok(a.u, r.st.u) && x_ok(a.delta, r.st.delta) && x_ok(a.z, r.st.z) &&
            x_ok(a.out, r.st.out);
    auto bc_ok = [&](int mode, const void *q, const Stride3 &s) {
        if (!al(q) || s.b % V != 0) return false;
        return mode == 1 ? (s.t == 1 && s.d % V == 0) : (s.d == 1 && s.t % V == 0);
    };
    if (L % V == 0 && bc_ok(1, a.B, r.st.B) && bc_ok(1, a.C, r.st.C)) r.bc_mode = 1;
    else if (N % V == 0 && bc_ok(2, a.B, r.st.B) && bc_ok(2, a.C, r.st.C)) r.bc_mode = 2;
    else r.bc_mode = 0;
    return r;
}

MSCAN_BOUNDS_TAKE(static_bounds_take)

cudaError_t launch_scan_fwd(const ScanArgs &a, const ScanPlan &pl, cudaStream_t st) {
    KParams kp;
    kp.u = a.u; kp.delta = a.delta; kp.B = a.B; kp.C = a.C; kp.z = a.z;
    kp.A = a.A; kp.D = a.D; kp.delta_bias = a.delta_bias;
    kp.out = a.out; kp.last_state = a.last_state; kp.h0 = a.h0;
    kp.dim = a.dim; kp.seqlen = a.seqlen;
    kp.n_groups = (a.dim + pl.channels_per_block - 1) / pl.channels_per_block;
    kp.dstate = a.dstate; kp.softplus = a.softplus;
    const StaticLayout lay = static_layout(a);
    kp.st = lay.st; kp.vec = lay.vec; kp.bc_mode = lay.bc_mode;
#ifdef MSCAN_BOUNDS_CHECK
    // byte ranges (bounds-checked build): one past the last element of each strided tensor
    const unsigned long long es = a.act == kBF16 ? 2 : 4;
    auto span = [&](const void *q, const Stride3 &x, int64_t rows) {
        const unsigned long long last = (unsigned long long)((a.batch - 1) * x.b + (rows - 1) * x.d +
                                                             (a.seqlen - 1) * x.t);
        return extent_of(q, (last + 1) * es);
    };
    kp.x_u = span(a.u, lay.st.u, a.dim);
    kp.x_delta = span(a.delta, lay.st.delta, a.dim);
    kp.x_z = span(a.z, lay.st.z, a.dim);
    kp.x_B = span(a.B, lay.st.B, a.dstate);
    kp.x_C = span(a.C, lay.st.C, a.dstate);
    kp.x_out = span(a.out, lay.st.out, a.dim);
    if (kp.x_out.bytes > (unsigned long long)g_out_extent_shrink) kp.x_out.bytes -= g_out_extent_shrink;
    else kp.x_out.bytes = 0;
    kp.x_A = extent_of(a.A, (unsigned long long)(a.dim * a.dstate) * 4);
    kp.x_D = extent_of(a.D, (unsigned long long)a.dim * 4);
    kp.x_bias = extent_of(a.delta_bias, (unsigned long long)a.dim * 4);
    kp.x_last = extent_of(a.last_state, (unsigned long long)(a.batch * a.dim * a.dstate) * 4);
    kp.x_h0 = extent_of(a.h0, (unsigned long long)(a.batch * a.dim * a.dstate) * 4);
#endif
#define X(T, NP_, R_, TH_) \
    if (a.act == act_of<T>() && pl.padded_dstate == NP_ && pl.lanes == R_ && pl.threads == TH_) \
        return lay.cl ? launch_impl<T, NP_, R_, TH_, true>(kp, pl.blocks, st)   \
                      : launch_impl<T, NP_, R_, TH_, false>(kp, pl.blocks, st);
    MSCAN_FOR_ALL(X)
#undef X
    return cudaErrorInvalidConfiguration;
}

// ------------------------------------------------------------ planning
static int padded_dstate(int n) { return n <= 8 ? 8 : n <= 16 ? 16 : n <= 32 ? 32 : 64; }

// Relative cost of one state-step for R lanes per channel (cross-lane readout
// sums and duplicated delta reads grow with R).
static double lane_overhead(int r) {
    switch (r) {
        case 1: return 1.00;
        case 2: return 1.05;
        case 4: return 1.30;  // B200, Mamba-2.8B layer: R = 4 1089 us vs R = 2 812 us
        case 8: return 1.50;
        default: return 1.80;
    }
}

int make_scan_plan(const ScanArgs &a, int want_lanes, int want_threads, int sm_count,
                   ScanPlan *pl) {
    const int np = padded_dstate(a.dstate);
    const int vbytes = 16;
    const int esize = a.act == kBF16 ? 2 : 4;
    const int vlen = vbytes / esize;
    auto aligned = [](const void *ptr) { return ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
    pl->vectorized = a.strides == nullptr && (a.seqlen % vlen == 0) && aligned(a.u) &&
                     aligned(a.delta) && aligned(a.z) && aligned(a.B) && aligned(a.C) &&
                     aligned(a.out);
    pl->padded_dstate = np;

    int lanes = want_lanes;
    if (lanes == 0) {
        // Pick R minimising (warps on the busiest sub-partition) x (states per
        // thread) x (per-state overhead): the scan is bound by per-SM-sub-
        // partition MUFU throughput, so balance across the 4 x SM sub-
        // partitions matters as much as the instruction count.
        const double smsp = 4.0 * (sm_count > 0 ? sm_count : 148);
        const double rows = (double)a.batch * (double)a.dim;
        double best = 1e300;
        for (int r = 1; r <= 16; r *= 2) {
            if (np % r || np / r > 16) continue;
            const double warps = rows * r / 32.0;
            double per = warps / smsp;
            double busiest = per <= 1.0 ? 1.0 : (double)(int64_t)(per + 0.999999);
            const double cost = busiest * (np / r) * lane_overhead(r);
            if (cost < best - 1e-9) { best = cost; lanes = r; }
        }
    }
    int threads = want_threads;
    if (threads == 0) {
        threads = 256;
        ScanPlan tmp;
        if (lookup_geom(a.act, np, lanes, 256, &tmp)) {
            const int64_t blocks256 = a.batch * ((a.dim + tmp.channels_per_block - 1) / tmp.channels_per_block);
            if (blocks256 < 2LL * (sm_count > 0 ? sm_count : 148)) threads = 128;
        }
    }
    if (!lookup_geom(a.act, np, lanes, threads, pl)) return -1;
    pl->lanes = lanes;
    pl->threads = threads;
    pl->blocks = a.batch * ((a.dim + pl->channels_per_block - 1) / pl->channels_per_block);
    if (pl->blocks <= 0 || pl->blocks > 0x7fffffffLL) return -1;
    if (pl->smem_bytes > 227 * 1024) return -1;
    return 0;
}

}  // namespace mscan
