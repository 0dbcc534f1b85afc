// scan_fwd_complex.cu -- the selective scan in complex-valued mode: a complex
// diagonal A and complex, input-dependent B and C (the complex SSM of the
// Mamba paper, Appendix E.4.1; the "complex number mode" on the roadmap of the
// "Mamba x JAX" page).  Per batch row b and channel d, time in order:
//   delta = softplus(delta_raw + bias[d])             (real)
//   Abar  = exp(delta A[d,n]) = 2^(delta Re A log2 e) (cos theta + i sin theta),
//           theta = delta Im A
//   h[n]  = Abar h[n] + (delta u) B[b,n,t]           (complex)
//   y     = Re(sum_n C[b,n,t] h[n]);  out = (y + D[d] u) silu(z)
// Complex tensors are interleaved (re, im) pairs: A (dim, N, 2) fp32, B and C
// (batch, N, L, 2) in the activation type, states (batch, dim, N, 2) fp32.
//
// With bf16 activations each state-step costs three special-function ops
// (ex2, sin, cos) instead of one, so the kernel is bound by the MUFU at a
// third of the real scan's rate; with fp32 activations they run on the FMA
// pipe instead.  Layout of the work as in the real static kernel: a block
// owns one batch row and CG = 128 / R channels, R lanes per channel split the 16
// (padded) states, tiles of 32 timesteps are copied to shared memory with
// 16-byte cp.async into a double buffer; a prologue forms delta and delta*u
// once per element and widens B / C to fp32 [t][n] complex pairs shared by
// every channel of the block; partial readouts of a channel's R lanes are
// summed with a transposed butterfly; the epilogue applies D and the gate.
// bf16 activations take Abar from the special-function unit; fp32 ones
// advance the state by (Abar - 1) h with Abar - 1 from FMA-pipe polynomials
// (abar_minus_one says why).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kCNP = 16;         // padded states (dstate <= 16)
constexpr int kCThreads = 128;   // threads per block
constexpr int kCTC = 32;         // timesteps per chunk

struct CParams {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    float *last_state;
    const float *h0;
    int64_t dim, seqlen;
    int n_groups;  // channel groups per batch row
    int dstate, softplus, vec;
};

template <typename T, int R>
struct CGeom {
    static constexpr int S = kCNP / R;                  // complex states per lane
    static constexpr int CG = kCThreads / R;            // channels per block
    static constexpr int V = 16 / (int)sizeof(T);       // elements per 16 bytes
    static constexpr int TC = kCTC;
    static constexpr int TCP = TC + 4;                  // fp32 row pitch
    static constexpr int VPR = TC / V;                  // vectors per channel row per chunk
    static constexpr int BVR = 2 * TC / V;              // vectors per B / C state row per chunk
    static constexpr int STAGE = 3 * CG * TC + 2 * kCNP * 2 * TC;  // raw elements per stage
    static constexpr size_t SMEM =
        (size_t)2 * CG * TCP * 4 + (size_t)2 * TC * kCNP * 8 + (size_t)2 * STAGE * sizeof(T);
};

__device__ __forceinline__ void cpa16(void *smem, const void *gmem, bool pred) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(s), "l"(gmem), "r"(pred ? 16 : 0) : "memory");
}

// sin and cos of x in [-pi, pi] on the special-function unit.
__device__ __forceinline__ void sincos_mufu(float x, float &s, float &c) {
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(s) : "f"(x));
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(c) : "f"(x));
}

// x - 2 pi k with k = rint(x / 2 pi), in [-pi, pi]: Cody-Waite reduction with
// 2 pi = kTwoPiHi + kTwoPiLo (kTwoPiHi the nearest float).
__device__ __forceinline__ float reduce_angle(float x) {
    constexpr float kInvTwoPi = 0.15915494309189535f;
    constexpr float kTwoPiHi = 6.28318548202514648f;
    constexpr float kTwoPiLo = -1.7484555314695172e-07f;
    const float k = rintf(x * kInvTwoPi);
    return fmaf(-k, kTwoPiLo, fmaf(-k, kTwoPiHi, x));
}

// sin t, cos t and cos t - 1 on the FMA pipe (|t| < 2^21).  Quadrant q =
// rint(2 t / pi) (adding 1.5 * 2^23 rounds to an integer held in the low
// bits), r = t - q pi / 2 by Cody-Waite with pi / 2 split in a float head and
// tail, so |r| <= pi / 4; sin r = r P(r^2), cos r - 1 = r^2 G(r^2), P and G
// the degree-3 Chebyshev fits from fit_sincos_poly.py in this directory
// (relative errors <= 9.3e-8 and 1.4e-7 in fp32); the quadrant then swaps
// and negates the pair.  In quadrant 0, cos t - 1 is r^2 G(r^2) itself,
// accurate however small; elsewhere |cos t - 1| >= 1 - cos(pi / 4) and c - 1
// is.
__device__ __forceinline__ void sincos_cm1(float t, float &s, float &c, float &cm1) {
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    constexpr float kTwoOverPi = 0.636619772367581343f;
    constexpr float kPio2Hi = 1.57079637050628662f;
    constexpr float kPio2Lo = -4.37113900018624284e-08f;
    const float tq = fmaf(t, kTwoOverPi, kRound);
    const float q = tq - kRound;
    const unsigned qi = __float_as_uint(tq);  // low bits: q mod 4
    float r = fmaf(-q, kPio2Hi, t);
    r = fmaf(-q, kPio2Lo, r);
    const float r2 = r * r;
    float ps = -1.950390433e-04f;
    ps = fmaf(ps, r2, 8.332035504e-03f);
    ps = fmaf(ps, r2, -1.666665077e-01f);
    ps = fmaf(ps, r2, 1.0f);
    const float sr = r * ps;
    float pc = 2.446378858e-05f;
    pc = fmaf(pc, r2, -1.388758887e-03f);
    pc = fmaf(pc, r2, 4.166664928e-02f);
    pc = fmaf(pc, r2, -0.5f);
    const float cm1r = r2 * pc;
    const float cr = fmaf(pc, r2, 1.0f);
    const bool swap = (qi & 1u) != 0;
    const float s0 = swap ? cr : sr, c0 = swap ? sr : cr;
    s = __uint_as_float(__float_as_uint(s0) ^ ((qi & 2u) << 30));        // negate in quadrants 2, 3
    c = __uint_as_float(__float_as_uint(c0) ^ (((qi + 1u) & 2u) << 30));  // negate in quadrants 1, 2
    cm1 = (qi & 3u) == 0 ? cm1r : c - 1.f;
}

// The fp32 path's softplus is softplus_precise (device_math.cuh): a relative
// error e in delta turns the rotation of a state with frequency Im A by
// e * delta * Im A per step, and over the ~1 / (delta |Re A|) steps the state
// remembers by e * Im A / |Re A| -- a factor of ~100 for the highest
// frequencies of the usual complex initialisation.  The one-op softplus_f has
// e up to 8.5e-7 for very negative inputs, enough to show at fp32 tolerance;
// softplus_precise keeps e near 1e-7.

// Abar - 1 for x = delta Re A, t = delta Im A, as (re, im):
//   e^x cos t - 1 = em1 cos t + (cos t - 1),   e^x sin t = (1 + em1) sin t,
// em1 = e^x - 1 from expm1_f (device_math.cuh: accurate relative to its own
// size near x = 0).  The state then advances as h + (Abar - 1) h: a
// step's error is relative to the small change of h, not to h.  A decay
// rounded to fp32 near 1 would carry the same relative error, 2^-24 or more,
// into h at every step, and those errors add up over the ~1 / (delta |Re A|)
// steps a state remembers -- the limit of the plain form in fp32.
__device__ __forceinline__ void abar_minus_one(float x, float t, float &dr, float &di) {
    const float em1 = expm1_f(x);
    float s, c, cm1;
    sincos_cm1(t, s, c, cm1);
    dr = fmaf(em1, c, cm1);
    di = fmaf(em1, s, s);
}

template <typename T, int R>
__global__ void __launch_bounds__(kCThreads) scan_fwd_complex_kernel(const CParams p) {
    using G = CGeom<T, R>;
    constexpr int S = G::S, CG = G::CG, V = G::V, TC = G::TC, TCP = G::TCP;
    constexpr int VPR = G::VPR, BVR = G::BVR, STAGE = G::STAGE;
    constexpr int OWN = 4 / R;  // outputs per lane per 4 timesteps
    // fp32 activations: Abar - 1 from FMA-pipe polynomials (abar_minus_one);
    // bf16, whose tolerance is 200x looser: Abar from the special-function
    // unit (ex2, sin, cos)
    constexpr bool kAccurate = sizeof(T) == 4;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *sDelta = reinterpret_cast<float *>(smem_raw);       // [CG][TCP]: delta, then y
    float *sDu = sDelta + CG * TCP;                            // [CG][TCP]: delta * u
    float2 *sB = reinterpret_cast<float2 *>(sDu + CG * TCP);   // [TC][kCNP]
    float2 *sC = sB + TC * kCNP;                               // [TC][kCNP]
    T *rawBase = reinterpret_cast<T *>(sC + TC * kCNP);        // 2 stages

    const int tid = threadIdx.x;
    const int64_t grp = blockIdx.x % p.n_groups;
    const int64_t b = blockIdx.x / p.n_groups;
    const int64_t d0 = grp * CG;
    const int64_t L = p.seqlen, Dm = p.dim;
    const int N = p.dstate;
    const bool has_z = p.z != nullptr;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B);
    const T *gC = static_cast<const T *>(p.C);
    T *gout = static_cast<T *>(p.out);
    const int64_t row0 = (b * Dm + d0) * L;  // this block's first channel row
    const int64_t bc0 = b * N * L * 2;       // B[b] / C[b], interleaved pairs

    // ---- this thread: channel c, lane r, complex states r*S .. r*S+S-1
    const int c = tid / R, r = tid % R;
    const int64_t d = d0 + c;
    float Are[S], Aim[S], hr[S], hi[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int n = r * S + s;
        const bool ok = d < Dm && n < N;
        Are[s] = ok ? __ldg(p.A + (d * N + n) * 2) * (kAccurate ? 1.f : kLog2e) : 0.f;
        Aim[s] = ok ? __ldg(p.A + (d * N + n) * 2 + 1) : 0.f;
        hr[s] = (ok && p.h0) ? __ldcg(p.h0 + ((b * Dm + d) * N + n) * 2) : 0.f;
        hi[s] = (ok && p.h0) ? __ldcg(p.h0 + ((b * Dm + d) * N + n) * 2 + 1) : 0.f;
    }

    auto issue_loads = [&](int64_t t0, int st) {
        T *rU = rawBase + st * STAGE;
        T *rD = rU + CG * TC;
        T *rZ = rD + CG * TC;
        T *rB = rZ + CG * TC;
        T *rC = rB + kCNP * 2 * TC;
        if (p.vec) {
            for (int vi = tid; vi < CG * VPR; vi += kCThreads) {
                const int pc = vi / VPR, tv = vi % VPR;
                const int64_t t = t0 + tv * V;
                const bool ok = (d0 + pc < Dm) && (t < L);
                const int64_t off = ok ? row0 + pc * L + t : 0;
                cpa16(rU + pc * TC + tv * V, gu + off, ok);
                cpa16(rD + pc * TC + tv * V, gd + off, ok);
                if (has_z) cpa16(rZ + pc * TC + tv * V, gz + off, ok);
            }
            for (int vi = tid; vi < 2 * kCNP * BVR; vi += kCThreads) {
                const int which = vi / (kCNP * BVR), rem = vi % (kCNP * BVR);
                const int n = rem / BVR, bv = rem % BVR;
                const int64_t e = 2 * t0 + bv * V;  // element along the interleaved row
                const bool ok = (n < N) && (e < 2 * L);
                const int64_t off = ok ? bc0 + (int64_t)n * 2 * L + e : 0;
                cpa16((which ? rC : rB) + n * 2 * TC + bv * V, (which ? gC : gB) + off, ok);
            }
        } else {
            for (int e = tid; e < CG * TC; e += kCThreads) {
                const int pc = e / TC, tt = e % TC;
                const int64_t t = t0 + tt;
                const bool ok = (d0 + pc < Dm) && (t < L);
                const int64_t off = row0 + pc * L + t;
                rU[e] = ok ? gu[off] : T(0.f);
                rD[e] = ok ? gd[off] : T(0.f);
                if (has_z) rZ[e] = ok ? gz[off] : T(0.f);
            }
            for (int e = tid; e < 2 * kCNP * 2 * TC; e += kCThreads) {
                const int which = e / (kCNP * 2 * TC), rem = e % (kCNP * 2 * TC);
                const int n = rem / (2 * TC), k = rem % (2 * TC);
                const bool ok = (n < N) && (2 * t0 + k < 2 * L);
                const int64_t off = bc0 + (int64_t)n * 2 * L + 2 * t0 + k;
                (which ? rC : rB)[rem] = ok ? (which ? gC : gB)[off] : T(0.f);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    issue_loads(0, 0);
    int stage = 0;
#pragma unroll 1
    for (int64_t t0 = 0; t0 < L; t0 += TC, stage ^= 1) {
        const T *rU = rawBase + stage * STAGE;
        const T *rD = rU + CG * TC;
        const T *rZ = rD + CG * TC;
        const T *rB = rZ + CG * TC;
        const T *rC = rB + kCNP * 2 * TC;
        const int tvalid = (L - t0) < TC ? (int)(L - t0) : TC;
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();

        // ---- prologue: delta and delta * u per element; B / C widened to
        // fp32 complex pairs [t][n]
        for (int vi = tid; vi < CG * VPR; vi += kCThreads) {
            const int pc = vi / VPR, tv = vi % VPR;
            const int64_t dd = d0 + pc;
            const float bias = (dd < Dm && p.delta_bias) ? __ldg(p.delta_bias + dd) : 0.f;
            float fu[V], fd[V];
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rD + pc * TC + tv * V), fd);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float dl = fd[i] + bias;
                if (p.softplus) dl = kAccurate ? softplus_precise(dl) : softplus_f(dl);
                if (tv * V + i >= tvalid) dl = 0.f;  // past the end: Abar = 1, no input
                fd[i] = dl;
                fu[i] = dl * fu[i];
            }
#pragma unroll
            for (int i = 0; i < V; i += 4) {
                *reinterpret_cast<float4 *>(sDelta + pc * TCP + tv * V + i) =
                    make_float4(fd[i], fd[i + 1], fd[i + 2], fd[i + 3]);
                *reinterpret_cast<float4 *>(sDu + pc * TCP + tv * V + i) =
                    make_float4(fu[i], fu[i + 1], fu[i + 2], fu[i + 3]);
            }
        }
        for (int vi = tid; vi < 2 * kCNP * BVR; vi += kCThreads) {
            const int which = vi / (kCNP * BVR), rem = vi % (kCNP * BVR);
            const int n = rem / BVR, bv = rem % BVR;
            float f[V];
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>((which ? rC : rB) + n * 2 * TC + bv * V), f);
            float2 *dst = (which ? sC : sB) + (bv * (V / 2)) * kCNP + n;
#pragma unroll
            for (int k = 0; k < V / 2; ++k) dst[k * kCNP] = make_float2(f[2 * k], f[2 * k + 1]);
        }

        if (t0 + TC < L) issue_loads(t0 + TC, stage ^ 1);
        __syncthreads();

        // ---- scan: thread (c, r) advances its S complex states
        {
            float *dRow = sDelta + c * TCP;
            const float *uRow = sDu + c * TCP;
#pragma unroll 1
            for (int tb = 0; tb < tvalid; tb += 4) {
                const float4 dl4 = *reinterpret_cast<const float4 *>(dRow + tb);
                const float4 du4 = *reinterpret_cast<const float4 *>(uRow + tb);
                const float dls[4] = {dl4.x, dl4.y, dl4.z, dl4.w};
                const float dus[4] = {du4.x, du4.y, du4.z, du4.w};
                float yp[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float dl = dls[q], du = dus[q];
                    const float4 *Bt = reinterpret_cast<const float4 *>(sB + (tb + q) * kCNP + r * S);
                    const float4 *Ct = reinterpret_cast<const float4 *>(sC + (tb + q) * kCNP + r * S);
                    float y = 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < S / 2; ++s2) {  // two complex states per 16-byte read
                        const float4 bb = Bt[s2], cc = Ct[s2];
                        const float br[2] = {bb.x, bb.z}, bi[2] = {bb.y, bb.w};
                        const float cr[2] = {cc.x, cc.z}, ci[2] = {cc.y, cc.w};
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const int s = 2 * s2 + k;
                            float nr, ni;
                            if (kAccurate) {
                                float dr, di;
                                abar_minus_one(dl * Are[s], dl * Aim[s], dr, di);
                                nr = hr[s] + fmaf(dr, hr[s], fmaf(-di, hi[s], du * br[k]));
                                ni = hi[s] + fmaf(dr, hi[s], fmaf(di, hr[s], du * bi[k]));
                            } else {
                                const float mag = ex2_mufu(dl * Are[s]);
                                float sn, cs;
                                sincos_mufu(reduce_angle(dl * Aim[s]), sn, cs);
                                const float ar = mag * cs, ai = mag * sn;
                                nr = fmaf(ar, hr[s], fmaf(-ai, hi[s], du * br[k]));
                                ni = fmaf(ar, hi[s], fmaf(ai, hr[s], du * bi[k]));
                            }
                            hr[s] = nr;
                            hi[s] = ni;
                            y = fmaf(cr[k], nr, fmaf(-ci[k], ni, y));
                        }
                    }
                    yp[q] = y;
                }
                // sum over the R lanes of the channel; lane r keeps outputs
                // [r * OWN, (r + 1) * OWN) of the four timesteps
                if (R >= 4) {
                    const bool up = (r & 2) != 0;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float send = up ? yp[i] : yp[i + 2];
                        const float keep = up ? yp[i + 2] : yp[i];
                        yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    }
                }
                if (R >= 2) {
                    constexpr int H = R >= 4 ? 1 : 2;  // live values per lane after the round
                    const bool up = (r & 1) != 0;
#pragma unroll
                    for (int i = 0; i < H; ++i) {
                        const float send = up ? yp[i] : yp[i + H];
                        const float keep = up ? yp[i + H] : yp[i];
                        yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                    }
                }
                __syncwarp();  // every lane of the channel has read dRow[tb .. tb + 4)
#pragma unroll
                for (int i = 0; i < OWN; ++i) dRow[tb + r * OWN + i] = yp[i];
            }
        }
        __syncthreads();

        // ---- epilogue: out = (y + D u) * silu(z)
        for (int vi = tid; vi < CG * VPR; vi += kCThreads) {
            const int pc = vi / VPR, tv = vi % VPR;
            const int64_t dd = d0 + pc;
            const int64_t t = t0 + tv * V;
            if (dd >= Dm || tv * V >= tvalid) continue;
            const float Dd = p.D ? __ldg(p.D + dd) : 0.f;
            float fu[V], fz[V], y[V];
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
            if (has_z) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rZ + pc * TC + tv * V), fz);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                float o = fmaf(Dd, fu[i], sDelta[pc * TCP + tv * V + i]);
                if (has_z) o *= silu_f(fz[i]);
                y[i] = o;
            }
            T *dst = gout + row0 + pc * L + t;
            if (p.vec) {
                stg16_stream(dst, Elem<T>::pack(y));
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (tv * V + i < tvalid) Elem<T>::store(dst + i, y[i]);
            }
        }
    }

    if (p.last_state != nullptr && d < Dm) {
        float *ls = p.last_state + (b * Dm + d) * N * 2;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int n = r * S + s;
            if (n < N) {
                ls[2 * n] = hr[s];
                ls[2 * n + 1] = hi[s];
            }
        }
    }
}

template <typename T, int R>
cudaError_t launch_r(const CParams &p0, int64_t batch, cudaStream_t st) {
    using G = CGeom<T, R>;
    CParams p = p0;
    const int64_t groups = (p.dim + G::CG - 1) / G::CG;
    const int64_t blocks = batch * groups;
    if (blocks <= 0 || blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    p.n_groups = (int)groups;
    auto kern = scan_fwd_complex_kernel<T, R>;
    if (G::SMEM > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)blocks, kCThreads, G::SMEM, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const CParams &p, int64_t batch, int lanes, cudaStream_t st) {
    switch (lanes) {
        case 1: return launch_r<T, 1>(p, batch, st);
        case 2: return launch_r<T, 2>(p, batch, st);
        default: return launch_r<T, 4>(p, batch, st);
    }
}

}  // namespace

// Lanes per channel: the one with the least work on the busiest SM
// sub-partition, counting 16 / R state-steps per warp-timestep and the
// cross-lane sums' overhead.
int complex_scan_lanes(int64_t batch, int64_t dim, int sm_count) {
    const double smsp = 4.0 * (sm_count > 0 ? sm_count : 148);
    const double rows = (double)batch * (double)dim;
    const double overhead[3] = {1.0, 1.04, 1.10};
    int best_r = 1;
    double best = 1e300;
    for (int i = 0, r = 1; r <= 4; ++i, r *= 2) {
        const double warps = rows * r / 32.0;
        const double per = warps / smsp;
        const double busiest = per <= 1.0 ? 1.0 : (double)(int64_t)(per + 0.999999);
        const double cost = busiest * (kCNP / r) * overhead[i];
        if (cost < best - 1e-9) { best = cost; best_r = r; }
    }
    return best_r;
}

cudaError_t launch_scan_fwd_complex(const ScanArgs &a, int lanes, cudaStream_t st) {
    CParams p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z;
    p.A = a.A; p.D = a.D; p.delta_bias = a.delta_bias;
    p.out = a.out; p.last_state = a.last_state; p.h0 = a.h0;
    p.dim = a.dim; p.seqlen = a.seqlen; p.n_groups = 0;
    p.dstate = a.dstate; p.softplus = a.softplus;
    const int V = a.act == kBF16 ? 8 : 4;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    p.vec = (a.seqlen % V == 0) && al(a.u) && al(a.delta) && al(a.z) && al(a.B) && al(a.C) && al(a.out);
    return a.act == kBF16 ? launch_t<__nv_bfloat16>(p, a.batch, lanes, st)
                          : launch_t<float>(p, a.batch, lanes, st);
}

}  // namespace mscan
