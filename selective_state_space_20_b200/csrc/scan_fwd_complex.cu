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
// third of the real scan's rate.  With fp32 activations the state, the decay
// and the readout are carried in fp64 (see kF64 below).  Layout of the work as in the real static kernel: a block
// owns one batch row and CG = 128 / R channels, R lanes per channel split the 16
// (padded) states, tiles of 32 timesteps are copied to shared memory with
// 16-byte cp.async into a double buffer; a prologue forms delta and delta*u
// once per element and widens B / C to fp32 [t][n] complex pairs shared by
// every channel of the block; partial readouts of a channel's R lanes are
// summed with a transposed butterfly; the epilogue applies D and the gate.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "bounds.cuh"
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
    // byte ranges of the pointer arguments, for the bounds-checked build
    MSCAN_EXTENTS(x_u, x_delta, x_z, x_B, x_C, x_A, x_D, x_bias, x_out, x_last, x_h0)
};

// fp32 activations carry delta, delta * u, the states and the readout in
// fp64 (see the kernel), bf16 ones in fp32.
template <typename T>
using CHi = typename std::conditional<sizeof(T) == 4, double, float>::type;

template <typename T, int R>
struct CGeom {
    using H = CHi<T>;
    static constexpr int S = kCNP / R;                  // complex states per lane
    static constexpr int CG = kCThreads / R;            // channels per block
    static constexpr int V = 16 / (int)sizeof(T);       // elements per 16 bytes
    static constexpr int TC = kCTC;
    static constexpr int TCP = TC + 4;                  // delta / delta u / y row pitch (elements of H)
    static constexpr int VPR = TC / V;                  // vectors per channel row per chunk
    static constexpr int BVR = 2 * TC / V;              // vectors per B / C state row per chunk
    static constexpr int STAGE = 3 * CG * TC + 2 * kCNP * 2 * TC;  // raw elements per stage
    static constexpr size_t SMEM =
        (size_t)2 * CG * TCP * sizeof(H) + (size_t)2 * TC * kCNP * 8 + (size_t)2 * STAGE * sizeof(T);
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

template <typename T, int R>
__global__ void __launch_bounds__(kCThreads) scan_fwd_complex_kernel(const CParams p) {
    using G = CGeom<T, R>;
    constexpr int S = G::S, CG = G::CG, V = G::V, TC = G::TC, TCP = G::TCP;
    constexpr int VPR = G::VPR, BVR = G::BVR, STAGE = G::STAGE;
    constexpr int OWN = 4 / R;  // outputs per lane per 4 timesteps
    // fp32 activations (tolerance 1e-4): delta, delta * u, the states, the
    // decay and the readout in fp64.  The complex recurrence amplifies
    // relative errors: a relative error e in delta turns a state by
    // e Im A / |Re A| over the ~1 / (delta |Re A|) steps it remembers (~100 e
    // for the highest frequencies of the usual initialisation), and an error
    // in a rotation angle or a bias in a decay adds up over those steps.
    // Exact arithmetic with delta alone rounded once to fp32 already measures
    // up to 4e-4 against the fp64 definition on long rows; in fp64 only the
    // final rounding of each output to fp32 remains.  bf16 activations
    // (tolerance 2e-2): everything in fp32, Abar from the special-function
    // unit (ex2, sin, cos).
    constexpr bool kF64 = sizeof(T) == 4;
    using H = CHi<T>;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    H *sDelta = reinterpret_cast<H *>(smem_raw);               // [CG][TCP]: delta, then y
    H *sDu = sDelta + CG * TCP;                                // [CG][TCP]: delta * u
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
    float Are[S], Aim[S];
    H hr[S], hi[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int n = r * S + s;
        const bool ok = d < Dm && n < N;
        const bool aok = ok && MSCAN_WITHIN(p.x_A, p.A + (d * N + n) * 2, 8, kSiteA);
        const bool hok = ok && p.h0 && MSCAN_WITHIN(p.x_h0, p.h0 + ((b * Dm + d) * N + n) * 2, 8, kSiteH0);
        Are[s] = aok ? __ldg(p.A + (d * N + n) * 2) * (kF64 ? 1.f : kLog2e) : 0.f;
        Aim[s] = aok ? __ldg(p.A + (d * N + n) * 2 + 1) : 0.f;
        hr[s] = hok ? __ldcg(p.h0 + ((b * Dm + d) * N + n) * 2) : 0.f;
        hi[s] = hok ? __ldcg(p.h0 + ((b * Dm + d) * N + n) * 2 + 1) : 0.f;
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
                cpa16(rU + pc * TC + tv * V, gu + off, ok && MSCAN_WITHIN(p.x_u, gu + off, 16, kSiteU));
                cpa16(rD + pc * TC + tv * V, gd + off, ok && MSCAN_WITHIN(p.x_delta, gd + off, 16, kSiteDelta));
                if (has_z) cpa16(rZ + pc * TC + tv * V, gz + off, ok && MSCAN_WITHIN(p.x_z, gz + off, 16, kSiteZ));
            }
            for (int vi = tid; vi < 2 * kCNP * BVR; vi += kCThreads) {
                const int which = vi / (kCNP * BVR), rem = vi % (kCNP * BVR);
                const int n = rem / BVR, bv = rem % BVR;
                const int64_t e = 2 * t0 + bv * V;  // element along the interleaved row
                const bool ok = (n < N) && (e < 2 * L);
                const int64_t off = ok ? bc0 + (int64_t)n * 2 * L + e : 0;
                cpa16((which ? rC : rB) + n * 2 * TC + bv * V, (which ? gC : gB) + off,
                      ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, (which ? gC : gB) + off, 16, which ? kSiteC : kSiteB));
            }
        } else {
            for (int e = tid; e < CG * TC; e += kCThreads) {
                const int pc = e / TC, tt = e % TC;
                const int64_t t = t0 + tt;
                const bool ok = (d0 + pc < Dm) && (t < L);
                const int64_t off = row0 + pc * L + t;
                rU[e] = (ok && MSCAN_WITHIN(p.x_u, gu + off, sizeof(T), kSiteU)) ? gu[off] : T(0.f);
                rD[e] = (ok && MSCAN_WITHIN(p.x_delta, gd + off, sizeof(T), kSiteDelta)) ? gd[off] : T(0.f);
                if (has_z) rZ[e] = (ok && MSCAN_WITHIN(p.x_z, gz + off, sizeof(T), kSiteZ)) ? gz[off] : T(0.f);
            }
            for (int e = tid; e < 2 * kCNP * 2 * TC; e += kCThreads) {
                const int which = e / (kCNP * 2 * TC), rem = e % (kCNP * 2 * TC);
                const int n = rem / (2 * TC), k = rem % (2 * TC);
                const bool ok = (n < N) && (2 * t0 + k < 2 * L);
                const int64_t off = bc0 + (int64_t)n * 2 * L + 2 * t0 + k;
                (which ? rC : rB)[rem] =
                    (ok && MSCAN_WITHIN(which ? p.x_C : p.x_B, (which ? gC : gB) + off, sizeof(T), which ? kSiteC : kSiteB))
                        ? (which ? gC : gB)[off] : T(0.f);
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
            const float bias = (dd < Dm && p.delta_bias && MSCAN_WITHIN(p.x_bias, p.delta_bias + dd, 4, kSiteBias))
                                   ? __ldg(p.delta_bias + dd) : 0.f;
            float fu[V], fd[V];
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rD + pc * TC + tv * V), fd);
            H hd[V], hu[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                H dl;
                if constexpr (kF64) {
                    dl = (double)fd[i] + (double)bias;
                    if (p.softplus) dl = fmax(dl, 0.0) + log1p(exp(-fabs(dl)));
                } else {
                    dl = fd[i] + bias;
                    if (p.softplus) dl = softplus_f(dl);
                }
                if (tv * V + i >= tvalid) dl = 0.f;  // past the end: Abar = 1, no input
                hd[i] = dl;
                hu[i] = dl * (H)fu[i];
            }
#pragma unroll
            for (int i = 0; i < V; ++i) {
                sDelta[pc * TCP + tv * V + i] = hd[i];
                sDu[pc * TCP + tv * V + i] = hu[i];
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
            H *dRow = sDelta + c * TCP;
            const H *uRow = sDu + c * TCP;
#pragma unroll 1
            for (int tb = 0; tb < tvalid; tb += 4) {
                H dls[4], dus[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    dls[q] = dRow[tb + q];
                    dus[q] = uRow[tb + q];
                }
                H yp[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const H dl = dls[q], du = dus[q];
                    const float4 *Bt = reinterpret_cast<const float4 *>(sB + (tb + q) * kCNP + r * S);
                    const float4 *Ct = reinterpret_cast<const float4 *>(sC + (tb + q) * kCNP + r * S);
                    H y = 0.f;
                    float2 yacc = f2(0.f, 0.f);  // bf16: (sum cr nr, sum ci ni), y = .x - .y
#pragma unroll
                    for (int s2 = 0; s2 < S / 2; ++s2) {  // two complex states per 16-byte read
                        const float4 bb = Bt[s2], cc = Ct[s2];
                        const float br[2] = {bb.x, bb.z}, bi[2] = {bb.y, bb.w};
                        const float cr[2] = {cc.x, cc.z}, ci[2] = {cc.y, cc.w};
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const int s = 2 * s2 + k;
                            H nr, ni;
                            if constexpr (kF64) {
                                const double mag = exp(dl * (double)Are[s]);
                                double sn, cs;
                                sincos(dl * (double)Aim[s], &sn, &cs);
                                const double ar = mag * cs, ai = mag * sn;
                                nr = fma(ar, hr[s], fma(-ai, hi[s], du * (double)br[k]));
                                ni = fma(ar, hi[s], fma(ai, hr[s], du * (double)bi[k]));
                                y = fma((double)cr[k], nr, fma(-(double)ci[k], ni, y));
                            } else {  // (re, im) pairs on the packed x2 instructions
                                const float2 x = __fmul2_rn(f2(dl, dl), f2(Are[s], Aim[s]));
                                const float mag = ex2_mufu(x.x);
                                float sn, cs;
                                sincos_mufu(reduce_angle(x.y), sn, cs);
                                const float2 a = __fmul2_rn(f2(mag, mag), f2(cs, sn));  // (ar, ai)
                                // (nr, ni) = (ar hr - ai hi, ar hi + ai hr) + du (br, bi)
                                float2 nn = __ffma2_rn(f2(-a.y, a.y), f2(hi[s], hr[s]),
                                                       __fmul2_rn(f2(du, du), f2(br[k], bi[k])));
                                nn = __ffma2_rn(f2(a.x, a.x), f2(hr[s], hi[s]), nn);
                                yacc = __ffma2_rn(f2(cr[k], ci[k]), nn, yacc);
                                nr = nn.x;
                                ni = nn.y;
                            }
                            hr[s] = nr;
                            hi[s] = ni;
                        }
                    }
                    if constexpr (!kF64) y = yacc.x - yacc.y;
                    yp[q] = y;
                }
                // sum over the R lanes of the channel; lane r keeps outputs
                // [r * OWN, (r + 1) * OWN) of the four timesteps
                if (R >= 4) {
                    const bool up = (r & 2) != 0;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const H send = up ? yp[i] : yp[i + 2];
                        const H keep = up ? yp[i + 2] : yp[i];
                        yp[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    }
                }
                if (R >= 2) {
                    constexpr int HV = R >= 4 ? 1 : 2;  // live values per lane after the round
                    const bool up = (r & 1) != 0;
#pragma unroll
                    for (int i = 0; i < HV; ++i) {
                        const H send = up ? yp[i] : yp[i + HV];
                        const H keep = up ? yp[i + HV] : yp[i];
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
            const float Dd = (p.D && MSCAN_WITHIN(p.x_D, p.D + dd, 4, kSiteD)) ? __ldg(p.D + dd) : 0.f;
            float fu[V], fz[V], y[V];
            Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rU + pc * TC + tv * V), fu);
            if (has_z) Elem<T>::unpack(*reinterpret_cast<const uint4 *>(rZ + pc * TC + tv * V), fz);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if constexpr (kF64) {
                    double o = fma((double)Dd, (double)fu[i], sDelta[pc * TCP + tv * V + i]);
                    if (has_z) o *= (double)fz[i] / (1.0 + exp(-(double)fz[i]));
                    y[i] = (float)o;
                } else {
                    float o = fmaf(Dd, fu[i], sDelta[pc * TCP + tv * V + i]);
                    if (has_z) o *= silu_f(fz[i]);
                    y[i] = o;
                }
            }
            T *dst = gout + row0 + pc * L + t;
            if (p.vec) {
                if (MSCAN_WITHIN(p.x_out, dst, 16, kSiteOut)) stg16_stream(dst, Elem<T>::pack(y));
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i)
                    if (tv * V + i < tvalid && MSCAN_WITHIN(p.x_out, dst + i, sizeof(T), kSiteOut))
                        Elem<T>::store(dst + i, y[i]);
            }
        }
    }

    if (p.last_state != nullptr && d < Dm) {
        float *ls = p.last_state + (b * Dm + d) * N * 2;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int n = r * S + s;
            if (n < N && MSCAN_WITHIN(p.x_last, ls + 2 * n, 8, kSiteLastState)) {
                ls[2 * n] = (float)hr[s];
                ls[2 * n + 1] = (float)hi[s];
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

MSCAN_BOUNDS_TAKE(complex_bounds_take)

cudaError_t launch_scan_fwd_complex(const ScanArgs &a, int lanes, cudaStream_t st) {
    CParams p;
    p.u = a.u; p.delta = a.delta; p.B = a.B; p.C = a.C; p.z = a.z;
    p.A = a.A; p.D = a.D; p.delta_bias = a.delta_bias;
    p.out = a.out; p.last_state = a.last_state; p.h0 = a.h0;
    p.dim = a.dim; p.seqlen = a.seqlen; p.n_groups = 0;
    p.dstate = a.dstate; p.softplus = a.softplus;
#ifdef MSCAN_BOUNDS_CHECK
    const unsigned long long es = a.act == kBF16 ? 2 : 4;
    const unsigned long long xb = (unsigned long long)(a.batch * a.dim * a.seqlen) * es;
    const unsigned long long bcb = (unsigned long long)(a.batch * a.dstate * a.seqlen) * 2 * es;
    const unsigned long long stb = (unsigned long long)(a.batch * a.dim * a.dstate) * 2 * 4;
    p.x_u = extent_of(a.u, xb);
    p.x_delta = extent_of(a.delta, xb);
    p.x_z = extent_of(a.z, xb);
    p.x_B = extent_of(a.B, bcb);
    p.x_C = extent_of(a.C, bcb);
    p.x_A = extent_of(a.A, (unsigned long long)(a.dim * a.dstate) * 2 * 4);
    p.x_D = extent_of(a.D, (unsigned long long)a.dim * 4);
    p.x_bias = extent_of(a.delta_bias, (unsigned long long)a.dim * 4);
    p.x_out = extent_of(a.out, xb > (unsigned long long)g_out_extent_shrink ? xb - g_out_extent_shrink : 0);
    p.x_last = extent_of(a.last_state, stb);
    p.x_h0 = extent_of(a.h0, stb);
#endif
    const int V = a.act == kBF16 ? 8 : 4;
    auto al = [](const void *q) { return q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    p.vec = (a.seqlen % V == 0) && al(a.u) && al(a.delta) && al(a.z) && al(a.B) && al(a.C) && al(a.out);
    return a.act == kBF16 ? launch_t<__nv_bfloat16>(p, a.batch, lanes, st)
                          : launch_t<float>(p, a.batch, lanes, st);
}

}  // namespace mscan
