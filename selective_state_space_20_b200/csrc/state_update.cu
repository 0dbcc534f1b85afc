// state_update.cu -- one recurrent step of the selective SSM with the fp32
// state resident in HBM, updated in place: the decoding form (one token per
// call) of the recurrence h = Abar h + Bbar u, y = C h + D u, gated by silu(z)
// ("Mamba SSM concept and implementation in Keras and TensorFlow", recurrent
// form; mamba-jax sample.py generation loop).
//
// The step is bound by HBM traffic: 2 * 4 * N bytes of state per channel
// against ~N exponentials.  The main kernel gives each (batch, channel) row
// a few lanes with two 16-byte state slices each (N = 16: two lanes), so a
// warp's state loads and stores cover whole 32-byte sectors and the per-row
// work (softplus, gate) is shared by fewer lanes; the row's readout is summed
// over its lanes with shuffles.  Thread indices are 32-bit where they fit
// (a 64-bit division by dim per thread cost ~20 % of the step).  A rows are
// re-read by every batch row and stay in L2, B and C rows are shared by all
// channels of a batch row and stay in L1.  Other state sizes and unaligned
// tensors take a thread-per-row kernel.  fp32 activations take the accurate decay of
// device_math.cuh (Decay<true>), bf16 ones one ex2 per state.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.cuh"
#include "device_math.cuh"
#include "internal.h"

namespace mscan {

struct SUParams {
    float *state;
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    int64_t rows, dim;
    int dstate;
    int softplus;
    // byte ranges of the pointer arguments, for the bounds-checked build
    MSCAN_EXTENTS(x_state, x_u, x_delta, x_B, x_C, x_z, x_A, x_D, x_bias, x_out)
};

// Loads that the bounds-checked build tests against the tensor's range (a
// load outside reads zero; see bounds.cuh).
#ifdef MSCAN_BOUNDS_CHECK
template <typename T>
__device__ __forceinline__ float load_chk(const Extent &e, const T *q, int site) {
    return MSCAN_WITHIN(e, q, sizeof(T), site) ? Elem<T>::load(q) : 0.f;
}
__device__ __forceinline__ float ldg_chk(const Extent &e, const float *q, int site) {
    return MSCAN_WITHIN(e, q, 4, site) ? __ldg(q) : 0.f;
}
#else
template <typename T>
__device__ __forceinline__ float load_plain(const T *q) { return Elem<T>::load(q); }
#define load_chk(e, q, site) load_plain(q)
#define ldg_chk(e, q, site) __ldg(q)
#endif

// NV > 0: dstate == NV, known at compile time, 16-byte state accesses.
// NV == 0: any dstate, scalar accesses.
template <typename T, int NV>
__global__ void __launch_bounds__(256)
state_update_kernel(const SUParams p) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= p.rows) return;
    const int64_t b = row / p.dim, d = row % p.dim;
    const int N = NV > 0 ? NV : p.dstate;
    const T *gu = static_cast<const T *>(p.u);
    const T *gd = static_cast<const T *>(p.delta);
    const T *gz = static_cast<const T *>(p.z);
    const T *gB = static_cast<const T *>(p.B) + b * N;
    const T *gC = static_cast<const T *>(p.C) + b * N;
    const float *Ad = p.A + d * N;
    using Dk = Decay<sizeof(T) == 4>;

    float dl = load_chk(p.x_delta, gd + row, kSiteDelta) +
               (p.delta_bias ? ldg_chk(p.x_bias, p.delta_bias + d, kSiteBias) : 0.f);
    if (p.softplus) dl = Dk::softplus(dl);
    const float ut = load_chk(p.x_u, gu + row, kSiteU);
    const float du = dl * ut;
    const float dl2 = dl * Dk::kScale;
    float *st = p.state + row * N;
    using HS = typename Dk::H;  // fp64 for fp32 activations
    HS y = 0.f;
    if (NV > 0) {
#pragma unroll
        for (int n = 0; n < N; n += 4) {
            const bool sok = MSCAN_WITHIN(p.x_state, st + n, 16, kSiteState);
            float4 h = sok ? *reinterpret_cast<const float4 *>(st + n) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 a4 = MSCAN_WITHIN(p.x_A, Ad + n, 16, kSiteA) ? __ldg(reinterpret_cast<const float4 *>(Ad + n))
                                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            HS hv[4] = {h.x, h.y, h.z, h.w};
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                hv[i] = Dk::step(dl2 * av[i], hv[i], du * load_chk(p.x_B, gB + n + i, kSiteB));
                y = fma((HS)load_chk(p.x_C, gC + n + i, kSiteC), hv[i], y);
            }
            if (sok)
                *reinterpret_cast<float4 *>(st + n) =
                    make_float4((float)hv[0], (float)hv[1], (float)hv[2], (float)hv[3]);
        }
    } else {
        for (int n = 0; n < N; ++n) {
            const bool sok = MSCAN_WITHIN(p.x_state, st + n, 4, kSiteState);
            const HS hn = Dk::step(dl2 * ldg_chk(p.x_A, Ad + n, kSiteA), (HS)(sok ? st[n] : 0.f),
                                   du * load_chk(p.x_B, gB + n, kSiteB));
            if (sok) st[n] = (float)hn;
            y = fma((HS)load_chk(p.x_C, gC + n, kSiteC), hn, y);
        }
    }
    float yo = (float)y;
    if (p.D) yo = (float)fma((HS)ldg_chk(p.x_D, p.D + d, kSiteD), (HS)ut, y);
    if (gz) yo *= silu_f(load_chk(p.x_z, gz + row, kSiteZ));
    T *o = static_cast<T *>(p.out) + row;
    if (MSCAN_WITHIN(p.x_out, o, sizeof(T), kSiteOut)) Elem<T>::store(o, yo);
}

// Four states per lane: bf16 / fp32 loads of four consecutive B or C values.
template <typename T> struct Quad;
template <> struct Quad<float> {
    __device__ __forceinline__ static float4 load(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
};
template <> struct Quad<__nv_bfloat16> {
    __device__ __forceinline__ static float4 load(const __nv_bfloat16 *p) {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        float4 f;
        Elem<__nv_bfloat16>::unpack2(w.x, f.x, f.y);
        Elem<__nv_bfloat16>::unpack2(w.y, f.z, f.w);
        return f;
    }
};

// NV / (4 V) = Q lanes per row (NV = dstate, a multiple of 4 up to 128);
// lane q of a row owns the V 16-byte state slices q, q + Q, ..., so each load
// or store instruction of a warp covers whole 32-byte sectors (a row's Q
// lanes side by side), and a row's readout is summed over its lanes with
// shuffles.  Every load is issued before the arithmetic.  W64: 64-bit thread
// indices (more than 2^31 lanes).
template <typename T, int NV, int V, bool W64>
__global__ void __launch_bounds__(256)
state_update_lanes_kernel(const SUParams p) {
    constexpr int Q = NV / (4 * V);
    static_assert(Q >= 1 && Q <= 32 && (Q & (Q - 1)) == 0 && Q * 4 * V == NV, "lanes per row: a power of two");
    using Idx = typename std::conditional<W64, int64_t, unsigned>::type;
    const Idx gid = (Idx)blockIdx.x * blockDim.x + threadIdx.x;
    const Idx rows = (Idx)p.rows, dim = (Idx)p.dim;
    const bool live = gid / Q < rows;
    const Idx row = live ? gid / Q : rows - 1;  // idle lanes still join the shuffles
    const int qi = (int)(gid % Q);
    const Idx b = row / dim, d = row - b * dim;
    using Dk = Decay<sizeof(T) == 4>;
    using HS = typename Dk::H;  // fp64 for fp32 activations

    float4 h4[V], a4[V], b4[V], c4[V];
    float4 *st = reinterpret_cast<float4 *>(p.state + (int64_t)row * NV) + qi;
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const float4 *a = reinterpret_cast<const float4 *>(p.A + (int64_t)d * NV) + qi + v * Q;
        const T *bq = static_cast<const T *>(p.B) + (int64_t)b * NV + 4 * (qi + v * Q);
        const T *cq = static_cast<const T *>(p.C) + (int64_t)b * NV + 4 * (qi + v * Q);
        h4[v] = MSCAN_WITHIN(p.x_state, st + v * Q, 16, kSiteState) ? st[v * Q] : zero4;
        a4[v] = MSCAN_WITHIN(p.x_A, a, 16, kSiteA) ? __ldg(a) : zero4;
        b4[v] = MSCAN_WITHIN(p.x_B, bq, 4 * sizeof(T), kSiteB) ? Quad<T>::load(bq) : zero4;
        c4[v] = MSCAN_WITHIN(p.x_C, cq, 4 * sizeof(T), kSiteC) ? Quad<T>::load(cq) : zero4;
    }
    const float dr = load_chk(p.x_delta, static_cast<const T *>(p.delta) + row, kSiteDelta);
    const float ut = load_chk(p.x_u, static_cast<const T *>(p.u) + row, kSiteU);
    const float zt = (p.z && qi == 0) ? load_chk(p.x_z, static_cast<const T *>(p.z) + row, kSiteZ) : 0.f;
    const float bias = p.delta_bias ? ldg_chk(p.x_bias, p.delta_bias + d, kSiteBias) : 0.f;
    const float Dd = (p.D && qi == 0) ? ldg_chk(p.x_D, p.D + d, kSiteD) : 0.f;

    float dl = dr + bias;
    if (p.softplus) dl = Dk::softplus(dl);
    const float du = dl * ut;
    const float dl2 = dl * Dk::kScale;
    HS y = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const HS hx = Dk::step(dl2 * a4[v].x, (HS)h4[v].x, du * b4[v].x);
        const HS hy = Dk::step(dl2 * a4[v].y, (HS)h4[v].y, du * b4[v].y);
        const HS hz = Dk::step(dl2 * a4[v].z, (HS)h4[v].z, du * b4[v].z);
        const HS hw = Dk::step(dl2 * a4[v].w, (HS)h4[v].w, du * b4[v].w);
        y += fma((HS)c4[v].x, hx, fma((HS)c4[v].y, hy, fma((HS)c4[v].z, hz, (HS)c4[v].w * hw)));
        h4[v] = make_float4((float)hx, (float)hy, (float)hz, (float)hw);
    }
#pragma unroll
    for (int o = Q / 2; o >= 1; o >>= 1) y += __shfl_xor_sync(0xffffffffu, y, o);
    if (!live) return;
#pragma unroll
    for (int v = 0; v < V; ++v)
        if (MSCAN_WITHIN(p.x_state, st + v * Q, 16, kSiteState)) st[v * Q] = h4[v];
    if (qi == 0) {
        float yo = (float)y;
        if (p.D) yo = (float)fma((HS)Dd, (HS)ut, y);
        if (p.z) yo *= silu_f(zt);
        T *o = static_cast<T *>(p.out) + row;
        if (MSCAN_WITHIN(p.x_out, o, sizeof(T), kSiteOut)) Elem<T>::store(o, yo);
    }
}

template <typename T, int NV>
static cudaError_t launch_lanes(const SUParams &kp, cudaStream_t st) {
    constexpr int threads = 256;
    constexpr int V = NV >= 8 ? 2 : 1;  // 16-byte state slices per lane
    constexpr int Q = NV / (4 * V);
    const int64_t lanes = kp.rows * Q;
    const int64_t blocks = (lanes + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (blocks * threads < 0x7fffffffLL)
        state_update_lanes_kernel<T, NV, V, false><<<(unsigned)blocks, threads, 0, st>>>(kp);
    else
        state_update_lanes_kernel<T, NV, V, true><<<(unsigned)blocks, threads, 0, st>>>(kp);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_rows(const SUParams &kp, cudaStream_t st) {
    const int threads = 256;
    const int64_t blocks = (kp.rows + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const bool vec = (reinterpret_cast<uintptr_t>(kp.state) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(kp.A) & 15) == 0;
    if (vec && kp.dstate == 16)
        state_update_kernel<T, 16><<<(unsigned)blocks, threads, 0, st>>>(kp);
    else if (vec && kp.dstate == 8)
        state_update_kernel<T, 8><<<(unsigned)blocks, threads, 0, st>>>(kp);
    else if (vec && kp.dstate == 32)
        state_update_kernel<T, 32><<<(unsigned)blocks, threads, 0, st>>>(kp);
    else if (vec && kp.dstate == 64)
        state_update_kernel<T, 64><<<(unsigned)blocks, threads, 0, st>>>(kp);
    else
        state_update_kernel<T, 0><<<(unsigned)blocks, threads, 0, st>>>(kp);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_typed(const SUParams &kp, cudaStream_t st) {
    auto al = [](const void *q, uintptr_t m) { return (reinterpret_cast<uintptr_t>(q) & (m - 1)) == 0; };
    const uintptr_t bc_align = 4 * sizeof(T);  // four B / C values per load
    if (al(kp.state, 16) && al(kp.A, 16) && al(kp.B, bc_align) && al(kp.C, bc_align)) {
        if (kp.dstate == 16) return launch_lanes<T, 16>(kp, st);
        if (kp.dstate == 8) return launch_lanes<T, 8>(kp, st);
        if (kp.dstate == 32) return launch_lanes<T, 32>(kp, st);
        if (kp.dstate == 64) return launch_lanes<T, 64>(kp, st);
        if (kp.dstate == 4) return launch_lanes<T, 4>(kp, st);
    }
    return launch_rows<T>(kp, st);
}

MSCAN_BOUNDS_TAKE(state_update_bounds_take)

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t st) {
    SUParams kp;
    kp.state = a.state; kp.u = a.u; kp.delta = a.delta; kp.B = a.B; kp.C = a.C; kp.z = a.z;
    kp.A = a.A; kp.D = a.D; kp.delta_bias = a.delta_bias; kp.out = a.out;
    kp.rows = a.batch * a.dim; kp.dim = a.dim; kp.dstate = a.dstate; kp.softplus = a.softplus;
#ifdef MSCAN_BOUNDS_CHECK
    const unsigned long long es = a.act == kBF16 ? 2 : 4, rows = (unsigned long long)(a.batch * a.dim);
    const unsigned long long xb = rows * es;
    kp.x_state = extent_of(a.state, rows * a.dstate * 4);
    kp.x_u = extent_of(a.u, xb);
    kp.x_delta = extent_of(a.delta, xb);
    kp.x_z = extent_of(a.z, xb);
    kp.x_B = extent_of(a.B, (unsigned long long)(a.batch * a.dstate) * es);
    kp.x_C = extent_of(a.C, (unsigned long long)(a.batch * a.dstate) * es);
    kp.x_A = extent_of(a.A, (unsigned long long)(a.dim * a.dstate) * 4);
    kp.x_D = extent_of(a.D, (unsigned long long)a.dim * 4);
    kp.x_bias = extent_of(a.delta_bias, (unsigned long long)a.dim * 4);
    kp.x_out = extent_of(a.out, xb > (unsigned long long)g_out_extent_shrink ? xb - g_out_extent_shrink : 0);
#endif
    if (a.act == kBF16) return launch_typed<__nv_bfloat16>(kp, st);
    return launch_typed<float>(kp, st);
}

}  // namespace mscan
