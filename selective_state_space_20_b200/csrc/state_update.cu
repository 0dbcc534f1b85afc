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
};

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

    float dl = Elem<T>::load(gd + row) + (p.delta_bias ? __ldg(p.delta_bias + d) : 0.f);
    if (p.softplus) dl = Dk::softplus(dl);
    const float ut = Elem<T>::load(gu + row);
    const float du = dl * ut;
    const float dl2 = dl * Dk::kScale;
    float *st = p.state + row * N;
    using HS = typename Dk::H;  // fp64 for fp32 activations
    HS y = 0.f;
    if (NV > 0) {
#pragma unroll
        for (int n = 0; n < N; n += 4) {
            float4 h = *reinterpret_cast<const float4 *>(st + n);
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(Ad + n));
            HS hv[4] = {h.x, h.y, h.z, h.w};
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                hv[i] = Dk::step(dl2 * av[i], hv[i], du * Elem<T>::load(gB + n + i));
                y = fma((HS)Elem<T>::load(gC + n + i), hv[i], y);
            }
            *reinterpret_cast<float4 *>(st + n) = make_float4((float)hv[0], (float)hv[1], (float)hv[2], (float)hv[3]);
        }
    } else {
        for (int n = 0; n < N; ++n) {
            const HS hn = Dk::step(dl2 * __ldg(Ad + n), (HS)st[n], du * Elem<T>::load(gB + n));
            st[n] = (float)hn;
            y = fma((HS)Elem<T>::load(gC + n), hn, y);
        }
    }
    float yo = (float)y;
    if (p.D) yo = (float)fma((HS)__ldg(p.D + d), (HS)ut, y);
    if (gz) yo *= silu_f(Elem<T>::load(gz + row));
    Elem<T>::store(static_cast<T *>(p.out) + row, yo);
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
#pragma unroll
    for (int v = 0; v < V; ++v) {
        h4[v] = st[v * Q];
        a4[v] = __ldg(reinterpret_cast<const float4 *>(p.A + (int64_t)d * NV) + qi + v * Q);
        b4[v] = Quad<T>::load(static_cast<const T *>(p.B) + (int64_t)b * NV + 4 * (qi + v * Q));
        c4[v] = Quad<T>::load(static_cast<const T *>(p.C) + (int64_t)b * NV + 4 * (qi + v * Q));
    }
    const float dr = Elem<T>::load(static_cast<const T *>(p.delta) + row);
    const float ut = Elem<T>::load(static_cast<const T *>(p.u) + row);
    const float zt = (p.z && qi == 0) ? Elem<T>::load(static_cast<const T *>(p.z) + row) : 0.f;
    const float bias = p.delta_bias ? __ldg(p.delta_bias + d) : 0.f;
    const float Dd = (p.D && qi == 0) ? __ldg(p.D + d) : 0.f;

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
    for (int v = 0; v < V; ++v) st[v * Q] = h4[v];
    if (qi == 0) {
        float yo = (float)y;
        if (p.D) yo = (float)fma((HS)Dd, (HS)ut, y);
        if (p.z) yo *= silu_f(zt);
        Elem<T>::store(static_cast<T *>(p.out) + row, yo);
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

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t st) {
    SUParams kp;
    kp.state = a.state; kp.u = a.u; kp.delta = a.delta; kp.B = a.B; kp.C = a.C; kp.z = a.z;
    kp.A = a.A; kp.D = a.D; kp.delta_bias = a.delta_bias; kp.out = a.out;
    kp.rows = a.batch * a.dim; kp.dim = a.dim; kp.dstate = a.dstate; kp.softplus = a.softplus;
    if (a.act == kBF16) return launch_typed<__nv_bfloat16>(kp, st);
    return launch_typed<float>(kp, st);
}

}  // namespace mscan
