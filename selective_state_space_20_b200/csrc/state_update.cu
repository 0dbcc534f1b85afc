// state_update.cu -- one recurrent step of the selective SSM with the fp32
// state resident in HBM, updated in place: the decoding form (one token per
// call) of the recurrence h = Abar h + Bbar u, y = C h + D u, gated by silu(z)
// ("Mamba SSM concept and implementation in Keras and TensorFlow", recurrent
// form; mamba-jax sample.py generation loop).
//
// The step is bound by HBM traffic: 2 * 4 * N bytes of state per channel
// against ~N exponentials.  One thread owns one (batch, channel) row and
// streams its N states with 16-byte loads and stores; A rows are re-read by
// every batch row and stay in L2, B and C rows are shared by all channels of a
// batch row and stay in L1.
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

    float dl = Elem<T>::load(gd + row) + (p.delta_bias ? __ldg(p.delta_bias + d) : 0.f);
    if (p.softplus) dl = softplus_f(dl);
    const float ut = Elem<T>::load(gu + row);
    const float du = dl * ut;
    const float dl2 = dl * kLog2e;
    float *st = p.state + row * N;
    float y = 0.f;
    if (NV > 0) {
#pragma unroll
        for (int n = 0; n < N; n += 4) {
            float4 h = *reinterpret_cast<const float4 *>(st + n);
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(Ad + n));
            float hv[4] = {h.x, h.y, h.z, h.w};
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = ex2_mufu(dl2 * av[i]);
                hv[i] = fmaf(a, hv[i], du * Elem<T>::load(gB + n + i));
                y = fmaf(Elem<T>::load(gC + n + i), hv[i], y);
            }
            *reinterpret_cast<float4 *>(st + n) = make_float4(hv[0], hv[1], hv[2], hv[3]);
        }
    } else {
        for (int n = 0; n < N; ++n) {
            const float a = ex2_mufu(dl2 * __ldg(Ad + n));
            const float hn = fmaf(a, st[n], du * Elem<T>::load(gB + n));
            st[n] = hn;
            y = fmaf(Elem<T>::load(gC + n), hn, y);
        }
    }
    if (p.D) y = fmaf(__ldg(p.D + d), ut, y);
    if (gz) y *= silu_f(Elem<T>::load(gz + row));
    Elem<T>::store(static_cast<T *>(p.out) + row, y);
}

template <typename T>
static cudaError_t launch_typed(const SUParams &kp, cudaStream_t st) {
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

cudaError_t launch_state_update(const StateUpdateArgs &a, cudaStream_t st) {
    SUParams kp;
    kp.state = a.state; kp.u = a.u; kp.delta = a.delta; kp.B = a.B; kp.C = a.C; kp.z = a.z;
    kp.A = a.A; kp.D = a.D; kp.delta_bias = a.delta_bias; kp.out = a.out;
    kp.rows = a.batch * a.dim; kp.dim = a.dim; kp.dstate = a.dstate; kp.softplus = a.softplus;
    if (a.act == kBF16) return launch_typed<__nv_bfloat16>(kp, st);
    return launch_typed<float>(kp, st);
}

}  // namespace mscan
