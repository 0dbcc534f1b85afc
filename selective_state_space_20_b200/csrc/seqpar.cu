// seqpar.cu -- the two small kernels that let a sequence be cut into shards
// scanned on different GPUs.  The recurrence h_t = Abar_t h_{t-1} + x_t is
// affine in h, so a shard of timesteps maps its initial state h to
//   exp(A * sum_t delta_t) (.) h + h_local,
// h_local being the shard's final state from a zero start (the diagonal
// decays multiply: prod_t exp(delta_t A) = exp(A sum_t delta_t)).  Each rank
// scans its shard from zero, the ranks exchange (sum of delta, h_local), every
// rank folds the shards before its own into its true initial state, and
// scans its shard again from that state.
//
//   delta_sum_kernel : S[b, d] = sum_t softplus(delta_raw[b, d, t] + bias[d])
//                      (or without softplus), accumulated in fp64 -- a shard
//                      may hold 10^5..10^6 steps, and an fp32 running sum
//                      would lose ~L * 2^-24 of it.
//   state_fold_kernel: h <- exp(A[d, n] * S_k[b, d]) * h + h_local_k[b, d, n]
//                      for k = 0 .. count - 1 in order, from h_init (or 0).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

constexpr int kSumThreads = 256;

// One block per (b, d) row: each thread sums a strided slice of the row in
// fp64, then the block adds the 256 partial sums in a fixed tree order.
template <typename T, bool SP>
__global__ void __launch_bounds__(kSumThreads) delta_sum_kernel(const T *__restrict__ delta,
                                                                const float *__restrict__ bias,
                                                                double *__restrict__ out, int64_t dim,
                                                                int64_t seqlen) {
    __shared__ double part[kSumThreads];
    const int64_t row = blockIdx.x;
    const float bi = bias ? __ldg(bias + row % dim) : 0.f;
    const T *src = delta + row * seqlen;
    double acc = 0.0;
    for (int64_t t = threadIdx.x; t < seqlen; t += kSumThreads) {
        const float x = Elem<T>::load(src + t) + bi;
        // full-precision softplus: an error e in the sum turns into e |A| S
        // in the carried decay exp(A S)
        acc += (double)(SP ? fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))) : x);
    }
    part[threadIdx.x] = acc;
    __syncthreads();
#pragma unroll
    for (int s = kSumThreads / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[row] = part[0];
}

// One thread per (b, d, n).  Each thread reads all of its inputs before it
// writes h_out, so h_out may be h_init or one of the h_local slices.
__global__ void __launch_bounds__(256) state_fold_kernel(const float *h_init,
                                                         const double *__restrict__ sums,
                                                         const float *__restrict__ A,
                                                         const float *h_local, float *h_out, int64_t batch, int64_t dim,
                                                         int64_t dstate, int count) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = batch * dim * dstate;
    if (i >= total) return;
    const int64_t row = i / dstate;  // b * dim + d
    const int64_t n = i % dstate, d = row % dim;
    const double a = (double)__ldg(A + d * dstate + n);
    double h = h_init ? (double)h_init[i] : 0.0;
    for (int k = 0; k < count; ++k) {
        const double s = sums[(int64_t)k * batch * dim + row];
        h = exp(a * s) * h + (double)h_local[(int64_t)k * total + i];
    }
    h_out[i] = (float)h;
}

}  // namespace

cudaError_t launch_delta_sum(const void *delta, const float *bias, int softplus, double *out,
                             int64_t batch, int64_t dim, int64_t seqlen, int act, cudaStream_t st) {
    const int64_t rows = batch * dim;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const unsigned grid = (unsigned)rows;
    if (act == kBF16) {
        const auto *d = static_cast<const __nv_bfloat16 *>(delta);
        if (softplus) delta_sum_kernel<__nv_bfloat16, true><<<grid, kSumThreads, 0, st>>>(d, bias, out, dim, seqlen);
        else delta_sum_kernel<__nv_bfloat16, false><<<grid, kSumThreads, 0, st>>>(d, bias, out, dim, seqlen);
    } else {
        const auto *d = static_cast<const float *>(delta);
        if (softplus) delta_sum_kernel<float, true><<<grid, kSumThreads, 0, st>>>(d, bias, out, dim, seqlen);
        else delta_sum_kernel<float, false><<<grid, kSumThreads, 0, st>>>(d, bias, out, dim, seqlen);
    }
    return cudaGetLastError();
}

cudaError_t launch_state_fold(const float *h_init, const double *sums, const float *A,
                              const float *h_local, float *h_out, int64_t batch, int64_t dim,
                              int64_t dstate, int count, cudaStream_t st) {
    const int64_t total = batch * dim * dstate;
    const int64_t blocks = (total + 255) / 256;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    state_fold_kernel<<<(unsigned)blocks, 256, 0, st>>>(h_init, sums, A, h_local, h_out, batch, dim,
                                                         dstate, count);
    return cudaGetLastError();
}

}  // namespace mscan
