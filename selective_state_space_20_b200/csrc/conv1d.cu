// conv1d.cu -- causal depthwise convolution over time, plus bias and silu:
// the step that turns the x half of the input projection into the scan's
// input u ("Mamba SSM concept and implementation in Keras and TensorFlow",
// MambaBlock: a Conv1D with one group per channel, channels-first, causal
// padding and a bias, cut to the input length, then swish):
//   v[b,d,t]   = bias[d] + sum_{k<K} w[d,k] * x[b,d,t-(K-1)+k],  x = 0 for t < 0
//   out[b,d,t] = silu(v) if requested, else v
// and its one-token form for decoding, which keeps each row's last K-1
// inputs as a state.
//
// The sequence kernel is a pure stream: 2 (bf16) or 4 (fp32) bytes read and
// written per element, so it is bound by HBM.  A warp covers four tiles of
// 32 consecutive 16-byte chunks of one row (1024 bf16 / 512 fp32 timesteps)
// with one load and one store per lane and tile; the K-1 inputs before a
// lane's chunk come from the lane before it by shuffle (at the span's start
// lane 0 reads them from memory), so every input byte is read once.  Rows that are not 16-byte aligned or whose length is not a
// whole number of chunks take a one-thread-per-output kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "bounds.cuh"
#include "device_math.cuh"
#include "internal.h"

namespace mscan {
namespace {

struct ConvParams {
    const void *x;
    const float *w, *bias;
    void *out;
    int64_t batch, dim, seqlen, x_batch_stride;
    int width, silu;
    MSCAN_EXTENTS(x_x, x_w, x_bias, x_out)  // byte ranges, for the bounds-checked build
};

template <typename T>
__device__ __forceinline__ float load_elem(const T *p) { return Elem<T>::load(p); }

// Loads and stores that the bounds-checked build tests against the tensor's
// range (a load outside reads zero, a store outside is dropped).
#ifdef MSCAN_BOUNDS_CHECK
template <typename T>
__device__ __forceinline__ float load_chk(const Extent &e, const T *q, int site) {
    return MSCAN_WITHIN(e, q, sizeof(T), site) ? Elem<T>::load(q) : 0.f;
}
__device__ __forceinline__ float ldg_chk(const Extent &e, const float *q, int site) {
    return MSCAN_WITHIN(e, q, 4, site) ? __ldg(q) : 0.f;
}
#else
#define load_chk(e, q, site) load_elem(q)
#define ldg_chk(e, q, site) __ldg(q)
#endif

// One warp per NT consecutive 32-chunk tiles of one row: every lane issues
// its NT 16-byte loads first (NT x 512 bytes in flight per warp), then the
// tiles are finished in order, each taking the inputs before a lane's chunk
// from the lane before it, and lane 0 from lane 31 of the previous tile.
// W64: 64-bit index arithmetic (more than 2^31 threads); otherwise 32-bit,
// whose divisions cost a fraction of the 64-bit ones.
template <typename T, int K, int NT, bool W64, bool SILU>
__global__ void __launch_bounds__(256) conv1d_tiles_kernel(const ConvParams p) {
    using Idx = typename std::conditional<W64, int64_t, unsigned>::type;
    constexpr int V = 16 / (int)sizeof(T);  // elements per 16-byte chunk
    constexpr int TILE = 32 * V;
    const int lane = threadIdx.x & 31;
    const Idx warp = ((Idx)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const Idx spans_per_row = ((Idx)p.seqlen + NT * TILE - 1) / (NT * TILE);
    const Idx row = warp / spans_per_row;
    if (row >= (Idx)(p.batch * p.dim)) return;  // whole warp leaves together
    const Idx b = row / (Idx)p.dim, d = row - b * (Idx)p.dim;
    const int64_t span0 = (int64_t)(warp - row * spans_per_row) * (NT * TILE);
    const T *xr = static_cast<const T *>(p.x) + (int64_t)b * p.x_batch_stride + (int64_t)d * p.seqlen;
    T *orow = static_cast<T *>(p.out) + (int64_t)row * p.seqlen;

    uint4 raw[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int64_t t0 = span0 + j * TILE + (int64_t)lane * V;
        raw[j] = (t0 < p.seqlen && MSCAN_WITHIN(p.x_x, xr + t0, 16, kSiteX)) ? ldg16_stream(xr + t0)
                                                                     : make_uint4(0u, 0u, 0u, 0u);
    }
    float carry[K];  // lane 0: the K-1 inputs before the span
#pragma unroll
    for (int k = 0; k < K - 1; ++k) {
        const int64_t s = span0 - (K - 1) + k;
        carry[k] = (lane == 0 && s >= 0) ? load_chk(p.x_x, xr + s, kSiteX) : 0.f;
    }
    float wk[K];
#pragma unroll
    for (int k = 0; k < K; ++k) wk[k] = ldg_chk(p.x_w, p.w + (int64_t)d * K + k, kSiteConvW);
    const float bias = p.bias ? ldg_chk(p.x_bias, p.bias + d, kSiteConvB) : 0.f;

#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int64_t t0 = span0 + j * TILE + (int64_t)lane * V;
        float f[V + K - 1];  // K-1 earlier inputs, then this chunk
        Elem<T>::unpack(raw[j], f + K - 1);
#pragma unroll
        for (int k = 0; k < K - 1; ++k) {
            const float prev = __shfl_up_sync(0xffffffffu, f[V + k], 1);
            const float last = __shfl_sync(0xffffffffu, f[V + k], 31);  // for the next tile
            f[k] = lane > 0 ? prev : carry[k];
            carry[k] = last;
        }
        if (t0 < p.seqlen) {  // seqlen is a whole number of chunks
            float o[V];
#pragma unroll
            for (int i = 0; i < V; i += 2) {  // output pairs on the packed x2 instructions
                float2 v = f2(bias, bias);
#pragma unroll
                for (int k = 0; k < K; ++k) v = __ffma2_rn(f2(wk[k], wk[k]), f2(f[i + k], f[i + 1 + k]), v);
                if (SILU) v = silu2_f(v);
                o[i] = v.x;
                o[i + 1] = v.y;
            }
            if (MSCAN_WITHIN(p.x_out, orow + t0, 16, kSiteOut)) stg16_stream(orow + t0, Elem<T>::pack(o));
        }
    }
}

// Any alignment and length: one thread per output.
template <typename T>
__global__ void __launch_bounds__(256) conv1d_scalar_kernel(const ConvParams p) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= p.batch * p.dim * p.seqlen) return;
    const int64_t t = i % p.seqlen, row = i / p.seqlen;
    const int64_t b = row / p.dim, d = row % p.dim;
    const T *xr = static_cast<const T *>(p.x) + b * p.x_batch_stride + d * p.seqlen;
    float v = p.bias ? ldg_chk(p.x_bias, p.bias + d, kSiteConvB) : 0.f;
    for (int k = 0; k < p.width; ++k) {
        const int64_t s = t - (p.width - 1) + k;
        if (s >= 0) v = fmaf(ldg_chk(p.x_w, p.w + d * p.width + k, kSiteConvW), load_chk(p.x_x, xr + s, kSiteX), v);
    }
    T *o = static_cast<T *>(p.out) + i;
    if (MSCAN_WITHIN(p.x_out, o, sizeof(T), kSiteOut)) Elem<T>::store(o, p.silu ? silu_f(v) : v);
}

struct ConvUpdateParams {
    float *state;
    const void *x;
    const float *w, *bias;
    void *out;
    int64_t batch, dim, x_batch_stride;
    int width, silu;
    MSCAN_EXTENTS(x_state, x_x, x_w, x_bias, x_out)  // byte ranges, for the bounds-checked build
};

// One thread per (batch, channel): read the K-1 kept inputs and the token,
// emit the output, shift the kept inputs.
template <typename T, int K>
__global__ void __launch_bounds__(256) conv1d_update_kernel(const ConvUpdateParams p) {
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= p.batch * p.dim) return;
    const int64_t b = row / p.dim, d = row % p.dim;
    constexpr int S = K - 1;
    float *st = p.state + row * S;
    float in[K];
#pragma unroll
    for (int k = 0; k < S; ++k) in[k] = MSCAN_WITHIN(p.x_state, st + k, 4, kSiteConvState) ? st[k] : 0.f;
    in[S] = load_chk(p.x_x, static_cast<const T *>(p.x) + b * p.x_batch_stride + d, kSiteX);
    float v = p.bias ? ldg_chk(p.x_bias, p.bias + d, kSiteConvB) : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) v = fmaf(ldg_chk(p.x_w, p.w + d * K + k, kSiteConvW), in[k], v);
    T *o = static_cast<T *>(p.out) + row;
    if (MSCAN_WITHIN(p.x_out, o, sizeof(T), kSiteOut)) Elem<T>::store(o, p.silu ? silu_f(v) : v);
#pragma unroll
    for (int k = 0; k < S; ++k)
        if (MSCAN_WITHIN(p.x_state, st + k, 4, kSiteConvState)) st[k] = in[k + 1];
}

template <typename T, int NT, bool SILU>
cudaError_t launch_tiles(const ConvParams &p, bool w64, unsigned g, int threads, cudaStream_t st) {
    switch (p.width * 2 + (w64 ? 1 : 0)) {
        case 2: conv1d_tiles_kernel<T, 1, NT, false, SILU><<<g, threads, 0, st>>>(p); break;
        case 3: conv1d_tiles_kernel<T, 1, NT, true, SILU><<<g, threads, 0, st>>>(p); break;
        case 4: conv1d_tiles_kernel<T, 2, NT, false, SILU><<<g, threads, 0, st>>>(p); break;
        case 5: conv1d_tiles_kernel<T, 2, NT, true, SILU><<<g, threads, 0, st>>>(p); break;
        case 6: conv1d_tiles_kernel<T, 3, NT, false, SILU><<<g, threads, 0, st>>>(p); break;
        case 7: conv1d_tiles_kernel<T, 3, NT, true, SILU><<<g, threads, 0, st>>>(p); break;
        case 9: conv1d_tiles_kernel<T, 4, NT, true, SILU><<<g, threads, 0, st>>>(p); break;
        default: conv1d_tiles_kernel<T, 4, NT, false, SILU><<<g, threads, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fwd_typed(const ConvParams &p, cudaStream_t st) {
    constexpr int V = 16 / (int)sizeof(T);
    const auto aligned = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    const bool tiles = aligned(p.x) && aligned(p.out) && p.seqlen % V == 0 && p.x_batch_stride % V == 0;
    const int threads = 256;
    if (tiles) {
        constexpr int TILE = 32 * V, NT = 4;  // 2: -10 %, 8: same (B200, bf16 4 x 5120 x 4096)
        const int64_t warps = p.batch * p.dim * ((p.seqlen + NT * TILE - 1) / (NT * TILE));
        const int64_t blocks = (warps * 32 + threads - 1) / threads;
        if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
        const bool w64 = blocks * threads >= 0x7fffffffLL || p.seqlen >= 0x7fffffffLL;
        return p.silu ? launch_tiles<T, NT, true>(p, w64, (unsigned)blocks, threads, st)
                      : launch_tiles<T, NT, false>(p, w64, (unsigned)blocks, threads, st);
    }
    const int64_t blocks = (p.batch * p.dim * p.seqlen + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    conv1d_scalar_kernel<T><<<(unsigned)blocks, threads, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_update_typed(const ConvUpdateParams &p, unsigned blocks, cudaStream_t st) {
    switch (p.width) {
        case 1: conv1d_update_kernel<T, 1><<<blocks, 256, 0, st>>>(p); break;
        case 2: conv1d_update_kernel<T, 2><<<blocks, 256, 0, st>>>(p); break;
        case 3: conv1d_update_kernel<T, 3><<<blocks, 256, 0, st>>>(p); break;
        default: conv1d_update_kernel<T, 4><<<blocks, 256, 0, st>>>(p); break;
    }
    return cudaGetLastError();
}

}  // namespace

MSCAN_BOUNDS_TAKE(conv1d_bounds_take)

cudaError_t launch_conv1d_fwd(const Conv1dArgs &a, cudaStream_t st) {
    ConvParams p;
    p.x = a.x; p.w = a.weight; p.bias = a.bias; p.out = a.out;
    p.batch = a.batch; p.dim = a.dim; p.seqlen = a.seqlen; p.x_batch_stride = a.x_batch_stride;
    p.width = a.width; p.silu = a.silu;
#ifdef MSCAN_BOUNDS_CHECK
    const unsigned long long es = a.act == kBF16 ? 2 : 4;
    const unsigned long long row = (unsigned long long)(a.dim * a.seqlen) * es;
    const unsigned long long ob = (unsigned long long)a.batch * row;
    p.x_x = extent_of(a.x, (unsigned long long)(a.batch - 1) * a.x_batch_stride * es + row);
    p.x_w = extent_of(a.weight, (unsigned long long)(a.dim * a.width) * 4);
    p.x_bias = extent_of(a.bias, (unsigned long long)a.dim * 4);
    p.x_out = extent_of(a.out, ob > (unsigned long long)g_out_extent_shrink ? ob - g_out_extent_shrink : 0);
#endif
    return a.act == kBF16 ? launch_fwd_typed<__nv_bfloat16>(p, st) : launch_fwd_typed<float>(p, st);
}

cudaError_t launch_conv1d_update(const Conv1dUpdateArgs &a, cudaStream_t st) {
    ConvUpdateParams p;
    p.state = a.state; p.x = a.x; p.w = a.weight; p.bias = a.bias; p.out = a.out;
    p.batch = a.batch; p.dim = a.dim; p.x_batch_stride = a.x_batch_stride;
    p.width = a.width; p.silu = a.silu;
#ifdef MSCAN_BOUNDS_CHECK
    const unsigned long long es = a.act == kBF16 ? 2 : 4, rows = (unsigned long long)(a.batch * a.dim);
    p.x_state = extent_of(a.state, rows * (a.width - 1) * 4);
    p.x_x = extent_of(a.x, (unsigned long long)(a.batch - 1) * a.x_batch_stride * es + (unsigned long long)a.dim * es);
    p.x_w = extent_of(a.weight, (unsigned long long)(a.dim * a.width) * 4);
    p.x_bias = extent_of(a.bias, (unsigned long long)a.dim * 4);
    p.x_out = extent_of(a.out, rows * es > (unsigned long long)g_out_extent_shrink ? rows * es - g_out_extent_shrink : 0);
#endif
    const int threads = 256;
    const int64_t blocks = (a.batch * a.dim + threads - 1) / threads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return a.act == kBF16 ? launch_update_typed<__nv_bfloat16>(p, (unsigned)blocks, st)
                          : launch_update_typed<float>(p, (unsigned)blocks, st);
}

}  // namespace mscan
