// scan_fwd_noalloc.cu -- mamba_scan_fwd_noalloc: the workspace-backed scan
// for callers that cannot hand the library any device memory of their own.
//
// The persistent schedule of mamba_scan_fwd_ws needs a device workspace (its
// work queue and the states carried between time chunks).  Here that
// workspace is a fixed array compiled into the library instead of caller
// memory, so the call itself allocates nothing.
//
// * The array lives in this file as a static __device__ variable.  Every GPU
//   that loads the library reserves it (kScratchBytes) until the process
//   exits.  Problems whose workspace would exceed it are rejected with
//   MAMBA_ERR_WORKSPACE before anything is enqueued.
// * A __device__ variable's name in host code is only a host-side stand-in,
//   not a device address.  The device address is looked up with
//   cudaGetSymbolAddress, once per device, with that device current, the
//   first time the entry point runs on it, and cached for later calls.
// * Every call shares the array.  mamba_scan_fwd_ws zeroes the part that
//   must start at zero (queue counters and slots) on the caller's stream
//   before each launch; calls whose work overlaps on the GPU (different
//   streams, or different host threads) race on the array and must not run
//   concurrently.
#include <cuda_runtime.h>

#include <mutex>

#include "mamba_scan.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scan_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices];  // device address of g_scan_scratch, per device

// Device address of the scratch array on the current device (set-up on the
// first call per device).
int scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MAMBA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scan_scratch);
        if (e != cudaSuccess || p == nullptr) return MAMBA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MAMBA_OK;
}

}  // namespace

extern "C" int mamba_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                                      const void *B, const void *C, const float *D,
                                      const void *z, const float *delta_bias,
                                      int delta_softplus, void *out, float *last_state,
                                      int64_t batch, int64_t dim, int64_t seqlen,
                                      int64_t dstate, int act_dtype, cudaStream_t stream) {
    // Size check first: pure host arithmetic, nothing touched on rejection.
    const size_t need = mamba_scan_workspace_size(batch, dim, seqlen, dstate, act_dtype);
    if (need > kScratchBytes) return MAMBA_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != MAMBA_OK) return rc;
    return mamba_scan_fwd_ws(u, delta, A, B, C, D, z, delta_bias, delta_softplus, out,
                             last_state, batch, dim, seqlen, dstate, act_dtype, nullptr,
                             scratch, kScratchBytes, stream);
}
