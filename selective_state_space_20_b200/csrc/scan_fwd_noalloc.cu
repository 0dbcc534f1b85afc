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
//   not a device address.  Every call looks the device address up with
//   cudaGetSymbolAddress on the current device and context (cheap once the
//   module is loaded), so a reset device or another context on the same
//   device never sees a stale address.  With lazily loaded modules (the
//   CUDA default) the first lookup on a device loads the module and thereby
//   reserves the array; that first call may fail with MAMBA_ERR_CUDA when
//   device memory is short, and it should come before any stream capture.
// * Every call shares the array.  mamba_scan_fwd_ws zeroes the part that
//   must start at zero (header and progress words) on the caller's stream
//   before each launch; calls whose work overlaps on the GPU (different
//   streams, or different host threads) race on the array and must not run
//   concurrently.
#include <cuda_runtime.h>

#include "mamba_scan.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB per device

__device__ __align__(256) unsigned char g_scan_scratch[kScratchBytes];

// Device address of the scratch array in the current context.
int scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MAMBA_ERR_DEVICE;
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scan_scratch);
    if (e != cudaSuccess || p == nullptr) return MAMBA_ERR_CUDA;
    *addr = p;
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
