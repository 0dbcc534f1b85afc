// bounds.cuh -- the bounds-checked build of the kernels (MSCAN_BOUNDS_CHECK).
//
// Every kernel launch carries, for each pointer argument, the byte range it
// may touch (an Extent, filled on the host from the sizes the caller passed).
// In the checked build each global access of the scan kernels (lane-split,
// one-lane, static, complex), the backward, the decode step and the conv1d
// kernels first asks MSCAN_WITHIN(): an access that would leave its range is
// skipped -- a load reads zeros, a store
// is dropped -- and the first such access of the launch is recorded (site and
// byte offset) in a word of its translation unit, which the host reads
// through mamba_get_device_status / mamba_debug_bounds_status.  Nothing traps
// or faults.  In the normal build MSCAN_WITHIN() is the constant true, its
// arguments are not compiled, and the launch parameters carry no ranges
// (MSCAN_EXTENTS declares them in the checked build only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mscan {

struct Extent {
    const void *base;
    unsigned long long bytes;  // 0: nothing may be touched
};

__host__ __device__ inline Extent extent_of(const void *p, unsigned long long bytes) {
    Extent e;
    e.base = p;
    e.bytes = p ? bytes : 0ull;
    return e;
}

// Access sites, reported with a violation.
enum BoundsSite : int {
    kSiteA = 1, kSiteBias, kSiteD, kSiteConvW, kSiteConvB, kSiteU, kSiteDelta, kSiteZ, kSiteB, kSiteC,
    kSiteHalo, kSiteUOut, kSiteOut, kSiteLastState, kSiteH0, kSiteCkpt, kSiteCarry, kSiteState, kSiteX,
    kSiteConvState
};

#ifdef MSCAN_BOUNDS_CHECK
constexpr bool kBoundsChecked = true;
namespace {
__device__ unsigned g_bounds_hit;  // one set per translation unit (its own module)
__device__ int g_bounds_site;
__device__ long long g_bounds_off;
}  // namespace

__device__ __forceinline__ bool within(const Extent &e, const void *p, unsigned n, int site) {
    const long long off = (long long)(static_cast<const char *>(p) - static_cast<const char *>(e.base));
    if (off >= 0 && (unsigned long long)off + n <= e.bytes) return true;
    if (atomicCAS(&g_bounds_hit, 0u, 1u) == 0u) {
        g_bounds_site = site;
        g_bounds_off = off;
    }
    return false;
}

#define MSCAN_WITHIN(e, q, n, site) ::mscan::within((e), (q), (n), (site))
#define MSCAN_EXTENTS(...) Extent __VA_ARGS__;

// Host: this translation unit's record (1 = a violation, with its site and
// offset), cleared; -1 when the words cannot be read.
#define MSCAN_BOUNDS_TAKE(fn)                                                                     \
    int fn(int *site, long long *off) {                                                           \
        unsigned hit = 0, zero = 0;                                                               \
        if (cudaMemcpyFromSymbol(&hit, g_bounds_hit, sizeof(hit)) != cudaSuccess) return -1;      \
        if (hit == 0) return 0;                                                                   \
        if (cudaMemcpyFromSymbol(site, g_bounds_site, sizeof(int)) != cudaSuccess ||              \
            cudaMemcpyFromSymbol(off, g_bounds_off, sizeof(long long)) != cudaSuccess ||          \
            cudaMemcpyToSymbol(g_bounds_hit, &zero, sizeof(zero)) != cudaSuccess)                 \
            return -1;                                                                            \
        return 1;                                                                                 \
    }
#else
// The normal build: no ranges in the launch parameters (their layout, and so
// the kernels' register allocation, stays exactly as without the checks) and
// no checks -- the macro arguments are not even compiled.
constexpr bool kBoundsChecked = false;
#define MSCAN_WITHIN(e, q, n, site) true
#define MSCAN_EXTENTS(...)
#define MSCAN_BOUNDS_TAKE(fn) \
    int fn(int *, long long *) { return 0; }
#endif

}  // namespace mscan
