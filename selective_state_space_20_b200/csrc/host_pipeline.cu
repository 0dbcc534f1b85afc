// host_pipeline.cu -- the scan on sequences that live in host memory: the
// (batch, channel) rows are cut into chunks, and for each chunk the inputs go
// host -> device on one stream, the scan runs on the caller's stream and the
// outputs go device -> host on a third, chunk by chunk through two device
// slots, so the two copy directions and the scan overlap.  Each chunk is a
// channel range of one batch row: its u / delta / z / out rows are one
// contiguous block of the host arrays, and it takes that batch row's B and C.
// The scan of a chunk is mamba_scan_fwd_init / mamba_scan_fwd_ws on the
// slot's device buffers.
#include <cuda_runtime.h>
#include <stdint.h>

#include "mamba_scan.h"

namespace {

constexpr int kTargetChunks = 16;  // chunks per call (the pipeline's depth)

size_t align16(size_t n) { return (n + 15) & ~(size_t)15; }

struct Plan {
    int64_t pieces;   // chunks per batch row
    int64_t cc;       // channels per chunk (the last of a row may hold fewer)
    size_t x_bytes;   // one (cc, L) activation block
    size_t bc_bytes;  // one (N, L) B or C row
    size_t slot;      // u, delta, z, out, B, C of one chunk
    size_t ls_bytes;  // last_state for the whole problem
    size_t ws_bytes;  // the scan's workspace for one chunk
    size_t total;
};

Plan make_plan(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act) {
    Plan p;
    const size_t es = act == MAMBA_BF16 ? 2 : 4;
    p.pieces = (kTargetChunks + batch - 1) / batch;
    if (p.pieces > dim) p.pieces = dim;
    if (p.pieces < 1) p.pieces = 1;
    p.cc = (dim + p.pieces - 1) / p.pieces;
    p.x_bytes = align16((size_t)(p.cc * seqlen) * es);
    p.bc_bytes = align16((size_t)(dstate * seqlen) * es);
    p.slot = 4 * p.x_bytes + 2 * p.bc_bytes;
    p.ls_bytes = align16((size_t)(batch * dim * dstate) * 4);
    p.ws_bytes = align16(mamba_scan_workspace_size(1, p.cc, seqlen, dstate, act));
    p.total = 2 * p.slot + p.ls_bytes + p.ws_bytes;
    return p;
}

}  // namespace

extern "C" {

size_t mamba_scan_host_scratch_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                                    int act_dtype) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return 0;
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0 || dstate > 64) return 0;
    if ((double)batch * (double)dim * (double)seqlen > (double)((int64_t)1 << 50)) return 0;
    return make_plan(batch, dim, seqlen, dstate, act_dtype).total;
}

int mamba_scan_fwd_host(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *delta_bias,
                        int delta_softplus, const float *h0, void *out, float *last_state,
                        int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int act_dtype,
                        void *scratch, size_t scratch_bytes, cudaStream_t stream) {
    if (act_dtype != MAMBA_F32 && act_dtype != MAMBA_BF16) return MAMBA_ERR_UNSUPPORTED;
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0) return MAMBA_ERR_SHAPE;
    if (dstate > 64) return MAMBA_ERR_UNSUPPORTED;
    if (!u || !delta || !A || !B || !C || !out) return MAMBA_ERR_NULL;
    const size_t need = mamba_scan_host_scratch_size(batch, dim, seqlen, dstate, act_dtype);
    if (need == 0) return MAMBA_ERR_SHAPE;
    if (!scratch || scratch_bytes < need || (reinterpret_cast<uintptr_t>(scratch) & 15) != 0)
        return MAMBA_ERR_WORKSPACE;
    const Plan pl = make_plan(batch, dim, seqlen, dstate, act_dtype);
    const size_t es = act_dtype == MAMBA_BF16 ? 2 : 4;
    unsigned char *base = static_cast<unsigned char *>(scratch);
    float *ls_dev = reinterpret_cast<float *>(base + 2 * pl.slot);
    void *ws = pl.ws_bytes ? base + 2 * pl.slot + pl.ls_bytes : nullptr;

    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[7] = {};  // start, in_ready[2], computed[2], slot_free[2]
    int rc = MAMBA_OK;
    auto cu = [&](cudaError_t e) {
        if (e != cudaSuccess && rc == MAMBA_OK) rc = MAMBA_ERR_CUDA;
        return e == cudaSuccess;
    };
    bool ok = cu(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking)) &&
              cu(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking));
    for (int i = 0; ok && i < 7; ++i) ok = cu(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming));
    cudaEvent_t start = ev[0], *in_ready = ev + 1, *computed = ev + 3, *slot_free = ev + 5;
    // both copy streams start after the work already queued on the caller's stream
    if (ok) ok = cu(cudaEventRecord(start, stream)) && cu(cudaStreamWaitEvent(s_in, start, 0)) &&
                 cu(cudaStreamWaitEvent(s_out, start, 0));

    const int64_t chunks = batch * pl.pieces;
    for (int64_t k = 0; ok && k < chunks; ++k) {
        const int s = (int)(k & 1);
        const int64_t b = k / pl.pieces, d0 = (k % pl.pieces) * pl.cc;
        if (d0 >= dim) continue;
        const int64_t nd = (dim - d0) < pl.cc ? dim - d0 : pl.cc;
        const size_t xb = (size_t)(nd * seqlen) * es, bcb = (size_t)(dstate * seqlen) * es;
        const size_t row = (size_t)((b * dim + d0) * seqlen) * es;
        unsigned char *slot = base + (size_t)s * pl.slot;
        void *du = slot, *dd = slot + pl.x_bytes, *dz = slot + 2 * pl.x_bytes, *dout = slot + 3 * pl.x_bytes;
        void *dB = slot + 4 * pl.x_bytes, *dC = slot + 4 * pl.x_bytes + pl.bc_bytes;
        // inputs (after the outputs of the chunk that last used this slot left)
        if (k >= 2) ok = cu(cudaStreamWaitEvent(s_in, slot_free[s], 0));
        ok = ok && cu(cudaMemcpyAsync(du, static_cast<const unsigned char *>(u) + row, xb, cudaMemcpyHostToDevice, s_in));
        ok = ok && cu(cudaMemcpyAsync(dd, static_cast<const unsigned char *>(delta) + row, xb, cudaMemcpyHostToDevice, s_in));
        if (z) ok = ok && cu(cudaMemcpyAsync(dz, static_cast<const unsigned char *>(z) + row, xb, cudaMemcpyHostToDevice, s_in));
        ok = ok && cu(cudaMemcpyAsync(dB, static_cast<const unsigned char *>(B) + (size_t)b * bcb, bcb,
                                      cudaMemcpyHostToDevice, s_in));
        ok = ok && cu(cudaMemcpyAsync(dC, static_cast<const unsigned char *>(C) + (size_t)b * bcb, bcb,
                                      cudaMemcpyHostToDevice, s_in));
        ok = ok && cu(cudaEventRecord(in_ready[s], s_in));
        // the scan of the chunk, on the caller's stream
        ok = ok && cu(cudaStreamWaitEvent(stream, in_ready[s], 0));
        if (ok) {
            const int64_t st = (b * dim + d0) * dstate;
            const int r = h0 ? mamba_scan_fwd_init(du, dd, A + d0 * dstate, dB, dC, D ? D + d0 : nullptr,
                                                   z ? dz : nullptr, delta_bias ? delta_bias + d0 : nullptr,
                                                   delta_softplus, h0 + st, dout, ls_dev + st, 1, nd, seqlen,
                                                   dstate, act_dtype, nullptr, ws, pl.ws_bytes, stream)
                             : mamba_scan_fwd_ws(du, dd, A + d0 * dstate, dB, dC, D ? D + d0 : nullptr,
                                                 z ? dz : nullptr, delta_bias ? delta_bias + d0 : nullptr,
                                                 delta_softplus, dout, ls_dev + st, 1, nd, seqlen, dstate,
                                                 act_dtype, nullptr, ws, pl.ws_bytes, stream);
            if (r != MAMBA_OK) {
                rc = r;
                ok = false;
            }
        }
        ok = ok && cu(cudaEventRecord(computed[s], stream));
        // outputs
        ok = ok && cu(cudaStreamWaitEvent(s_out, computed[s], 0));
        ok = ok && cu(cudaMemcpyAsync(static_cast<unsigned char *>(out) + row, dout, xb, cudaMemcpyDeviceToHost, s_out));
        ok = ok && cu(cudaEventRecord(slot_free[s], s_out));
    }
    if (ok && last_state)
        ok = cu(cudaMemcpyAsync(last_state, ls_dev, (size_t)(batch * dim * dstate) * 4, cudaMemcpyDeviceToHost, s_out));
    // the caller's stream continues after everything this call enqueued --
    // also after an error, so that synchronising it still covers every copy
    if (s_in && s_out && ev[0] && ev[1]) {
        cu(cudaEventRecord(ev[0], s_out));
        cu(cudaStreamWaitEvent(stream, ev[0], 0));
        cu(cudaEventRecord(ev[1], s_in));
        cu(cudaStreamWaitEvent(stream, ev[1], 0));
    }
    for (int i = 0; i < 7; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    return rc;
}

}  // extern "C"
