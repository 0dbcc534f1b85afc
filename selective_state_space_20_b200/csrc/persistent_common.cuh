// persistent_common.cuh -- pieces shared by the persistent scan kernels: the
// launch parameters, the two schedules (a ready queue of (channel group, time
// chunk) units, and a balanced static split of the sub-chunks over the
// workers), asynchronous global -> shared copies and acquire/release flags.
//
// Ready queue.  Unit u = j * n_groups + g is chunk j of channel group g.  All
// chunk-0 units are ready at launch and occupy the first n_groups pop slots
// implicitly.  Finishing chunk j < n_chunks - 1 of a group writes that
// group's carried state, then appends unit (j + 1, g) to the queue (slot =
// atomic counter, value released after the carry).  A pop at slot s >=
// n_groups waits for queue entry s - n_groups.  Every popped unit is already
// being run by a resident worker, so the entries a waiter needs are always
// produced: the scheme cannot deadlock, whatever the residency.  Waits are
// bounded all the same; a worker that gives up raises the error word, which
// makes every other waiter give up too.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.cuh"

namespace mscan {
namespace persist {

constexpr int kWarps = 4;                  // workers per block
constexpr int kNS = 16;                    // max states per channel (dstate <= 16)
constexpr unsigned kSpinLimit = 1u << 22;  // polls before a waiter gives up
constexpr unsigned kUnitDone = 0xffffffffu;
constexpr unsigned kUnitAbort = 0xfffffffeu;

struct Params {
    const void *u, *delta, *B, *C, *z;
    const float *A, *D, *delta_bias;
    void *out;
    float *last_state;
    const float *h0;       // initial state (batch, dim, dstate) or null (zeros)
    // fused conv1d prologue (lane-split kernel): u holds x; weights
    // right-aligned to 4 taps on load; u_out optional; batch strides of x, z
    const float *conv_w, *conv_b;
    int conv_k;
    void *u_out;
    int64_t u_bstride, z_bstride;
    int64_t dim, seqlen;
    int dstate;
    int softplus;
    int group_channels;    // channels per unit: 32 (one lane per channel) or 16 (lane pairs)
    int groups_per_batch;  // ceil(dim / group_channels)
    int n_groups;          // batch * groups_per_batch
    int n_chunks;          // chunks per group
    int chunk_len;         // timesteps per chunk
    unsigned *hdr;         // workspace: [pop counter, push counter, error, unused]
    unsigned *queue;       // ready-queue schedule: n_groups * (n_chunks - 1) entries
    unsigned *progress;    // balanced schedule: per group, sub-chunks whose carry is out
    int subs_per_chain;    // balanced schedule: sub-chunks per group (ceil(seqlen / TC))
    int stall_group;       // test hook: this group's pieces never publish their carry (-1: none)
    float *carry;          // workspace: n_groups * 32 lanes * states-per-lane floats
    // optional: the state entering every 32nd timestep, for the backward pass
    // ([batch * ckpt_gpb][ckpt_nsup][32 channels][16 states] fp32)
    float *ckpt;
    int ckpt_gpb, ckpt_nsup;
    // lane-split block-local kernel: u / delta / z / out as (batch, L, dim)
    // and B / C as (batch, L, N), all dense (else (batch, dim, L) / (batch, N, L))
    int channels_last;
    // lane-split kernel: the final state alone (no C, readout, gate or out)
    int state_only;
    // byte ranges of the pointer arguments, for the bounds-checked build
    MSCAN_EXTENTS(x_u, x_delta, x_z, x_B, x_C, x_A, x_D, x_bias, x_out, x_last, x_h0, x_conv_w, x_conv_b, x_u_out,
                  x_ckpt, x_carry)
};

__device__ __forceinline__ void cp16(void *smem, const void *gmem, bool pred) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(s), "l"(gmem), "r"(pred ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Next unit for this warp (call from all lanes; lane 0 talks to the queue).
// Returns kUnitDone when the queue is drained, kUnitAbort after a timeout.
// The trailing __syncwarp orders every lane's later carry loads after lane
// 0's acquire.
__device__ __forceinline__ unsigned pop_unit(const Params &p, int lane) {
    const int n_units = p.n_groups * p.n_chunks;
    unsigned unit = kUnitDone;
    if (lane == 0) {
        const unsigned s = atomicAdd(p.hdr + 0, 1u);
        if ((int)s < n_units) {
            if ((int)s < p.n_groups) {
                unit = s;  // chunk 0 of group s
            } else {
                const unsigned *slot = p.queue + (s - p.n_groups);
                unsigned v = 0, spins = 0, ns = 32;
                while ((v = ld_acquire(slot)) == 0u) {
                    if (++spins > kSpinLimit || ld_acquire(p.hdr + 2) != 0u) break;
                    __nanosleep(ns);
                    if (ns < 1024) ns <<= 1;
                }
                if (v == 0u) atomicOr(p.hdr + 2, 1u);
                unit = v == 0u ? kUnitAbort : v - 1u;
            }
        }
    }
    unit = __shfl_sync(0xffffffffu, unit, 0);
    __syncwarp();
    return unit;
}

// Publish the successor of a finished unit.  Every lane must have written
// its part of the carry before the call (the __syncwarp orders them before
// lane 0's fence and release).
__device__ __forceinline__ void push_unit(const Params &p, int lane, unsigned next_unit) {
    __syncwarp();
    if (lane == 0) {
        __threadfence();
        const unsigned slot = atomicAdd(p.hdr + 1, 1u);
        st_release(p.queue + slot, next_unit + 1u);
    }
}

// ------------------------------------------------------ balanced schedule
// The (group, sub-chunk) grid, flattened group-major into T = n_groups * S
// sub-chunks, is cut into one contiguous range per worker, w * T / P ..
// (w + 1) * T / P.  A range holds at most three kinds of piece: the start of
// the group where it ends (from sub-chunk 0), whole groups, and the rest of
// the group where it starts.  A worker runs them in that order.  Only the
// last kind depends on another worker -- the one before it, which cut that
// group and runs its part first -- so every wait points to a lower worker
// and is over almost as soon as it begins.  The carried state of a group
// passes through one workspace slot: its producer writes it, then publishes
// the sub-chunk position in progress[g]; the consumer waits until progress[g]
// reaches its first sub-chunk.  Pieces of one group run strictly one after
// the other, so the slot is never overwritten before it has been read.
//
// Block-local variant (no workspace): each block takes a contiguous range of
// whole groups and splits it the same way among its own warps; a carried
// state then only ever passes from warp w - 1 to warp w of one block, through
// one shared-memory slot per warp boundary (a warp publishes at most once:
// at the end of its range, if that falls inside a group).
struct Piece {
    int g;       // group
    int sb, se;  // sub-chunks [sb, se) of the group
};

// One worker's range, run in field order: head, whole groups, tail.
struct Range {
    Piece head;          // the group where the range ends, from sub-chunk 0 (se == 0: none)
    int full_b, full_e;  // whole groups [full_b, full_e)
    Piece tail;          // the group where the range starts (se == 0: none); its
                         // sb > 0 means it continues another worker's piece
};

// Worker w of P over groups [g0, g0 + n_groups) of S sub-chunks each.
__device__ __forceinline__ Range worker_range_of(long long n_groups, long long S, int g0, long long w,
                                                 long long P) {
    const long long T = n_groups * S;
    const long long s = w * T / P, e = (w + 1) * T / P;
    Range r;
    r.head = Piece{0, 0, 0};
    r.tail = Piece{0, 0, 0};
    r.full_b = r.full_e = 0;
    if (s >= e) return r;
    const int cs = g0 + (int)(s / S), os = (int)(s % S);
    const int ce = g0 + (int)(e / S), oe = (int)(e % S);
    if (cs == ce) {  // inside one group
        r.tail = Piece{cs, os, oe};
        return r;
    }
    if (oe > 0) r.head = Piece{ce, 0, oe};
    r.full_b = os > 0 ? cs + 1 : cs;
    r.full_e = ce;
    if (os > 0) r.tail = Piece{cs, os, (int)S};
    return r;
}

// Worker w of P over every group of the launch.
__device__ __forceinline__ Range worker_range(const Params &p, long long w, long long P) {
    return worker_range_of(p.n_groups, p.subs_per_chain, 0, w, P);
}

// Wait (lane 0 polls, bounded in time) until group g's carry covers sub-chunk
// position `pos`; false after a timeout or when another worker gave up.
__device__ __forceinline__ bool wait_progress(const Params &p, int lane, int g, int pos) {
    unsigned ok = 1;
    if (lane == 0) {
        const unsigned *f = p.progress + g;
        if (ld_acquire(f) < (unsigned)pos) {
            unsigned long long t0, t;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
            unsigned ns = 32;
            while (ld_acquire(f) < (unsigned)pos) {
                asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
                if (ld_acquire(p.hdr + 2) != 0u || t - t0 > 2000000000ull) {
                    atomicOr(p.hdr + 2, 1u);
                    ok = 0;
                    break;
                }
                __nanosleep(ns);
                if (ns < 1024) ns <<= 1;
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();  // every lane's carry loads come after lane 0's acquire
    return ok != 0;
}

// Publish that group g's carry now covers sub-chunk position `pos`.  Every
// lane must have written its part of the carry before the call.
__device__ __forceinline__ void publish_progress(const Params &p, int lane, int g, int pos) {
    __syncwarp();
    if (lane == 0) {
        __threadfence();
        st_release(p.progress + g, (unsigned)pos);
    }
}

}  // namespace persist
}  // namespace mscan
