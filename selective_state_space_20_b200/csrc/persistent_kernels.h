// persistent_kernels.h -- launchers of the two persistent scan kernels
// (internal; planning and workspace layout live in persistent_host.cu).
#pragma once

#include <cuda_runtime.h>

#include "persistent_common.cuh"

namespace mscan {

// One lane per channel, all states in one thread; units of 32 channels; each
// scan warp paired with a helper warp (blocks of four pairs, one per SM).
int persistent_spec_sub_chunk();
int persistent_spec_pairs_per_sm();
cudaError_t launch_persistent_spec(const persist::Params &kp, int act, int grid, cudaStream_t st);

// R = 2 or 4 lanes per channel, 16 / R states each; groups of 32 / R
// channels; the balanced split over every worker that fits on the device
// (launched cooperatively, all resident).
int persistent_split_sub_chunk(int lanes, int act);
int persistent_split_blocks_per_sm(int lanes);
cudaError_t launch_persistent_split(const persist::Params &kp, int lanes, int act, int sm_count,
                                   cudaStream_t st);

// The same kernel in its block-local form: one block per SM (LocalWarps
// warps) splits whole channel groups among its warps; carries in shared
// memory, no workspace.  take_local_error reads and clears the device word a
// block-local launch sets when a bounded wait ran out.
int local_split_warps(int lanes);
cudaError_t launch_local_split(const persist::Params &kp, int lanes, int act, int sm_count, cudaStream_t st);
int take_local_error(unsigned *flag);

}  // namespace mscan
