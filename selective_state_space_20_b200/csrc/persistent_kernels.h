// persistent_kernels.h -- launchers of the two persistent scan kernels
// (internal; planning and workspace layout live in persistent_host.cu).
#pragma once

#include <cuda_runtime.h>

#include "persistent_common.cuh"

namespace mscan {

// One lane per channel, all states in one thread; units of 32 channels.
int persistent_lanes1_sub_chunk(int act);
int persistent_lanes1_blocks_per_sm();
cudaError_t launch_persistent_lanes1(const persist::Params &kp, int act, int grid, cudaStream_t st);

// Two lanes per channel, half of the states each; units of 16 channels.
int persistent_lanes2_sub_chunk(int act);
int persistent_lanes2_blocks_per_sm();
cudaError_t launch_persistent_lanes2(const persist::Params &kp, int act, int grid, cudaStream_t st);

}  // namespace mscan
