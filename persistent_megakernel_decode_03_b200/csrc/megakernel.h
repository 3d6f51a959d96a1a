// Launch interface of the persistent decode megakernel.
#pragma once

#include <cuda_runtime.h>

#include "mk_internal.h"

namespace mk {

size_t megakernel_smem_bytes();
// One launch of `grid` CTAs (one per SM) on `stream`: cooperative (the CTAs of a
// step wait on one another), or plain for a task list without waits inside the
// launch (one phase of the kernel-per-op baseline).
cudaError_t megakernel_launch(const Params& p, int grid, cudaStream_t stream, bool cooperative = true);
// Tensor parallelism emulated on one GPU: L.n ranks' steps in one cooperative launch
// of `grid` CTAs (a multiple of L.n; each rank's Params carry its cta0 and ncta).
// Head dimension 128 only.
cudaError_t megakernel_launch_tp_emulated(const TpLaunch& L, int grid, cudaStream_t stream);
bool megakernel_supports(int heads_per_group, int head_dim);
cudaError_t megakernel_occupancy(int heads_per_group, int head_dim, int* blocks_per_sm);

}  // namespace mk
