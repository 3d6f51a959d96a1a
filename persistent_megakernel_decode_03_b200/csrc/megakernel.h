// Launch interface of the persistent decode megakernel.
#pragma once

#include <cuda_runtime.h>

#include "mk_internal.h"

namespace mk {

size_t megakernel_smem_bytes();
// One cooperative launch of `grid` CTAs (one per SM) on `stream`.
cudaError_t megakernel_launch(const Params& p, int grid, cudaStream_t stream);
bool megakernel_supports(int heads_per_group, int head_dim);
cudaError_t megakernel_occupancy(int heads_per_group, int head_dim, int* blocks_per_sm);

}  // namespace mk
