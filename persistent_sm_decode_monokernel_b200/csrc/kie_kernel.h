// Launch entry points of the persistent decode kernel (kie_kernel.cu).
#pragma once

#include <cuda_runtime.h>

#include "kie_params.h"

namespace kie {

// Sets the dynamic shared-memory limit of the kernel instance for head
// dimension `hd` (64 or 128) and reports how many CTAs fit on one SM.
cudaError_t mono_configure(int hd, int smem_bytes, int* blocks_per_sm);

// Cooperative launch (all CTAs co-resident) of `grid` persistent CTAs.
cudaError_t mono_launch(const MonoParams& p, int hd, int grid, int smem_bytes, cudaStream_t s);

}  // namespace kie
