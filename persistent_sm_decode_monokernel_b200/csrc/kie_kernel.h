// Launch entry points of the persistent decode kernel (kie_kernel.cu).
#pragma once

#include <cuda_runtime.h>

#include <cuda_fp16.h>

#include "kie_params.h"

namespace kie {

// Dynamic shared memory the persistent kernels may use per CTA on the
// current device: the opt-in maximum per block minus their static shared
// memory (the parameter block's shared copy).
cudaError_t dynamic_smem_limit(int* out);

// Sets the dynamic shared-memory limit of the kernel instance for head
// dimension `hd` (64 or 128) and reports how many CTAs fit on one SM.
cudaError_t mono_configure(int hd, int smem_bytes, int* blocks_per_sm);

// Cooperative launch (all CTAs co-resident) of `grid` persistent CTAs.
cudaError_t mono_launch(const MonoParams& p, int hd, int grid, int smem_bytes, cudaStream_t s);

// FP8 E4M3 quantisation of one fp16 matrix W[N][K] (row-major, K a multiple
// of 16): codes[N][K] and one fp32 scale per row, the weight stream's rule.
cudaError_t quantize_launch(const __half* W, int N, int K, unsigned char* codes, float* scales,
                            cudaStream_t s);

// Copies the weight matrices into `packed`, each CTA's one-token stream at
// p.packed_off[cta], in the order the decode kernel streams them.
cudaError_t repack_launch(const MonoParams& p, unsigned char* packed, cudaStream_t s);

// Standalone weight-stream GEMV (the LM-head stage over an arbitrary
// matrix): y = W x, `iters` times; mode 0 streams without computing.
// gemv_configure raises the kernel's dynamic shared-memory limit to the
// current device's opt-in maximum (the same value on every call).
cudaError_t gemv_configure();
cudaError_t gemv_launch(const MonoParams& p, int mode, const float* x, float* y, int iters,
                        int grid, int smem_bytes, cudaStream_t s);

}  // namespace kie
