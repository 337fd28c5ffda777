// Batched prefill kernels (kie_prefill.cu): a tcgen05 GEMM over the prompt's
// positions and the small kernels between the projections.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace kie {
namespace pf {

// D[M][N] = A[M][K] B[N][K]^T with A, B fp16 row-major described by 2-D
// tensor maps of 64 x 128 boxes with 128-byte swizzle (K a multiple of 64);
// mode 0 stores D to out (fp32, leading dimension ldo, 16-byte aligned rows),
// mode 1 adds D to it.  *err (device) gets a nonzero code if a bounded wait
// gave up.
cudaError_t gemm_tn(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, float* out,
                    int ldo, int mode, int* err, cudaStream_t s);
cudaError_t gemm_configure();
int gemm_smem_bytes();

// x[t] = E[ids[t]] (fp32 rows)
cudaError_t embed_rows(const int* ids, const __half* emb, int T, int d, float* x, cudaStream_t s);
// out[t] = fp16(g * x[t] / rms(x[t]))
cudaError_t rmsnorm_rows(const float* x, const __half* g, int T, int d, float eps, __half* out,
                         cudaStream_t s);
// RoPE of the q and k parts of qkv rows (position = row), K and V of layer
// `layer` into the padded fp16 cache, q / sqrt(hd) as fp16 [T][H*hd]
cudaError_t rope_kv(const float* qkv, const float2* rope, int T, int H, int KV, int hd, int max_seq,
                    int layer, __half* kv, __half* q16, cudaStream_t s);
// causal attention of every position over the cached K, V of positions <= it
cudaError_t attention(const __half* q16, const __half* kv, int T, int H, int KV, int hd, int max_seq,
                      int layer, __half* o16, cudaStream_t s);
// h = fp16(silu(gate) * up), gu rows [gate (F) | up (F)]
cudaError_t swiglu(const float* gu, int T, int F, __half* h, cudaStream_t s);

}  // namespace pf
}  // namespace kie
