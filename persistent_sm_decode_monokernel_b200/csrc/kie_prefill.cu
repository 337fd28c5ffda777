// Batched prefill: the prompt's positions go through every layer at once,
// so the projections are matrix-matrix products and run on the 5th-generation
// tensor cores (tcgen05), with the causal attention over the prompt, RoPE,
// the KV-cache writes, the norms and SwiGLU in small kernels between them.
// The pages' resident program runs prefill as well as decode (revietech.ru,
// "Kog выжимает максимум из GPU: 3000 токенов/с", section "Что такое
// monokernel"); at batch 1 the decode steps are GEMVs, but a prompt of P
// tokens is P columns at once, a dense contraction.
//
// GEMM (kie_gemm_tn_kernel): D[M][N] = A[M][K] B[N][K]^T, A and B fp16
// row-major (both K-major), D fp32.  One CTA per 128 x 128 tile of D:
//   * warp 0, one lane: TMA loads of 128 x 64 tiles of A and B (128-byte
//     swizzle) into a 4-stage shared-memory pipeline (mbarriers with
//     transaction counts);
//   * warp 1, one lane: per stage four tcgen05.mma (M 128, N 128, K 16,
//     fp16 inputs, fp32 accumulators in tensor memory), then tcgen05.commit
//     to the stage's "empty" barrier; after the last stage, to "done";
//   * warps 0-3: tcgen05.ld of the accumulators (warp w reads tensor-memory
//     lanes 32w .. 32w+31 = rows of the tile) and the epilogue: store D, or
//     add it to an fp32 residual.
// Every wait is bounded; on expiry the CTA records an error and still frees
// its tensor memory.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kie_device.cuh"
#include "kie_prefill.h"

namespace kie {
namespace pf {

namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64, kStages = 4;
constexpr int kTileBytes = kBM * kBK * 2;            // one A or B stage tile (16 KB)
constexpr int kGemmThreads = 128;
constexpr long long kWaitNs = 2000000000LL;          // bound of every wait (2 s)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded wait on an mbarrier phase; false on timeout (error recorded).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, int* err, int where) {
  if (dev::mbar_try_wait(bar, parity)) return true;
  const long long t0 = dev::globaltimer();
  for (unsigned it = 1;; ++it) {
    if (dev::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u && dev::globaltimer() - t0 > kWaitNs) {
      atomicCAS(err, 0, where);
      return false;
    }
  }
}

// 2-D TMA tile load (box kBK x rows at element coordinates x, y), completion
// counted on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with 128-byte swizzle:
// rows of 128 bytes (64 fp16 of K), 8-row groups 1024 bytes apart (stride
// byte offset), descriptor version 1, swizzle mode 2 (128 B).  The tile
// starts at a 1024-byte boundary; `start` may be advanced by 32-byte steps
// within a row for the K = 16 slices of one MMA each.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t start) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFFu);           // start address, bits 0-13
  d |= (uint64_t)1u << 16;                           // leading byte offset (unused here)
  d |= (uint64_t)(1024u >> 4) << 32;                 // stride byte offset, bits 32-45
  d |= (uint64_t)1u << 46;                           // descriptor version
  d |= (uint64_t)2u << 61;                           // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: fp32 accumulators, fp16 A and B, both
// K-major, N = kBN, M = kBM.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

// D = A B^T over a grid of (N / kBN, M / kBM) tiles (rounded up); mode 0
// stores D into out[m][n] (leading dimension ldo), mode 1 adds it to out.
__global__ void __launch_bounds__(kGemmThreads, 1)
    kie_gemm_tn_kernel(const __grid_constant__ CUtensorMap map_a,
                       const __grid_constant__ CUtensorMap map_b, int M, int N, int K, float* out,
                       int ldo, int mode, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned stage tiles, then the barriers and the TMEM address
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* tiles = base;                                  // [stage][A | B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kStages * 2 * kTileBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 1);
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kStages, done = full0 + 16 * kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  const int nk = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(full0 + 8 * s, 1);
      dev::mbar_init(empty0 + 8 * s, 1);
    }
    dev::mbar_init(done, 1);
    dev::mbar_fence_init();
  }
  if (warp == 0) {   // 128 columns of tensor memory: the 128 x 128 fp32 accumulator
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t d_tmem = *tmem_slot;

  bool ok = true;
  if (warp == 0 && lane == 0) {
    // producer: A rows m0.., B rows n0.., K slice kb
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kStages;
      ok = wait_phase(empty0 + 8 * s, ((kb / kStages) + 1) & 1, err, 1);
      if (!ok) break;
      dev::mbar_arrive_expect_tx(full0 + 8 * s, 2 * kTileBytes);
      const uint32_t a_dst = smem_u32(tiles + (size_t)s * 2 * kTileBytes);
      tma_load_2d(a_dst, &map_a, kb * kBK, m0, full0 + 8 * s);
      tma_load_2d(a_dst + kTileBytes, &map_b, kb * kBK, n0, full0 + 8 * s);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kStages;
      ok = wait_phase(full0 + 8 * s, (kb / kStages) & 1, err, 2);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a = smem_u32(tiles + (size_t)s * 2 * kTileBytes), b = a + kTileBytes;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)
        umma_f16(d_tmem, sw128_desc(a + 32 * k), sw128_desc(b + 32 * k), (kb | k) != 0 ? 1u : 0u);
      umma_commit(empty0 + 8 * s);   // the stage's tiles may be overwritten once these MMAs are done
    }
    umma_commit(done);               // all MMAs issued so far (also on a failed wait)
  }
  // epilogue: every warp waits for the accumulator, then reads its 32 rows
  const bool got = wait_phase(done, 0, err, 3);
  __syncwarp();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const int m = m0 + warp * 32 + lane;
  if (got) {
#pragma unroll 1
    for (int c = 0; c < kBN; c += 16) {
      float v[16];
      tmem_ld16(d_tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      if (m < M) {
        float* o = out + (size_t)m * ldo + n0 + c;
        if (n0 + c + 16 <= N) {
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            float4* q = reinterpret_cast<float4*>(o + i);
            if (mode == 0) {
              *q = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            } else {
              float4 r = *q;
              r.x += v[i];
              r.y += v[i + 1];
              r.z += v[i + 2];
              r.w += v[i + 3];
              *q = r;
            }
          }
        } else {
          for (int i = 0; i < 16 && n0 + c + i < N; ++i) o[i] = mode == 0 ? v[i] : o[i] + v[i];
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(d_tmem) : "memory");
}

int gemm_smem_bytes() { return kStages * 2 * kTileBytes + 1024 + 128; }

cudaError_t gemm_tn(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, float* out,
                    int ldo, int mode, int* err, cudaStream_t s) {
  const dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM);
  kie_gemm_tn_kernel<<<grid, kGemmThreads, gemm_smem_bytes(), s>>>(a, b, M, N, K, out, ldo, mode, err);
  return cudaGetLastError();
}

cudaError_t gemm_configure() {
  return cudaFuncSetAttribute((const void*)kie_gemm_tn_kernel,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes());
}

// ----------------------------------------------------------- small kernels

// out[t][:] = fp16(g * x[t] / sqrt(mean(x[t]^2) + eps)), one block per row.
__global__ void kie_rmsnorm_rows_kernel(const float* x, const __half* g, int d, float eps,
                                        __half* out) {
  const int t = blockIdx.x;
  const float* xr = x + (size_t)t * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
  __shared__ float red[32];
  ss = dev::warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = dev::warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float rs = 1.0f / sqrtf(red[0] / (float)d + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    out[(size_t)t * d + i] = __float2half_rn(xr[i] * rs * __half2float(g[i]));
}

// x[t][:] = E[ids[t]] (fp32)
__global__ void kie_embed_rows_kernel(const int* ids, const __half* emb, int d, float* x) {
  const int t = blockIdx.x;
  const __half* e = emb + (size_t)ids[t] * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) x[(size_t)t * d + i] = __half2float(e[i]);
}

// RoPE on q and k rows of position t, K and V (fp16, RNE) into the cache of
// layer `layer`, q (times 1/sqrt(hd)) as fp16 for the attention kernel.
// qkv: [T][H*hd | KV*hd | KV*hd] fp32.
__global__ void kie_rope_kv_kernel(const float* qkv, const float2* rope, int H, int KV, int hd,
                                   int max_seq, int layer, __half* kv, __half* q16) {
  const int t = blockIdx.x;
  const int half = hd / 2, nq = H * hd, nkv = KV * hd, kvs = hd + 8;
  const float* row = qkv + (size_t)t * (nq + 2 * nkv);
  const float2* cs = rope + (size_t)t * half;
  const float scale = 1.0f / sqrtf((float)hd);
  __half* kbase = kv + (size_t)layer * 2 * KV * max_seq * kvs;
  __half* vbase = kbase + (size_t)KV * max_seq * kvs;
  for (int u = threadIdx.x; u < (H + KV) * half; u += blockDim.x) {
    const bool isq = u < H * half;
    const int uu = isq ? u : u - H * half;
    const int h = uu / half, i = uu - h * half;
    const float* src = isq ? row + h * hd : row + nq + h * hd;
    const float a = src[i], b = src[i + half];
    const float2 c = cs[i];
    const float lo = a * c.x - b * c.y, hi = b * c.x + a * c.y;
    if (isq) {
      q16[(size_t)t * nq + h * hd + i] = __float2half_rn(lo * scale);
      q16[(size_t)t * nq + h * hd + i + half] = __float2half_rn(hi * scale);
    } else {
      __half* kd = kbase + ((size_t)h * max_seq + t) * kvs;
      kd[i] = __float2half_rn(lo);
      kd[i + half] = __float2half_rn(hi);
    }
  }
  for (int e = threadIdx.x; e < nkv; e += blockDim.x) {
    const int h = e / hd, i = e - h * hd;
    vbase[((size_t)h * max_seq + t) * kvs + i] = __float2half_rn(row[nq + nkv + e]);
  }
}

// Causal attention over the prompt for one (block of 32 query positions,
// query head): scores against the cached K (fp16) of positions 0 .. t,
// online softmax in fp32, weighted sum of the cached V; o as fp16
// [T][H*hd].  One warp per query position (lane owns hd/32 dims); the
// block's warps share 32-position K and V tiles staged in shared memory.
template <int HD>
__global__ void __launch_bounds__(1024) kie_prefill_attn_kernel(const __half* q16, const __half* kv,
                                                                int T, int H, int KV, int max_seq,
                                                                int layer, __half* o16) {
  constexpr int DPL = HD / 32;                       // dims per lane
  constexpr int TK = 32;                             // key positions per tile
  __shared__ __align__(16) __half ks[TK][HD], vs[TK][HD];
  const int h = blockIdx.y, j = h / (H / KV);
  const int t0 = blockIdx.x * 32, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = t0 + w;
  const int kvs = HD + 8;
  const __half* K = kv + (((size_t)layer * 2 + 0) * KV + j) * (size_t)max_seq * kvs;
  const __half* V = kv + (((size_t)layer * 2 + 1) * KV + j) * (size_t)max_seq * kvs;
  float q[DPL], o[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    q[i] = t < T ? __half2float(q16[(size_t)t * H * HD + h * HD + lane * DPL + i]) : 0.f;
    o[i] = 0.f;
  }
  float mrun = -INFINITY, lrun = 0.f;
  const int last = min(T - 1, t0 + 31);              // last key any warp of the block needs
  for (int u0 = 0; u0 <= last; u0 += TK) {
    __syncthreads();
    // stage K and V rows u0 .. u0+TK-1 (16 bytes a thread per matrix)
    for (int e = threadIdx.x; e < TK * HD / 8; e += blockDim.x) {
      const int r = e / (HD / 8), c = (e - r * (HD / 8)) * 8;
      const bool in = u0 + r <= last;
      *reinterpret_cast<uint4*>(&ks[r][c]) =
          in ? *reinterpret_cast<const uint4*>(K + (size_t)(u0 + r) * kvs + c) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(&vs[r][c]) =
          in ? *reinterpret_cast<const uint4*>(V + (size_t)(u0 + r) * kvs + c) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    if (t < T) {
      const int nu = min(TK, t - u0 + 1);           // keys of this tile at or before t
      for (int r = 0; r < nu; ++r) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) s = fmaf(q[i], __half2float(ks[r][lane * DPL + i]), s);
        s = dev::warp_sum(s);
        const float mnew = fmaxf(mrun, s);
        const float al = __expf(mrun - mnew), pw = __expf(s - mnew);
        lrun = lrun * al + pw;
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[i] = o[i] * al + pw * __half2float(vs[r][lane * DPL + i]);
        mrun = mnew;
      }
    }
  }
  if (t < T) {
    const float inv = 1.0f / lrun;
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      o16[(size_t)t * H * HD + h * HD + lane * DPL + i] = __float2half_rn(o[i] * inv);
  }
}

// h[t][f] = fp16(silu(g) * u) from gu = [T][2F] (gate columns 0..F-1, up F..2F-1)
__global__ void kie_swiglu_kernel(const float* gu, int F, __half* h) {
  const int t = blockIdx.x;
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float g = gu[(size_t)t * 2 * F + f], u = gu[(size_t)t * 2 * F + F + f];
    h[(size_t)t * F + f] = __float2half_rn(g / (1.0f + expf(-g)) * u);
  }
}

cudaError_t embed_rows(const int* ids, const __half* emb, int T, int d, float* x, cudaStream_t s) {
  kie_embed_rows_kernel<<<T, 256, 0, s>>>(ids, emb, d, x);
  return cudaGetLastError();
}
cudaError_t rmsnorm_rows(const float* x, const __half* g, int T, int d, float eps, __half* out,
                         cudaStream_t s) {
  kie_rmsnorm_rows_kernel<<<T, 256, 0, s>>>(x, g, d, eps, out);
  return cudaGetLastError();
}
cudaError_t rope_kv(const float* qkv, const float2* rope, int T, int H, int KV, int hd, int max_seq,
                    int layer, __half* kv, __half* q16, cudaStream_t s) {
  kie_rope_kv_kernel<<<T, 256, 0, s>>>(qkv, rope, H, KV, hd, max_seq, layer, kv, q16);
  return cudaGetLastError();
}
cudaError_t attention(const __half* q16, const __half* kv, int T, int H, int KV, int hd, int max_seq,
                      int layer, __half* o16, cudaStream_t s) {
  const dim3 grid((T + 31) / 32, H);
  if (hd == 64)
    kie_prefill_attn_kernel<64><<<grid, 1024, 0, s>>>(q16, kv, T, H, KV, max_seq, layer, o16);
  else
    kie_prefill_attn_kernel<128><<<grid, 1024, 0, s>>>(q16, kv, T, H, KV, max_seq, layer, o16);
  return cudaGetLastError();
}
cudaError_t swiglu(const float* gu, int T, int F, __half* h, cudaStream_t s) {
  kie_swiglu_kernel<<<T, 256, 0, s>>>(gu, F, h);
  return cudaGetLastError();
}

}  // namespace pf
}  // namespace kie
