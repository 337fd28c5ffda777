// Host side of the C ABI declared in include/kie.h: validation, planning,
// scratch ownership, launches of the persistent decode kernel and session
// state (position, fed ids).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "kie.h"
#include "kie_guard.h"
#include "kie_kernel.h"
#include "kie_params.h"
#include "kie_plan.h"
#include "kie_prefill.h"
#include "kie_units.h"

using kie::DevStatus;
using kie::LayerW;
using kie::MonoParams;

struct kie_ctx {
  kie_model_desc desc{};
  kie::Shape shape{};
  int device = 0;
  cudaStream_t stream = nullptr;

  // caller-owned device memory
  std::vector<LayerW> hlayers;
  const __half *tok_emb = nullptr, *final_norm = nullptr, *lm_head = nullptr;
  __half* kv = nullptr;

  // library-owned device memory
  LayerW* dlayers = nullptr;
  float2* rope = nullptr;
  int2* ranges = nullptr;
  unsigned long long* tagged = nullptr;
  size_t tagged_words = 0;
  unsigned long long *x_attn = nullptr, *x_ffn = nullptr, *hbuf = nullptr, *qbuf = nullptr,
                     *kvnew = nullptr, *obuf = nullptr, *slots = nullptr, *cands = nullptr;
  unsigned long long* partials = nullptr;
  int* d_ids = nullptr;               // fed ids of a launch [max_seq]
  unsigned char* d_io = nullptr;      // DevStatus + out ids [max_seq]
  unsigned long long* cta_stats = nullptr;
  unsigned char* h_io = nullptr;      // pinned mirror of d_io
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;

  // plan
  std::vector<std::vector<int2>> hranges;
  int grid = 0, ring_bytes = 0, chunk_bytes = 65536, smem = 0, max_split = 1, min_split_len = 64;
  unsigned char* packed = nullptr;            // weight matrices in per-CTA stream order
  unsigned long long* packed_off = nullptr;   // [grid]
  size_t packed_bytes = 0;
  int w8 = 0;                                 // packed stream: 0 fp16, 1 fp8 E4M3 + row scales
  // batched prefill (tensor-core GEMMs over the prompt) and its scratch,
  // grown to the longest prompt seen
  int batched_prefill = 1;
  int tmem_park = 1;
  int pf_cap = 0;
  int* pf_ids = nullptr;
  float *pf_x = nullptr, *pf_qkv = nullptr, *pf_gu = nullptr;
  __half *pf_a = nullptr, *pf_q = nullptr;
  int* pf_err = nullptr;
  cudaEvent_t pf_ev0 = nullptr, pf_ev1 = nullptr;
  float* wscale = nullptr;                    // fp8: row scales, each CTA's in stream order
  unsigned long long* wscale_off = nullptr;   // fp8: [grid] offsets (floats) into wscale
  kie::SmemLayout sm{};

  // session
  int pos = 0;
  bool primed = false;             // a prefill ran; next_tok is valid
  std::vector<int32_t> fed;        // fed[t] = id fed at position t
  int32_t next_tok = 0;            // id to feed at position pos
  unsigned int epoch = 0;
  bool failed = false;

  // options and capture
  long long timeout_ns = 2000000000LL;
  unsigned poll_ns = 0;
  long long l2_prefetch = 0;
  int fault_cta = -1, fault_step = -1, fault_layer = -1, fault_stage = -1;
  float* capture = nullptr;
  int capture_rows = 0;
  // token selection: temperature 0 = greedy; ids that end a decode (empty:
  // the model descriptor's eos_id, if any)
  double temperature = 0.0;
  unsigned long long seed = 0;
  int top_k = 0;          // 0: no top-k restriction of the draw
  double top_p = 1.0;     // 1: no top-p restriction
  std::vector<int32_t> eos_ids;
  unsigned long long* trace = nullptr;
  int trace_cta = 0, trace_steps = 0, trace_clock = 0;

  kie_stats stats{};
  std::string err;
};

namespace {

constexpr size_t kStatusBytes = sizeof(DevStatus);

// Attention partials: per CTA, G rows of 2 + head_dim/2 tagged words.
size_t partial_bytes(const kie_ctx* c) {
  const size_t G = c->desc.n_heads / c->desc.n_kv_heads;
  return sizeof(unsigned long long) * (size_t)c->grid * G * (c->desc.head_dim / 2 + 2);
}

kie_status set_err(kie_ctx* c, kie_status s, const std::string& msg) {
  if (c) c->err = msg;
  return s;
}

kie_status cuda_fail(kie_ctx* c, cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorString(e);
  if (c) c->failed = true;
  return set_err(c, KIE_ERR_CUDA, m);
}

#define KIE_CUDA(c, call)                                   \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return cuda_fail((c), e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kie::Shape shape_of(const kie_model_desc& d) {
  return kie::Shape{d.n_layers, d.d_model, d.n_heads, d.n_kv_heads, d.head_dim, d.ffn_dim,
                    d.vocab};
}

void free_all(kie_ctx* c) {
  cudaFree(c->dlayers);
  cudaFree(c->rope);
  cudaFree(c->ranges);
  cudaFree(c->tagged);
  cudaFree(c->partials);
  cudaFree(c->d_ids);
  cudaFree(c->d_io);
  cudaFree(c->cta_stats);
  cudaFree(c->packed);
  cudaFree(c->packed_off);
  cudaFree(c->wscale);
  cudaFree(c->wscale_off);
  cudaFree(c->pf_ids);
  cudaFree(c->pf_x);
  cudaFree(c->pf_qkv);
  cudaFree(c->pf_gu);
  cudaFree(c->pf_a);
  cudaFree(c->pf_q);
  cudaFree(c->pf_err);
  if (c->pf_ev0) cudaEventDestroy(c->pf_ev0);
  if (c->pf_ev1) cudaEventDestroy(c->pf_ev1);
  if (c->h_io) cudaFreeHost(c->h_io);
  if (c->ev0) cudaEventDestroy(c->ev0);
  if (c->ev1) cudaEventDestroy(c->ev1);
}

// One launch of the persistent kernel over n_steps forward passes starting
// at position pos0.  Step i feeds ids[i] when `forced`, else first_tok for
// i = 0 and the previous pick afterwards; steps i >= lm_from pick an id.
kie_status launch(kie_ctx* c, int n_steps, int pos0, const int32_t* host_ids, bool forced,
                  int first_tok, int lm_from, int* n_done_out) {
  const kie_model_desc& d = c->desc;
  const unsigned need = (unsigned)n_steps * (unsigned)(d.n_layers + 1) + 2u;
  if ((unsigned long long)c->epoch + need >= 0xFFFFFF00ull) {
    KIE_CUDA(c, cudaMemsetAsync(c->tagged, 0, c->tagged_words * 8, c->stream));
    KIE_CUDA(c, cudaMemsetAsync(c->partials, 0, partial_bytes(c), c->stream));
    c->epoch = 0;
  }
  if (forced) {
    KIE_CUDA(c, cudaMemcpyAsync(c->d_ids, host_ids, sizeof(int32_t) * n_steps,
                                cudaMemcpyHostToDevice, c->stream));
  }
  KIE_CUDA(c, cudaMemsetAsync(c->d_io, 0, kStatusBytes, c->stream));

  MonoParams p{};
  p.L = d.n_layers;
  p.d = d.d_model;
  p.H = d.n_heads;
  p.KV = d.n_kv_heads;
  p.hd = d.head_dim;
  p.F = d.ffn_dim;
  p.V = d.vocab;
  p.G = d.n_heads / d.n_kv_heads;
  p.eps = d.rms_eps;
  p.max_seq = d.max_seq;
  if (!c->eos_ids.empty()) {
    p.n_eos = (int)c->eos_ids.size();
    for (int k = 0; k < p.n_eos; ++k) p.eos_ids[k] = c->eos_ids[k];
  } else if (d.eos_id >= 0) {
    p.n_eos = 1;
    p.eos_ids[0] = d.eos_id;
  }
  p.sample = c->temperature > 0.0 ? 1 : 0;
  p.inv_temp = c->temperature > 0.0 ? 1.0 / c->temperature : 0.0;
  p.seed = c->seed;
  p.top_k = c->top_k;
  p.top_p = c->top_p;
  p.cands = c->cands;
  p.layers = c->dlayers;
  p.tok_emb = c->tok_emb;
  p.final_norm = c->final_norm;
  p.lm_head = c->lm_head;
  p.kv = c->kv;
  p.rope = c->rope;
  p.ranges = c->ranges;
  p.grid = c->grid;
  p.ring_bytes = c->ring_bytes;
  p.chunk_bytes = c->chunk_bytes;
  p.packed = c->packed;
  p.packed_off = c->packed_off;
  p.w8 = c->w8;
  p.wscale = c->wscale;
  p.wscale_off = c->wscale_off;
  p.max_split = c->max_split;
  p.min_split_len = c->min_split_len;
  p.sm = c->sm;
  p.x_attn = c->x_attn;
  p.x_ffn = c->x_ffn;
  p.hbuf = c->hbuf;
  p.qbuf = c->qbuf;
  p.kvnew = c->kvnew;
  p.obuf = c->obuf;
  p.slots = c->slots;
  p.partials = c->partials;
  p.n_steps = n_steps;
  p.pos0 = pos0;
  p.first_tok = first_tok;
  p.forced = forced ? c->d_ids : nullptr;
  p.lm_from = lm_from;
  p.e0 = c->epoch;
  p.capture = c->capture;
  p.capture_rows = c->capture_rows;
  p.out_ids = reinterpret_cast<int*>(c->d_io + kStatusBytes);
  p.status = reinterpret_cast<DevStatus*>(c->d_io);
  p.cta_stats = c->cta_stats;
  p.timeout_ns = c->timeout_ns;
  p.poll_ns = c->poll_ns;
  p.l2_prefetch = c->l2_prefetch;
  p.tmem_park = c->tmem_park;
  p.trace = c->trace;
  p.trace_cta = c->trace_cta;
  p.trace_steps = c->trace_steps;
  p.trace_clock = c->trace_clock;
  p.fault_cta = c->fault_cta;
  p.fault_step = c->fault_step;
  p.fault_layer = c->fault_layer;
  p.fault_stage = c->fault_stage;

  KIE_CUDA(c, cudaEventRecord(c->ev0, c->stream));
  KIE_CUDA(c, kie::mono_launch(p, d.head_dim, c->grid, c->smem, c->stream));
  KIE_CUDA(c, cudaEventRecord(c->ev1, c->stream));
  KIE_CUDA(c, cudaMemcpyAsync(c->h_io, c->d_io, kStatusBytes + sizeof(int32_t) * n_steps,
                              cudaMemcpyDeviceToHost, c->stream));
  KIE_CUDA(c, cudaStreamSynchronize(c->stream));
  c->epoch += need;
  c->stats.launches += 1;
  float ms = 0.f;
  cudaEventElapsedTime(&ms, c->ev0, c->ev1);
  c->stats.last_device_ms = ms;

  const DevStatus* st = reinterpret_cast<const DevStatus*>(c->h_io);
  c->stats.last_steps = st->n_done;
  *n_done_out = st->n_done;
  if (st->code != kie::DEV_OK) {
    c->failed = true;
    char buf[256];
    std::snprintf(buf, sizeof buf,
                  "device %s in CTA %d (step %d, layer %d, stage %d, site %d)",
                  st->code == kie::DEV_TIMEOUT ? "wait timeout" : "protocol violation", st->cta,
                  st->step, st->layer, st->stage, st->where);
    return set_err(c, st->code == kie::DEV_TIMEOUT ? KIE_ERR_TIMEOUT : KIE_ERR_PROTOCOL, buf);
  }
  return KIE_OK;
}

// (Re)builds the library's stream-ordered copy of the weight matrices for
// the current partition, chunk size and weight format (fp16, or fp8 E4M3
// with row scales computed on the device first).  Reads the caller's
// matrices.
kie_status repack(kie_ctx* c) {
  std::vector<unsigned long long> off(c->grid), soff(c->grid);
  size_t total = 0, srows = 0;
  for (int i = 0; i < c->grid; ++i) {
    off[i] = total;
    total += (kie::stream_bytes(c->shape, c->hranges, i, c->w8 ? 1 : 2) + 511) / 512 * 512;
    soff[i] = srows;
    srows += kie::stream_rows(c->shape, c->hranges, i);
  }
  cudaFree(c->packed);
  c->packed = nullptr;
  cudaFree(c->wscale);
  c->wscale = nullptr;
  if (!c->packed_off) KIE_CUDA(c, cudaMalloc(&c->packed_off, sizeof(unsigned long long) * c->grid));
  KIE_CUDA(c, cudaMalloc(&c->packed, total));
  c->packed_bytes = total;
  KIE_CUDA(c, cudaMemcpyAsync(c->packed_off, off.data(), sizeof(unsigned long long) * c->grid,
                              cudaMemcpyHostToDevice, c->stream));
  if (c->w8) {
    if (!c->wscale_off)
      KIE_CUDA(c, cudaMalloc(&c->wscale_off, sizeof(unsigned long long) * c->grid));
    KIE_CUDA(c, cudaMalloc(&c->wscale, sizeof(float) * srows));
    KIE_CUDA(c, cudaMemcpyAsync(c->wscale_off, soff.data(), sizeof(unsigned long long) * c->grid,
                                cudaMemcpyHostToDevice, c->stream));
  }
  MonoParams p{};
  p.L = c->desc.n_layers;
  p.d = c->desc.d_model;
  p.H = c->desc.n_heads;
  p.KV = c->desc.n_kv_heads;
  p.hd = c->desc.head_dim;
  p.F = c->desc.ffn_dim;
  p.V = c->desc.vocab;
  p.layers = c->dlayers;
  p.lm_head = c->lm_head;
  p.ranges = c->ranges;
  p.grid = c->grid;
  p.chunk_bytes = c->chunk_bytes;
  p.sm = c->sm;   // the unit plan reads the result-slot count
  p.packed_off = c->packed_off;
  p.w8 = c->w8;
  p.wscale = c->wscale;
  p.wscale_off = c->wscale_off;
  KIE_CUDA(c, kie::repack_launch(p, c->packed, c->stream));
  KIE_CUDA(c, cudaStreamSynchronize(c->stream));
  return KIE_OK;
}

// ------------------------------------------------------- batched prefill

using TmapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, resolved through the runtime (the library
// links no driver library); null if the driver does not offer it.
TmapEncodeFn tmap_encoder() {
  static const TmapEncodeFn fn = []() -> TmapEncodeFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<TmapEncodeFn>(f);
  }();
  return fn;
}

// Tensor map of an fp16 row-major matrix [rows][cols] (cols a multiple of
// 64, base 16-byte aligned): boxes of 64 columns x 128 rows, 128-byte
// swizzle, rows past the end read as zeros.
bool make_map(CUtensorMap* m, const void* base, int rows, int cols) {
  const TmapEncodeFn enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool batched_prefill_possible(const kie_ctx* c, int n) {
  return c->batched_prefill && !c->w8 && n >= 2 && tmap_encoder() != nullptr;
}

// Positions 0 .. T-1 of `ids` through every layer at once: K and V of each
// position written to the cache (the decode kernel's layout), nothing else
// kept.  Per layer: RMSNorm, Q / K / V GEMMs, RoPE + cache writes, causal
// attention, O GEMM added to the residual, RMSNorm, gate and up GEMMs,
// SwiGLU, down GEMM added to the residual.
kie_status batched_prefill(kie_ctx* c, const int32_t* ids, int T) {
  const kie_model_desc& d = c->desc;
  const int D = d.d_model, F = d.ffn_dim, H = d.n_heads, KV = d.n_kv_heads, hd = d.head_dim;
  const int nq = H * hd, nkv = KV * hd, nqkv = nq + 2 * nkv;
  cudaStream_t st = c->stream;
  if (T > c->pf_cap) {
    cudaFree(c->pf_ids);
    cudaFree(c->pf_x);
    cudaFree(c->pf_qkv);
    cudaFree(c->pf_gu);
    cudaFree(c->pf_a);
    cudaFree(c->pf_q);
    c->pf_ids = nullptr;
    c->pf_x = c->pf_qkv = c->pf_gu = nullptr;
    c->pf_a = c->pf_q = nullptr;
    c->pf_cap = 0;
    const size_t wide = (size_t)std::max(std::max(D, F), nq);
    KIE_CUDA(c, cudaMalloc(&c->pf_ids, sizeof(int) * T));
    KIE_CUDA(c, cudaMalloc(&c->pf_x, sizeof(float) * T * (size_t)D));
    KIE_CUDA(c, cudaMalloc(&c->pf_qkv, sizeof(float) * T * (size_t)nqkv));
    KIE_CUDA(c, cudaMalloc(&c->pf_gu, sizeof(float) * T * 2 * (size_t)F));
    KIE_CUDA(c, cudaMalloc(&c->pf_a, sizeof(__half) * T * wide));
    KIE_CUDA(c, cudaMalloc(&c->pf_q, sizeof(__half) * T * (size_t)nq));
    if (!c->pf_err) KIE_CUDA(c, cudaMalloc(&c->pf_err, sizeof(int)));
    KIE_CUDA(c, kie::pf::gemm_configure());
    c->pf_cap = T;
  }
  CUtensorMap a_d, a_nq, a_f;   // views of the fp16 activation buffer
  if (!make_map(&a_d, c->pf_a, T, D) || !make_map(&a_nq, c->pf_a, T, nq) ||
      !make_map(&a_f, c->pf_a, T, F))
    return set_err(c, KIE_ERR_CUDA, "tensor map of the prefill activations");
  KIE_CUDA(c, cudaMemcpyAsync(c->pf_ids, ids, sizeof(int) * T, cudaMemcpyHostToDevice, st));
  KIE_CUDA(c, cudaMemsetAsync(c->pf_err, 0, sizeof(int), st));
  KIE_CUDA(c, kie::pf::embed_rows(c->pf_ids, c->tok_emb, T, D, c->pf_x, st));
  for (int l = 0; l < d.n_layers; ++l) {
    const LayerW& w = c->hlayers[l];
    CUtensorMap bq, bk, bv, bo, bg, bu, bd;
    if (!make_map(&bq, w.wq, nq, D) || !make_map(&bk, w.wk, nkv, D) || !make_map(&bv, w.wv, nkv, D) ||
        !make_map(&bo, w.wo, D, nq) || !make_map(&bg, w.wg, F, D) || !make_map(&bu, w.wu, F, D) ||
        !make_map(&bd, w.wd, D, F))
      return set_err(c, KIE_ERR_CUDA, "tensor map of a weight matrix");
    KIE_CUDA(c, kie::pf::rmsnorm_rows(c->pf_x, w.attn_norm, T, D, d.rms_eps, c->pf_a, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_d, bq, T, nq, D, c->pf_qkv, nqkv, 0, c->pf_err, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_d, bk, T, nkv, D, c->pf_qkv + nq, nqkv, 0, c->pf_err, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_d, bv, T, nkv, D, c->pf_qkv + nq + nkv, nqkv, 0, c->pf_err, st));
    KIE_CUDA(c, kie::pf::rope_kv(c->pf_qkv, c->rope, T, H, KV, hd, d.max_seq, l, c->kv, c->pf_q, st));
    KIE_CUDA(c, kie::pf::attention(c->pf_q, c->kv, T, H, KV, hd, d.max_seq, l, c->pf_a, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_nq, bo, T, D, nq, c->pf_x, D, 1, c->pf_err, st));
    KIE_CUDA(c, kie::pf::rmsnorm_rows(c->pf_x, w.ffn_norm, T, D, d.rms_eps, c->pf_a, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_d, bg, T, F, D, c->pf_gu, 2 * F, 0, c->pf_err, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_d, bu, T, F, D, c->pf_gu + F, 2 * F, 0, c->pf_err, st));
    KIE_CUDA(c, kie::pf::swiglu(c->pf_gu, T, F, c->pf_a, st));
    KIE_CUDA(c, kie::pf::gemm_tn(a_f, bd, T, D, F, c->pf_x, D, 1, c->pf_err, st));
  }
  int err = 0;
  KIE_CUDA(c, cudaMemcpyAsync(&err, c->pf_err, sizeof(int), cudaMemcpyDeviceToHost, st));
  KIE_CUDA(c, cudaStreamSynchronize(st));
  if (err != 0) {
    c->failed = true;
    return set_err(c, KIE_ERR_TIMEOUT, "a bounded wait of the prefill GEMM gave up");
  }
  return KIE_OK;
}

kie_status usable(kie_ctx* c) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (c->failed) return set_err(c, KIE_ERR_STATE, "context failed earlier; destroy it");
  c->err.clear();
  return KIE_OK;
}

}  // namespace

extern "C" {

size_t kie_kv_cache_bytes(const kie_model_desc* d) {
  if (!d || kie_check_desc(d) != KIE_OK) return 0;
  return (size_t)2 * d->n_layers * d->n_kv_heads * (size_t)d->max_seq * (d->head_dim + kie::kKvPad) *
         2;
}

kie_status kie_check_desc(const kie_model_desc* d) {
  if (!d) return KIE_ERR_INVALID_ARG;
  if (d->n_layers < 1 || d->d_model < 1 || d->n_heads < 1 || d->n_kv_heads < 1 ||
      d->head_dim < 1 || d->ffn_dim < 1 || d->vocab < 1 || d->max_seq < 1)
    return KIE_ERR_INVALID_ARG;
  if (!(d->rms_eps >= 0.f) || !(d->rope_base > 0.f) || !std::isfinite(d->rope_base))
    return KIE_ERR_INVALID_ARG;
  if (d->eos_id < -1 || d->eos_id >= d->vocab) return KIE_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return KIE_ERR_UNSUPPORTED;
  if (d->n_heads % d->n_kv_heads != 0) return KIE_ERR_UNSUPPORTED;
  if (d->n_heads / d->n_kv_heads > kie::kMaxGroup) return KIE_ERR_UNSUPPORTED;
  if (d->d_model % 256 || d->ffn_dim % 256 || (d->n_heads * d->head_dim) % 256)
    return KIE_ERR_UNSUPPORTED;
  return KIE_OK;
}

kie_status kie_plan_units(const kie_model_desc* d, int32_t grid, int32_t stage, int32_t cta,
                          int32_t* begin, int32_t* end) {
  return kie::no_throw([&]() -> kie_status {
    if (!d || !begin || !end) return KIE_ERR_INVALID_ARG;
    kie_status s = kie_check_desc(d);
    if (s != KIE_OK) return s;
    if (grid < 1 || stage < 0 || stage >= kie::N_STAGES || cta < 0 || cta >= grid)
      return KIE_ERR_INVALID_ARG;
    const auto r = kie::partition(shape_of(*d), grid, stage);
    *begin = r[cta].x;
    *end = r[cta].y;
    return KIE_OK;
  });
}

kie_status kie_plan_gemv_work(const kie_model_desc* d, int32_t grid, int32_t stage, int32_t cta,
                              int32_t chunk_bytes, int32_t fp8, int32_t* out) {
  return kie::no_throw([&]() -> kie_status {
    if (!d || !out) return KIE_ERR_INVALID_ARG;
    kie_status s = kie_check_desc(d);
    if (s != KIE_OK) return s;
    if (grid < 1 || stage < 0 || stage >= kie::N_STAGES || cta < 0 || cta >= grid ||
        chunk_bytes < 8192 || chunk_bytes % 512 || chunk_bytes > (1 << 20) || (fp8 != 0 && fp8 != 1))
      return KIE_ERR_INVALID_ARG;
    const kie::Shape sh = shape_of(*d);
    std::vector<std::vector<int2>> ranges(kie::N_STAGES);
    for (int st = 0; st < kie::N_STAGES; ++st) ranges[st] = kie::partition(sh, grid, st);
    kie::StagePlan pl{};
    pl.rows = kie::rows_in_range(sh, stage, ranges[stage][cta].x, ranges[stage][cta].y);
    pl.kp = kie::stage_k(sh, stage) / kie::kPieceElems;
    const int slots = kie::gemv_slots(sh, ranges, grid, chunk_bytes);
    kie::plan_units(pl, chunk_bytes, kie::piece_bytes(fp8), slots);
    out[0] = pl.rows;
    out[1] = pl.kp;
    out[2] = pl.nr;
    out[3] = pl.S;
    out[4] = pl.nb;
    out[5] = slots;
    return KIE_OK;
  });
}

kie_status kie_create(const kie_model_desc* d, const kie_weights* w, void* kv_cache,
                      void* cuda_stream, kie_ctx** out) {
  return kie::no_throw([&]() -> kie_status {
    if (!out) return KIE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!d || !w || !kv_cache || !w->layers || !w->tok_emb || !w->final_norm || !w->lm_head)
      return KIE_ERR_INVALID_ARG;
    kie_status s = kie_check_desc(d);
    if (s != KIE_OK) return s;
    if (!aligned16(kv_cache) || !aligned16(w->tok_emb) || !aligned16(w->final_norm) ||
        !aligned16(w->lm_head))
      return KIE_ERR_INVALID_ARG;
    for (int l = 0; l < d->n_layers; ++l) {
      const kie_layer_weights& lw = w->layers[l];
      const void* ps[] = {lw.attn_norm, lw.wq, lw.wk, lw.wv, lw.wo, lw.ffn_norm, lw.w_gate, lw.w_up,
                          lw.w_down};
      for (const void* q : ps)
        if (!q || !aligned16(q)) return KIE_ERR_INVALID_ARG;
    }

    kie_ctx* c = new kie_ctx();
    c->desc = *d;
    c->shape = shape_of(*d);
    c->stream = static_cast<cudaStream_t>(cuda_stream);
    c->tok_emb = static_cast<const __half*>(w->tok_emb);
    c->final_norm = static_cast<const __half*>(w->final_norm);
    c->lm_head = static_cast<const __half*>(w->lm_head);
    c->kv = static_cast<__half*>(kv_cache);
    for (int l = 0; l < d->n_layers; ++l) {
      const kie_layer_weights& lw = w->layers[l];
      c->hlayers.push_back(LayerW{static_cast<const __half*>(lw.attn_norm),
                                  static_cast<const __half*>(lw.wq), static_cast<const __half*>(lw.wk),
                                  static_cast<const __half*>(lw.wv), static_cast<const __half*>(lw.wo),
                                  static_cast<const __half*>(lw.ffn_norm),
                                  static_cast<const __half*>(lw.w_gate),
                                  static_cast<const __half*>(lw.w_up),
                                  static_cast<const __half*>(lw.w_down)});
    }
    auto fail = [&](kie_status st) {
      free_all(c);
      delete c;
      return st;
    };
    auto cuda_bad = [&](cudaError_t e) { return e != cudaSuccess; };

    if (cuda_bad(cudaGetDevice(&c->device))) return fail(KIE_ERR_CUDA);
    int n_sm = 0, smem_optin = 0;
    if (cuda_bad(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, c->device)) ||
        cuda_bad(kie::dynamic_smem_limit(&smem_optin)))
      return fail(KIE_ERR_CUDA);

    // grid: one CTA per SM, but never more CTAs than units of the smallest stage
    int grid = n_sm;
    for (int st = 0; st < kie::N_STAGES; ++st)
      grid = std::min(grid, kie::stage_units(c->shape, st));
    c->grid = grid;
    c->hranges.resize(kie::N_STAGES);
    for (int st = 0; st < kie::N_STAGES; ++st) c->hranges[st] = kie::partition(c->shape, grid, st);
    // 32 KB chunks (measured fastest on the 2.2B and 8B models), else 16 KB
    bool planned = false;
    for (int cb : {32768, 16384}) {
      c->chunk_bytes = cb;
      if ((planned = kie::plan_smem(c->shape, grid, cb, smem_optin, c->hranges, &c->sm,
                                    &c->ring_bytes)))
        break;
    }
    if (!planned) return fail(KIE_ERR_UNSUPPORTED);
    c->smem = c->sm.total;
    int per_sm = 0;
    if (cuda_bad(kie::mono_configure(d->head_dim, c->smem, &per_sm))) return fail(KIE_ERR_CUDA);
    if (per_sm < 1) return fail(KIE_ERR_UNSUPPORTED);
    c->max_split = std::max(1, std::min(grid / d->n_kv_heads, kie::kMaxSplitCombine));

    const int G = d->n_heads / d->n_kv_heads;
    const size_t qd = (size_t)d->n_heads * d->head_dim, kvd = (size_t)d->n_kv_heads * d->head_dim;
    // activation vectors, argmax slots, top-k candidate lists
    c->tagged_words = 2 * (size_t)d->d_model + d->ffn_dim + qd + 2 * kvd + qd + 2 * (size_t)grid +
                      2 * (size_t)kie::kMaxTopK * grid;
    std::vector<int2> flat;
    for (auto& v : c->hranges) flat.insert(flat.end(), v.begin(), v.end());
    const size_t half = d->head_dim / 2;
    std::vector<float2> rope((size_t)d->max_seq * half);
    for (int t = 0; t < d->max_seq; ++t)
      for (size_t i = 0; i < half; ++i) {
        const double th = std::pow((double)d->rope_base, -2.0 * (double)i / d->head_dim);
        const double a = (double)t * th;
        rope[(size_t)t * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }

    if (cuda_bad(cudaMalloc(&c->dlayers, sizeof(LayerW) * d->n_layers)) ||
        cuda_bad(cudaMalloc(&c->rope, sizeof(float2) * rope.size())) ||
        cuda_bad(cudaMalloc(&c->ranges, sizeof(int2) * flat.size())) ||
        cuda_bad(cudaMalloc(&c->tagged, 8 * c->tagged_words)) ||
        cuda_bad(cudaMalloc(&c->partials, partial_bytes(c))) ||
        cuda_bad(cudaMalloc(&c->d_ids, sizeof(int32_t) * d->max_seq)) ||
        cuda_bad(cudaMalloc(&c->d_io, kStatusBytes + sizeof(int32_t) * d->max_seq)) ||
        cuda_bad(cudaMalloc(&c->cta_stats, sizeof(unsigned long long) * kie::kStatsPerCta * grid)) ||
        cuda_bad(cudaMallocHost(&c->h_io, kStatusBytes + sizeof(int32_t) * d->max_seq)) ||
        cuda_bad(cudaEventCreate(&c->ev0)) || cuda_bad(cudaEventCreate(&c->ev1)))
      return fail(KIE_ERR_CUDA);
    unsigned long long* t = c->tagged;
    c->x_attn = t;  t += d->d_model;
    c->x_ffn = t;   t += d->d_model;
    c->hbuf = t;    t += d->ffn_dim;
    c->qbuf = t;    t += qd;
    c->kvnew = t;   t += 2 * kvd;
    c->obuf = t;    t += qd;
    c->slots = t;   t += 2 * (size_t)grid;
    c->cands = t;
    if (cuda_bad(cudaMemcpyAsync(c->dlayers, c->hlayers.data(), sizeof(LayerW) * d->n_layers,
                                 cudaMemcpyHostToDevice, c->stream)) ||
        cuda_bad(cudaMemcpyAsync(c->rope, rope.data(), sizeof(float2) * rope.size(),
                                 cudaMemcpyHostToDevice, c->stream)) ||
        cuda_bad(cudaMemcpyAsync(c->ranges, flat.data(), sizeof(int2) * flat.size(),
                                 cudaMemcpyHostToDevice, c->stream)) ||
        cuda_bad(cudaMemsetAsync(c->tagged, 0, 8 * c->tagged_words, c->stream)) ||
        cuda_bad(cudaMemsetAsync(c->partials, 0, partial_bytes(c), c->stream)) ||
        cuda_bad(cudaMemsetAsync(c->cta_stats, 0, sizeof(unsigned long long) * kie::kStatsPerCta * grid,
                                 c->stream)) ||
        cuda_bad(cudaStreamSynchronize(c->stream)))
      return fail(KIE_ERR_CUDA);

    if (repack(c) != KIE_OK) return fail(KIE_ERR_CUDA);
    c->stats.grid = grid;
    c->stats.ring_bytes = c->ring_bytes;
    c->stats.chunk_bytes = c->chunk_bytes;
    c->stats.smem_bytes = c->smem;
    *out = c;
    return KIE_OK;
  });
}

kie_status kie_prefill(kie_ctx* c, const int32_t* ids, int32_t n, int32_t* first_id) {
  return kie::no_throw([&]() -> kie_status {
    kie_status s = usable(c);
    if (s != KIE_OK) return s;
    if (!ids || n < 1) return set_err(c, KIE_ERR_INVALID_ARG, "prefill needs n >= 1 ids");
    if (n > c->desc.max_seq) return set_err(c, KIE_ERR_CAPACITY, "prompt longer than max_seq");
    for (int i = 0; i < n; ++i)
      if (ids[i] < 0 || ids[i] >= c->desc.vocab)
        return set_err(c, KIE_ERR_INVALID_ARG, "prompt id out of range");
    c->primed = false;
    int done = 0;
    if (!c->pf_ev0) {
      KIE_CUDA(c, cudaEventCreate(&c->pf_ev0));
      KIE_CUDA(c, cudaEventCreate(&c->pf_ev1));
    }
    KIE_CUDA(c, cudaEventRecord(c->pf_ev0, c->stream));
    const bool batched = batched_prefill_possible(c, n);
    int32_t g0 = 0;
    if (batched) {
      // positions 0 .. n-2 at once, then the last one as a decode step that
      // picks the first id
      s = batched_prefill(c, ids, n - 1);
      if (s != KIE_OK) return s;
      s = launch(c, 1, n - 1, ids + n - 1, true, 0, 0, &done);
      if (s != KIE_OK) return s;
      g0 = reinterpret_cast<const int32_t*>(c->h_io + kStatusBytes)[0];
    } else {
      s = launch(c, n, 0, ids, true, 0, n - 1, &done);
      if (s != KIE_OK) return s;
      g0 = reinterpret_cast<const int32_t*>(c->h_io + kStatusBytes)[n - 1];
    }
    KIE_CUDA(c, cudaEventRecord(c->pf_ev1, c->stream));
    KIE_CUDA(c, cudaEventSynchronize(c->pf_ev1));
    float pms = 0.f;
    cudaEventElapsedTime(&pms, c->pf_ev0, c->pf_ev1);
    c->stats.last_prefill_ms = pms;
    c->stats.last_prefill_batched = batched ? 1 : 0;
    c->fed.assign(ids, ids + n);
    c->pos = n;
    c->next_tok = g0;
    c->primed = true;
    if (first_id) *first_id = g0;
    c->stats.pos = c->pos;
    return KIE_OK;
  });
}

static kie_status decode_impl(kie_ctx* c, int32_t n, const int32_t* forced_ids,
                              int32_t* out_ids, int32_t* n_out) {
  return kie::no_throw([&]() -> kie_status {
    kie_status s = usable(c);
    if (s != KIE_OK) return s;
    if (n_out) *n_out = 0;
    if (n < 0) return set_err(c, KIE_ERR_INVALID_ARG, "n_steps < 0");
    if (!c->primed) return set_err(c, KIE_ERR_STATE, "decode before prefill");
    if (n == 0) return KIE_OK;
    if (!out_ids && !forced_ids) return set_err(c, KIE_ERR_INVALID_ARG, "out_ids is NULL");
    if ((long long)c->pos + n > c->desc.max_seq)
      return set_err(c, KIE_ERR_CAPACITY, "decode would pass max_seq positions");
    if (forced_ids)
      for (int i = 0; i < n; ++i)
        if (forced_ids[i] < 0 || forced_ids[i] >= c->desc.vocab)
          return set_err(c, KIE_ERR_INVALID_ARG, "forced id out of range");
    int done = 0;
    s = launch(c, n, c->pos, forced_ids, forced_ids != nullptr, c->next_tok, 0, &done);
    if (s != KIE_OK) return s;
    const int32_t* picks = reinterpret_cast<const int32_t*>(c->h_io + kStatusBytes);
    if (out_ids) std::memcpy(out_ids, picks, sizeof(int32_t) * done);
    for (int i = 0; i < done; ++i) {
      c->fed.push_back(forced_ids ? forced_ids[i] : (i == 0 ? c->next_tok : picks[i - 1]));
    }
    c->pos += done;
    if (done > 0) c->next_tok = picks[done - 1];
    if (n_out) *n_out = done;
    c->stats.pos = c->pos;
    return KIE_OK;
  });
}

kie_status kie_decode(kie_ctx* c, int32_t n, int32_t* out_ids, int32_t* n_out) {
  return decode_impl(c, n, nullptr, out_ids, n_out);
}

kie_status kie_decode_forced(kie_ctx* c, const int32_t* ids, int32_t n, int32_t* out_ids) {
  return kie::no_throw([&]() -> kie_status {
    if (c && n > 0 && !ids) return set_err(c, KIE_ERR_INVALID_ARG, "ids is NULL");
    std::vector<int32_t> tmp;
    if (!out_ids && n > 0) {
      tmp.resize(n);
      out_ids = tmp.data();
    }
    return decode_impl(c, n, ids, out_ids, nullptr);
  });
}

kie_status kie_rewind(kie_ctx* c, int32_t pos) {
  kie_status s = usable(c);
  if (s != KIE_OK) return s;
  if (!c->primed) return set_err(c, KIE_ERR_STATE, "rewind before prefill");
  if (pos < 1 || pos > c->pos) return set_err(c, KIE_ERR_INVALID_ARG, "rewind out of range");
  if (pos < c->pos) {
    c->next_tok = c->fed[pos];
    c->fed.resize(pos);
    c->pos = pos;
  }
  c->stats.pos = c->pos;
  return KIE_OK;
}

kie_status kie_set_logits_capture(kie_ctx* c, float* dev_logits, int32_t rows) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (dev_logits && rows < 1) return set_err(c, KIE_ERR_INVALID_ARG, "capacity_rows < 1");
  c->capture = dev_logits;
  c->capture_rows = dev_logits ? rows : 0;
  return KIE_OK;
}

static_assert(KIE_MAX_EOS_IDS == kie::kMaxEosIds, "EOS id set size");

kie_status kie_set_sampling(kie_ctx* c, float temperature, uint64_t seed) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (!std::isfinite(temperature) || temperature < 0.f)
    return set_err(c, KIE_ERR_INVALID_ARG, "temperature must be finite and >= 0");
  // Below 1e-20 the scaled logits would leave the fp32 range the kernel
  // compares in, and the draw is the greedy pick anyway (T -> 0 limit).
  c->temperature = temperature < 1e-20f ? 0.0 : (double)temperature;
  c->seed = seed;
  return KIE_OK;
}

static_assert(KIE_MAX_TOP_K == kie::kMaxTopK, "top-k bound");

kie_status kie_set_sampling_filter(kie_ctx* c, int32_t top_k, float top_p) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (top_k < 0 || top_k > KIE_MAX_TOP_K)
    return set_err(c, KIE_ERR_INVALID_ARG, "top_k must be in 0 .. KIE_MAX_TOP_K");
  if (!(top_p > 0.f && top_p <= 1.f))
    return set_err(c, KIE_ERR_INVALID_ARG, "top_p must be in (0, 1]");
  if (top_p < 1.f && top_k == 0)
    return set_err(c, KIE_ERR_UNSUPPORTED,
                   "top_p < 1 needs a top_k bound (1 .. KIE_MAX_TOP_K) in the kernel");
  c->top_k = top_k;
  c->top_p = (double)top_p;
  return KIE_OK;
}

kie_status kie_set_eos_ids(kie_ctx* c, const int32_t* ids, int32_t n) {
  return kie::no_throw([&]() -> kie_status {
    if (!c) return KIE_ERR_INVALID_ARG;
    if (n < 0 || n > KIE_MAX_EOS_IDS) return set_err(c, KIE_ERR_INVALID_ARG, "eos id count out of range");
    if (n > 0 && !ids) return set_err(c, KIE_ERR_INVALID_ARG, "ids is NULL");
    for (int i = 0; i < n; ++i)
      if (ids[i] < 0 || ids[i] >= c->desc.vocab)
        return set_err(c, KIE_ERR_INVALID_ARG, "eos id out of range");
    c->eos_ids.assign(ids, ids + n);
    return KIE_OK;
  });
}

kie_status kie_quantize_e4m3(const void* W, int32_t N, int32_t K, void* codes, float* scales,
                            void* cuda_stream) {
  if (!W || !codes || !scales || N < 1 || K < 16 || K % 16) return KIE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return KIE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (kie::quantize_launch(static_cast<const __half*>(W), N, K, static_cast<unsigned char*>(codes),
                           scales, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return KIE_ERR_CUDA;
  return KIE_OK;
}

kie_status kie_gemv_f16(const void* W, const float* x, float* y, int32_t N, int32_t K,
                        int32_t iters, int32_t mode, int32_t chunk_bytes, void* stream,
                        float* ms_out, double* stats_out) {
  return kie::no_throw([&]() -> kie_status {
    if (!W || !x || (!y && mode == 1) || N < 1 || K < 256 || K % 256 || iters < 1 ||
        (mode != 0 && mode != 1) || chunk_bytes < 8192 || chunk_bytes % 512)
      return KIE_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(x)) return KIE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0, n_sm = 0, smem_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        kie::dynamic_smem_limit(&smem_optin) != cudaSuccess)
      return KIE_ERR_CUDA;
    const int grid = std::min(n_sm, N);
    // one layer whose four layer stages own no rows; the LM-head stage is W
    kie::Shape sh{1, K, 1, 1, 64, 256, N};
    std::vector<std::vector<int2>> ranges(kie::N_STAGES, std::vector<int2>(grid, make_int2(0, 0)));
    ranges[kie::ST_LM] = kie::partition(sh, grid, kie::ST_LM);
    std::vector<int2> flat;
    for (auto& v : ranges) flat.insert(flat.end(), v.begin(), v.end());
    int maxrows = 0;
    std::vector<unsigned long long> off(grid);
    size_t total = 0;
    for (int c = 0; c < grid; ++c) {
      maxrows = std::max(maxrows, ranges[kie::ST_LM][c].y - ranges[kie::ST_LM][c].x);
      off[c] = total;
      total += (size_t)(ranges[kie::ST_LM][c].y - ranges[kie::ST_LM][c].x) * K * 2;
    }
    kie::SmemLayout L{};
    L.xs_bytes = (K * 4 + 127) / 128 * 128;
    L.rowacc_rows = kie::result_slots(maxrows, K / kie::kPieceElems, chunk_bytes);
    L.resid_rows = 0;
    const int rowacc_bytes = (L.rowacc_rows * 4 + 127) / 128 * 128;
    const int bars = 2 * kie::kRingBars * 8;
    const int fixed = bars + L.xs_bytes + rowacc_bytes + kie::kEngineMisc;
    const int ring = (smem_optin - fixed) / 512 * 512;
    if (ring < 2 * chunk_bytes) return KIE_ERR_UNSUPPORTED;
    L.ring_off = 0;
    L.bar_off = ring;
    L.xs_off = L.bar_off + bars;
    L.rowacc_off = L.xs_off + L.xs_bytes;
    L.misc_off = L.rowacc_off + rowacc_bytes;
    L.total = L.misc_off + kie::kEngineMisc;

    int2* d_ranges = nullptr;
    DevStatus* d_status = nullptr;
    unsigned long long* d_stats = nullptr;
    unsigned long long* d_off = nullptr;
    unsigned char* d_packed = nullptr;
    LayerW* d_layer = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    kie_status ret = KIE_OK;
    if (cudaMalloc(&d_ranges, sizeof(int2) * flat.size()) != cudaSuccess ||
        cudaMalloc(&d_status, sizeof(DevStatus)) != cudaSuccess ||
        cudaMalloc(&d_stats, sizeof(unsigned long long) * kie::kStatsPerCta * grid) != cudaSuccess ||
        cudaMalloc(&d_off, sizeof(unsigned long long) * grid) != cudaSuccess ||
        cudaMalloc(&d_packed, total) != cudaSuccess ||
        cudaMalloc(&d_layer, sizeof(LayerW)) != cudaSuccess ||
        cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
      ret = KIE_ERR_CUDA;
    }
    MonoParams p{};
    if (ret == KIE_OK) {
      p.L = 1;
      p.d = K;
      p.H = 1;
      p.KV = 1;
      p.hd = 64;
      p.F = 256;
      p.V = N;
      p.G = 1;
      p.layers = d_layer;
      p.lm_head = static_cast<const __half*>(W);
      p.ranges = d_ranges;
      p.grid = grid;
      p.ring_bytes = ring;
      p.chunk_bytes = chunk_bytes;
      p.packed = d_packed;
      p.packed_off = d_off;
      p.sm = L;
      p.status = d_status;
      p.cta_stats = d_stats;
      p.timeout_ns = 2000000000LL;
      p.poll_ns = 128;
      p.fault_cta = -1;
      if (cudaMemcpyAsync(d_ranges, flat.data(), sizeof(int2) * flat.size(),
                          cudaMemcpyHostToDevice, st) != cudaSuccess ||
          cudaMemcpyAsync(d_off, off.data(), sizeof(unsigned long long) * grid,
                          cudaMemcpyHostToDevice, st) != cudaSuccess ||
          cudaMemsetAsync(d_status, 0, sizeof(DevStatus), st) != cudaSuccess ||
          cudaMemsetAsync(d_stats, 0, sizeof(unsigned long long) * kie::kStatsPerCta * grid, st) !=
              cudaSuccess ||
          cudaMemsetAsync(d_layer, 0, sizeof(LayerW), st) != cudaSuccess ||
          kie::repack_launch(p, d_packed, st) != cudaSuccess ||
          kie::gemv_configure() != cudaSuccess || cudaEventRecord(e0, st) != cudaSuccess ||
          kie::gemv_launch(p, mode, x, y, iters, grid, L.total, st) != cudaSuccess ||
          cudaEventRecord(e1, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
        ret = KIE_ERR_CUDA;
    }
    if (ret == KIE_OK) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, e0, e1);
      if (ms_out) *ms_out = ms;
      DevStatus hs{};
      cudaMemcpy(&hs, d_status, sizeof hs, cudaMemcpyDeviceToHost);
      if (hs.code != kie::DEV_OK) ret = hs.code == kie::DEV_TIMEOUT ? KIE_ERR_TIMEOUT : KIE_ERR_PROTOCOL;
      if (stats_out) {
        std::vector<unsigned long long> h((size_t)kie::kStatsPerCta * grid);
        cudaMemcpy(h.data(), d_stats, sizeof(unsigned long long) * h.size(), cudaMemcpyDeviceToHost);
        double stream = 0, prod = 0;
        for (int c = 0; c < grid; ++c) {
          stream += (double)h[(size_t)kie::kStatsPerCta * c + 2];
          prod += (double)h[(size_t)kie::kStatsPerCta * c + 3];
        }
        stats_out[0] = stream / grid;
        stats_out[1] = prod / grid;
        stats_out[2] = grid;
        stats_out[3] = ring;
      }
    }
    cudaFree(d_ranges);
    cudaFree(d_status);
    cudaFree(d_stats);
    cudaFree(d_off);
    cudaFree(d_packed);
    cudaFree(d_layer);
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    return ret;
  });
}

kie_status kie_set_trace(kie_ctx* c, uint64_t* dev_buf, int32_t capacity, int32_t cta) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (dev_buf && (capacity < 1 || cta < -1 || cta >= c->grid))
    return set_err(c, KIE_ERR_INVALID_ARG, "bad trace buffer or CTA");
  const int per = c->desc.n_layers * kie::kTracePerLayer + 4;
  c->trace = reinterpret_cast<unsigned long long*>(dev_buf);
  c->trace_cta = cta;
  c->trace_steps = dev_buf ? capacity / (per * (cta < 0 ? c->grid : 1)) : 0;
  return KIE_OK;
}

kie_status kie_set_option(kie_ctx* c, kie_option opt, int64_t v) {
  return kie::no_throw([&]() -> kie_status {
    if (!c) return KIE_ERR_INVALID_ARG;
    switch (opt) {
      case KIE_OPT_TIMEOUT_NS:
        if (v < 1000) return KIE_ERR_INVALID_ARG;
        c->timeout_ns = v;
        return KIE_OK;
      case KIE_OPT_CHUNK_BYTES: {
        if (c->failed) return set_err(c, KIE_ERR_STATE, "context failed earlier; destroy it");
        if (v < 8192 || v % 512 || v > (1 << 20)) return KIE_ERR_INVALID_ARG;
        int smem_optin = 0;
        if (kie::dynamic_smem_limit(&smem_optin) != cudaSuccess)
          return set_err(c, KIE_ERR_CUDA, "device attribute query failed");
        kie::SmemLayout sm{};
        int ring = 0;
        if (!kie::plan_smem(c->shape, c->grid, (int)v, smem_optin, c->hranges, &sm, &ring))
          return set_err(c, KIE_ERR_UNSUPPORTED, "chunk size does not fit shared memory");
        int per_sm = 0;
        if (kie::mono_configure(c->desc.head_dim, sm.total, &per_sm) != cudaSuccess || per_sm < 1)
          return set_err(c, KIE_ERR_UNSUPPORTED, "kernel does not fit with this chunk size");
        c->chunk_bytes = (int)v;
        c->sm = sm;
        c->ring_bytes = ring;
        c->smem = sm.total;
        c->stats.ring_bytes = ring;
        c->stats.chunk_bytes = (int)v;
        c->stats.smem_bytes = sm.total;
        return repack(c);
      }
      case KIE_OPT_MIN_SPLIT_LEN:
        if (v < 1 || v > (1 << 20)) return KIE_ERR_INVALID_ARG;
        c->min_split_len = (int)v;
        return KIE_OK;
      case KIE_OPT_TRACE_CLOCK:
        c->trace_clock = v ? 1 : 0;
        return KIE_OK;
      case KIE_OPT_POLL_BACKOFF_NS:
        if (v < 0 || v > 100000) return KIE_ERR_INVALID_ARG;
        c->poll_ns = (unsigned)v;
        return KIE_OK;
      case KIE_OPT_BATCHED_PREFILL:
        if (v != 0 && v != 1) return KIE_ERR_INVALID_ARG;
        c->batched_prefill = (int)v;
        return KIE_OK;
      case KIE_OPT_TMEM_PARK:
        if (v != 0 && v != 1) return KIE_ERR_INVALID_ARG;
        c->tmem_park = (int)v;
        return KIE_OK;
      case KIE_OPT_WEIGHT_FP8: {
        if (c->failed) return set_err(c, KIE_ERR_STATE, "context failed earlier; destroy it");
        if (v != 0 && v != 1) return KIE_ERR_INVALID_ARG;
        if ((int)v == c->w8) return KIE_OK;
        c->w8 = (int)v;
        const kie_status st = repack(c);
        if (st != KIE_OK) c->failed = true;
        return st;
      }
      case KIE_OPT_L2_PREFETCH_BYTES:
        if (v < 0 || v % 512 || v > (16 << 20)) return KIE_ERR_INVALID_ARG;
        c->l2_prefetch = v;
        return KIE_OK;
      case KIE_OPT_FAULT_CTA: c->fault_cta = (int)v; return KIE_OK;
      case KIE_OPT_FAULT_STEP: c->fault_step = (int)v; return KIE_OK;
      case KIE_OPT_FAULT_LAYER: c->fault_layer = (int)v; return KIE_OK;
      case KIE_OPT_FAULT_STAGE: c->fault_stage = (int)v; return KIE_OK;
    }
    return KIE_ERR_INVALID_ARG;
  });
}

kie_status kie_get_stats(const kie_ctx* cc, kie_stats* out) {
  if (!cc || !out) return KIE_ERR_INVALID_ARG;
  kie_ctx* c = const_cast<kie_ctx*>(cc);
  *out = c->stats;
  if (c->stats.launches > 0 && c->cta_stats) {
    const int K = kie::kStatsPerCta;
    std::vector<unsigned long long> st((size_t)K * c->grid);
    if (cudaMemcpy(st.data(), c->cta_stats, sizeof(unsigned long long) * st.size(),
                   cudaMemcpyDeviceToHost) == cudaSuccess) {
      double loop = 0, sync = 0, stream = 0, prod = 0, mx = 0;
      for (int i = 0; i < c->grid; ++i) {
        loop += (double)st[K * i];
        sync += (double)st[K * i + 1];
        stream += (double)st[K * i + 2];
        prod += (double)st[K * i + 3];
        if (st[K * i] > 0) mx = std::max(mx, (double)st[K * i + 1] / (double)st[K * i]);
      }
      out->loop_cycles = loop / c->grid;
      out->sync_wait_cycles = sync / c->grid;
      out->stream_wait_cycles = stream / c->grid;
      out->producer_wait_cycles = prod / c->grid;
      out->sync_wait_max_frac = mx;
    }
  }
  return KIE_OK;
}

const char* kie_status_str(kie_status s) {
  switch (s) {
    case KIE_OK: return "ok";
    case KIE_ERR_INVALID_ARG: return "invalid argument";
    case KIE_ERR_UNSUPPORTED: return "unsupported shape";
    case KIE_ERR_CUDA: return "CUDA error";
    case KIE_ERR_CAPACITY: return "KV cache capacity exceeded";
    case KIE_ERR_STATE: return "invalid state";
    case KIE_ERR_TIMEOUT: return "device wait timed out";
    case KIE_ERR_PROTOCOL: return "device protocol violation";
    case KIE_ERR_TOO_LARGE: return "size exceeds the fixed scratch of the no-allocation entry point";
    case KIE_ERR_HOST_MEMORY: return "host memory allocation failed";
  }
  return "unknown status";
}

const char* kie_last_error(const kie_ctx* c) { return c ? c->err.c_str() : ""; }

kie_status kie_destroy(kie_ctx* c) {
  if (!c) return KIE_ERR_INVALID_ARG;
  if (c->stream) cudaStreamSynchronize(c->stream);
  free_all(c);
  delete c;
  return KIE_OK;
}

}  // extern "C"
