/*
 * kie.h -- C ABI of the batch-1 decode monokernel library (libkie.so).
 *
 * The library runs batch-1 autoregressive decode of a dense
 * decoder-only transformer as ONE persistent CUDA kernel per call: every
 * layer and every token step (RMSNorm, QKV GEMV, RoPE, KV-cache append,
 * attention over the cache, O projection, SwiGLU FFN GEMVs, LM-head GEMV,
 * argmax, EOS check) runs inside the resident kernel with no per-op launch
 * and no host round-trip.  This is the "monokernel" of revietech.ru, "Kog
 * выжимает максимум из GPU: 3000 токенов/с", section "Что такое monokernel":
 * one resident program for prefill, decode, LM-head token selection and the
 * EOS check, without returning to the CPU and without a launch per token.
 * The projections are matrix-vector products on the vector ALUs, not tensor
 * cores (same page, section "Архитектура и особенности", "GEMV вместо GEMM").
 * Token selection is greedy (argmax, lowest index on ties) by default, or
 * temperature sampling inside the kernel (kie_set_sampling); a set of up to
 * KIE_MAX_EOS_IDS ids ends a decode (kie_set_eos_ids).
 *
 * Model (pre-norm decoder; the pages never print the block, this is the
 * reading the library implements):
 *   h = E[tok];  per layer:  a = RMSNorm(h; g_attn);  q,k,v = Wq a, Wk a, Wv a;
 *   RoPE on q and k (pairs (i, i+hd/2), angle pos*base^(-2i/hd), 0-based pos);
 *   K,V appended to the cache;  o_h = softmax(q_h K_j^T / sqrt(hd)) V_j over
 *   positions 0..pos with j = h / (n_heads / n_kv_heads);  h += Wo o;
 *   b = RMSNorm(h; g_ffn);  h += Wd (silu(Wg b) * (Wu b));
 *   logits = Wlm RMSNorm(h; g_final);  next = argmax(logits).
 *   RMSNorm(x; g) = g * x / sqrt(mean(x^2) + eps).  No biases, untied head.
 *
 * Data layout and ownership
 *   - All weights are fp16, row-major [out][in] (row r of W holds the
 *     weights of output r); norm gains are fp16 [d_model].  Wq rows
 *     h*hd .. h*hd+hd-1 belong to query head h, Wk/Wv rows likewise to KV
 *     head j, Wo columns follow the same head order.  Shapes:
 *       tok_emb, lm_head [vocab][d_model]; wq [n_heads*hd][d_model];
 *       wk, wv [n_kv_heads*hd][d_model]; wo [d_model][n_heads*hd];
 *       w_gate, w_up [ffn_dim][d_model]; w_down [d_model][ffn_dim].
 *     Every pointer must be device memory, 16-byte aligned.
 *   - The KV cache is one device buffer of kie_kv_cache_bytes() bytes,
 *     16-byte aligned, laid out fp16 [n_layers][2][n_kv_heads][max_seq][hd + 8]
 *     (index 0 = K after RoPE, 1 = V; the last 8 elements of each position's
 *     row are padding, never read, so that consecutive rows copied into
 *     shared memory fall in different banks).
 *   - The CALLER owns the weights and the KV cache.  kie_create copies the
 *     weight matrices (wq..w_down, lm_head) into a library-owned buffer laid
 *     out in the order each CTA streams them, so that every streamed chunk
 *     is one contiguous bulk copy; after kie_create the library reads only
 *     tok_emb and the norm gains from the caller (these must stay valid and
 *     unmodified until kie_destroy), and the caller's matrices are read
 *     again by the batched prefill (KIE_OPT_BATCHED_PREFILL, on by default
 *     for fp16 streams), KIE_OPT_CHUNK_BYTES and KIE_OPT_WEIGHT_FP8.  The KV cache must stay valid until
 *     kie_destroy.  The library owns the packed copy and its scratch
 *     (activation words, attention partials, the RoPE table, id buffers),
 *     allocated in kie_create and freed in kie_destroy.
 *
 * Errors
 *   Every call returns a kie_status; nothing is thrown across the ABI.
 *   Calls are synchronous: they return after the device work they enqueue
 *   on the context's stream has finished.  Device-side waits are bounded:
 *   a wait that exceeds the timeout (KIE_OPT_TIMEOUT_NS) makes the kernel
 *   exit and the call return KIE_ERR_TIMEOUT.  After KIE_ERR_TIMEOUT,
 *   KIE_ERR_PROTOCOL or KIE_ERR_CUDA from a launch the context is failed:
 *   every later call except kie_destroy, kie_get_stats and kie_last_error
 *   returns KIE_ERR_STATE.  A context is not thread-safe; use one per host
 *   thread.
 */
#ifndef KIE_H
#define KIE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KIE_API __attribute__((visibility("default")))
#else
#define KIE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KIE_OK = 0,
  KIE_ERR_INVALID_ARG = 1,  /* NULL pointer, bad size, misaligned pointer */
  KIE_ERR_UNSUPPORTED = 2,  /* shape the kernel does not handle (see kie_check_desc) */
  KIE_ERR_CUDA = 3,         /* a CUDA runtime call failed (kie_last_error has the text) */
  KIE_ERR_CAPACITY = 4,     /* the call would write past max_seq positions */
  KIE_ERR_STATE = 5,        /* decode before prefill, or the context is failed */
  KIE_ERR_TIMEOUT = 6,      /* a device-side wait gave up (bounded spin) */
  KIE_ERR_PROTOCOL = 7,     /* a device-side consistency check failed */
  KIE_ERR_TOO_LARGE = 8,    /* larger than the fixed scratch of kie_gemv_f16_noalloc */
  KIE_ERR_HOST_MEMORY = 9   /* a host allocation failed (no C++ exception crosses the ABI) */
} kie_status;

/* Model shape.  Supported: head_dim 64 or 128; n_heads a multiple of
 * n_kv_heads with n_heads/n_kv_heads <= 8; d_model, ffn_dim and
 * n_heads*head_dim multiples of 256; max_seq >= 1; eos_id in [-1, vocab). */
typedef struct {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t ffn_dim;
  int32_t vocab;
  float rope_base;
  float rms_eps;
  int32_t max_seq;   /* capacity of the KV cache in positions */
  int32_t eos_id;    /* -1: no end-of-sequence id */
} kie_model_desc;

typedef struct {
  const void *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *w_gate, *w_up, *w_down;
} kie_layer_weights;

typedef struct {
  const void *tok_emb;
  const void *final_norm;
  const void *lm_head;
  const kie_layer_weights *layers;  /* HOST array [n_layers] of device pointers;
                                       copied by kie_create */
} kie_weights;

typedef struct kie_ctx kie_ctx;

typedef struct {
  int32_t pos;              /* positions held in the KV cache */
  int32_t grid;             /* persistent CTAs (one per SM) */
  int32_t ring_bytes;       /* shared-memory weight ring per CTA */
  int32_t chunk_bytes;      /* largest weight chunk (one bulk copy) */
  int32_t smem_bytes;       /* dynamic shared memory per CTA */
  int32_t last_steps;       /* forward passes run by the last launch */
  float last_device_ms;     /* device time of the last launch (CUDA events) */
  uint64_t launches;        /* kernel launches made by this context */
  /* Per-CTA cycle counters of the last launch, averaged over CTAs, as seen
   * by consumer thread 0: cycles in the persistent loop, cycles spent
   * polling for other CTAs' outputs (the intra-kernel sync), and cycles
   * spent waiting for the weight stream to land in shared memory (for the
   * GEMV units warp 0 computes itself: each unit belongs to one warp). */
  double loop_cycles;
  double sync_wait_cycles;
  double stream_wait_cycles;
  double producer_wait_cycles; /* producer cycles waiting for a free ring slot */
  double sync_wait_max_frac;   /* max over CTAs of sync_wait/loop */
  double last_prefill_ms;      /* device time of the last kie_prefill (CUDA events) */
  int32_t last_prefill_batched; /* 1: it ran the batched tensor-core path */
} kie_stats;

typedef enum {
  KIE_OPT_TIMEOUT_NS = 1,     /* bound of every device-side wait (default 2e9) */
  KIE_OPT_CHUNK_BYTES = 2,    /* largest weight chunk -- one GEMV work unit, one bulk
                                 copy -- in bytes (>= 8192, multiple of 512;
                                 default 32768, or 16384 where two 32 KB chunks do not
                                 fit the ring); re-plans the ring and rebuilds the packed
                                 weight copy, so the caller's matrices must still be valid */
  KIE_OPT_MIN_SPLIT_LEN = 3,  /* minimum positions per attention split (default 64) */
  KIE_OPT_FAULT_CTA = 4,      /* test hook: CTA that withholds one publication (-1 off) */
  KIE_OPT_FAULT_STEP = 5,     /* test hook: step of the withheld publication */
  KIE_OPT_FAULT_LAYER = 6,    /* test hook: layer of the withheld publication */
  KIE_OPT_FAULT_STAGE = 7,    /* test hook: 0 QKV, 1 O, 2 gate/up, 3 down, 4 LM */
  KIE_OPT_POLL_BACKOFF_NS = 8, /* sleep between re-polls of another CTA's data (default 0) */
  KIE_OPT_TRACE_CLOCK = 9,     /* stage trace in SM cycles (1) instead of ns (0, default) */
  KIE_OPT_L2_PREFETCH_BYTES = 10, /* per CTA, weight-stream bytes requested into L2 ahead of
                                    the shared-memory ring (multiple of 512, <= 16 MiB;
                                    0 = off, the default) */
  KIE_OPT_WEIGHT_FP8 = 11,     /* 1: stream the weight matrices as FP8 E4M3 with one fp32
                                  scale per row (the pages' roadmap FP8 quantisation,
                                  revietech.ru, "Kog выжимает максимум из GPU: 3000
                                  токенов/с", section "Ограничения подхода"): half the
                                  bytes per token.  Each row r of Wq, Wk, Wv, Wo, W_gate,
                                  W_up, W_down and the LM head becomes s_r = max|W_r| / 448
                                  (fp32; 1 for a zero row) and the codes E4M3(W_rc / s_r)
                                  (fp32 division, round to nearest even, saturated at 448;
                                  the codes of kie_quantize_e4m3); the GEMVs multiply the
                                  codes, as fp16, with the fp16 inputs, accumulate in fp32
                                  and scale the row sums.  The embedding, norm gains, KV
                                  cache and everything else stay as they are.  0: fp16
                                  weights (the default).  Rebuilds the packed weight copy
                                  from the caller's matrices, which must still be valid */
  KIE_OPT_BATCHED_PREFILL = 12, /* 1 (default): kie_prefill runs positions 0 .. n-2 of the
                                  prompt through all layers at once -- the projections
                                  as tcgen05 tensor-core GEMMs over the positions, causal
                                  attention over the prompt, the K/V of every position
                                  written to the cache -- and the last position as one
                                  step of the decode kernel, which picks the first id.
                                  It reads the caller's fp16 weight matrices, which must
                                  then stay valid; contexts streaming FP8 weights, and
                                  0, run every position as a decode step instead */
  KIE_OPT_TMEM_PARK = 13       /* 1 (default): while a CTA's consumer warps wait for the
                                  other CTAs' outputs, each moves the weight chunks of the
                                  next GEMV that have already reached its shared-memory
                                  ring into its own 32 KB of tensor memory and frees their
                                  ring space, so the weight stream runs further ahead
                                  (fp16 streams only); 0: off */
} kie_option;

/* Bytes of the caller-provided KV cache: 2*n_layers*n_kv_heads*max_seq*(head_dim+8)*2.
 * This is MORE than the unpadded 2*n_layers*n_kv_heads*max_seq*head_dim*2 of
 * a plain [layer][K|V][kv_head][pos][head_dim] fp16 cache: every position's
 * row carries 8 unused fp16 elements (see the layout above), 3% more at
 * head_dim 128 and 6% at 64.  Size the buffer with this call, not with the
 * unpadded formula.  Returns 0 for a NULL or invalid desc.  Host only. */
KIE_API size_t kie_kv_cache_bytes(const kie_model_desc *desc);

/* Checks a shape against the limits above.  Host only, no CUDA call. */
KIE_API kie_status kie_check_desc(const kie_model_desc *desc);

/* Creates a context on the current CUDA device (the pages' resident decode
 * program, revietech.ru, "Kog выжимает максимум из GPU: 3000 токенов/с",
 * section "Что такое monokernel", set up once per model: plan, packed
 * weight stream, scratch).  `kv_cache` is the
 * caller's device buffer (kie_kv_cache_bytes bytes); `cuda_stream` is a
 * cudaStream_t (NULL = legacy default stream).  On success *out receives
 * the context; on failure *out is set to NULL. */
KIE_API kie_status kie_create(const kie_model_desc *desc, const kie_weights *weights,
                      void *kv_cache, void *cuda_stream, kie_ctx **out);

/* Prefill, the first phase the pages' resident program runs (same page and
 * section): runs the prompt through the model in one launch, writing K/V for
 * positions 0..n-1 (the session restarts at position 0), and returns in
 * *first_id the id picked (greedy or sampled, kie_set_sampling) from the
 * last position's logits.
 * prompt_ids: HOST array [n] with ids in [0, vocab).  first_id may be NULL. */
KIE_API kie_status kie_prefill(kie_ctx *ctx, const int32_t *prompt_ids, int32_t n,
                       int32_t *first_id);

/* Decode with token selection and the end-id check inside the kernel, no
 * launch per token and no return to the CPU between tokens (same page and
 * section).  Runs n_steps decode steps in ONE launch.  Step i feeds the
 * previous id (the id from kie_prefill or the last id of the previous
 * decode call for i = 0) at the next position and writes the picked id to
 * out_ids[i] (HOST array [n_steps]).  Stops after emitting an end id
 * (eos_id, or the set of kie_set_eos_ids); *n_out
 * (nullable) receives the number of ids written.  n_steps = 0 is a no-op. */
KIE_API kie_status kie_decode(kie_ctx *ctx, int32_t n_steps, int32_t *out_ids,
                      int32_t *n_out);

/* Teacher-forced decode, one launch: step i feeds ids[i] (HOST [n]) at the
 * next position instead of the previous pick, and still writes the
 * pick to out_ids[i] (HOST [n], nullable).  Afterwards the session
 * continues from the last pick.  Used to compare logits against a
 * reference on a fixed token stream. */
KIE_API kie_status kie_decode_forced(kie_ctx *ctx, const int32_t *ids, int32_t n,
                             int32_t *out_ids);

/* Moves the session back to `pos` positions (1 <= pos <= current): the
 * next decode step runs at position `pos` and feeds the id that was fed
 * (or picked) for that position.  K/V of positions >= pos are rewritten by
 * later steps.  Host-side only. */
KIE_API kie_status kie_rewind(kie_ctx *ctx, int32_t pos);

/* Logit capture (measurement / parity): while set, every launch writes the
 * fp32 logits of each step that picks an id to dev_logits[row][vocab],
 * row = index among those steps, for rows < capacity_rows.  dev_logits is a
 * device buffer owned by the caller; NULL turns capture off. */
KIE_API kie_status kie_set_logits_capture(kie_ctx *ctx, float *dev_logits,
                                  int32_t capacity_rows);

/* Stage trace (measurement): while set, CTA `cta` of every launch writes
 * %globaltimer stamps (ns) to dev_buf, a device buffer of `capacity` u64
 * owned by the caller; cta = -1 traces every CTA, laid out
 * [step][cta][slot] (grid CTAs per step, see kie_get_stats).  Per step and
 * CTA it writes n_layers*24 + 4 slots: for each
 * layer QKV begin, QKV input ready, QKV done, attention done, O input
 * ready, O done, gate/up input ready, gate/up done, down input ready, down
 * done, and (CTAs with attention work) q ready, attention math done,
 * partial published, combine done, first K/V tile landed, first block's
 * softmax done (slots 10-15); slots 16-19 and 21: ns the first consumer
 * warp waited for streamed chunks in QKV, O, gate/up, down and attention
 * (durations, not stamps); slots 22, 23, 20: when the producer started
 * issuing the layer's QKV chunks, had issued them, and had issued the
 * attention tiles; then LM-head begin, input ready, GEMV done,
 * pick known.  Steps beyond the
 * capacity are not traced.  NULL turns tracing off. */
KIE_API kie_status kie_set_trace(kie_ctx *ctx, uint64_t *dev_buf, int32_t capacity, int32_t cta);

/* Token selection (the pages' in-kernel "LM-head sampling", revietech.ru,
 * "Kog выжимает максимум из GPU: 3000 токенов/с", section "Что такое
 * monokernel"; the pages give no sampler, temperature sampling is the
 * reading taken).  temperature == 0: greedy argmax (the default).
 * temperature > 0: every step that picks an id draws it from
 * softmax(logits / temperature) inside the kernel, as the argmax over the
 * vocabulary of  logit_i / temperature + G_i,  G_i = -log(-log(U_i)), with
 *   U_i = ((w >> 11) + 0.5) * 2^-53,
 *   w   = word (i % 4) of Philox4x64-10(counter = (i / 4, t, 0, 0), key = (seed, 0))
 * (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011)
 * and t the 0-based position of the token whose logits are sampled.  A draw
 * depends only on (seed, t, logits), so kie_rewind followed by the same
 * decode reproduces it.  Applies to kie_prefill's first id, kie_decode and
 * kie_decode_forced.  0 < temperature < 1e-20 is taken as 0 (greedy, the
 * limit of the draw; the scaled logits would overflow fp32).  Returns KIE_ERR_INVALID_ARG for a NULL ctx or a
 * temperature that is negative, infinite or NaN.  Host only. */
KIE_API kie_status kie_set_sampling(kie_ctx *ctx, float temperature, uint64_t seed);

/* Restriction of the sampled draw (kie_set_sampling with temperature > 0;
 * greedy picks ignore it).  The pages name LM-head sampling without a
 * sampler (revietech.ru, "Kog выжимает максимум из GPU: 3000 токенов/с",
 * section "Что такое monokernel"); top-k and nucleus (top-p) filtering are
 * the readings taken.  top_k in 1 .. KIE_MAX_TOP_K keeps the top_k largest
 * logits of the step (ties by the lower id); top_p in (0, 1) then keeps, of
 * those, the shortest prefix ordered by probability under
 * softmax(logits / temperature) restricted to them whose mass reaches top_p
 * (computed in fp64 from the fp32 logits).  The draw is the Gumbel-max draw
 * of kie_set_sampling over the kept ids, with the same noise.  top_k = 0
 * and top_p = 1 switch the restriction off (the default).  Returns
 * KIE_ERR_INVALID_ARG for a NULL ctx, top_k outside 0 .. KIE_MAX_TOP_K or
 * top_p outside (0, 1], and KIE_ERR_UNSUPPORTED for top_p < 1 with
 * top_k = 0 (the kernel bounds the nucleus by a top-k set).  Each picking
 * step then exchanges every CTA's top_k candidates once more between the
 * CTAs.  Host only. */
#define KIE_MAX_TOP_K 64
KIE_API kie_status kie_set_sampling_filter(kie_ctx *ctx, int32_t top_k, float top_p);

/* Ids that end a decode: a step whose picked id is one of ids[0 .. n) is
 * the last one (it is written and counted in *n_out).  n = 0 goes back to
 * the model descriptor's eos_id (none if -1).  ids: HOST array, copied.
 * KIE_ERR_INVALID_ARG for a NULL ctx, n outside 0 .. KIE_MAX_EOS_IDS, a NULL
 * ids with n > 0 or an id outside [0, vocab).  Host only. */
#define KIE_MAX_EOS_IDS 8
KIE_API kie_status kie_set_eos_ids(kie_ctx *ctx, const int32_t *ids, int32_t n);

KIE_API kie_status kie_set_option(kie_ctx *ctx, kie_option opt, int64_t value);
KIE_API kie_status kie_get_stats(const kie_ctx *ctx, kie_stats *out);
KIE_API const char *kie_status_str(kie_status s);
/* Text of the last error on this context ("" if none); valid until the next call. */
KIE_API const char *kie_last_error(const kie_ctx *ctx);
/* Ends a context (the counterpart of kie_create; same page and section):
 * frees the library-owned packed weights and scratch; the caller's weights
 * and KV cache are not touched.  KIE_ERR_INVALID_ARG for NULL. */
KIE_API kie_status kie_destroy(kie_ctx *ctx);

/* The decode kernel's weight-stream GEMV engine run alone, for unit tests
 * and bandwidth measurement: y[N] = W[N][K] x[K] with W fp16 row-major and
 * x, y fp32 (all device pointers, 16-byte aligned; K a multiple of 256),
 * computed `iters` times in one launch of one CTA per SM (the rows split as
 * the LM-head stage splits the vocabulary).  mode 1 computes y; mode 0
 * only streams W through the shared-memory ring (y untouched).
 * chunk_bytes: largest streamed chunk (>= 8192, multiple of 512).  *ms_out
 * (nullable): device time of the GEMV launch.  stats_out (nullable, 4
 * doubles): mean per-CTA cycles the consumers waited for the stream, mean
 * producer cycles waiting for ring space, CTAs, ring bytes.  Allocates and
 * frees its own scratch, including a stream-ordered copy of W; synchronous
 * on `cuda_stream`. */
KIE_API kie_status kie_gemv_f16(const void *W, const float *x, float *y, int32_t N, int32_t K,
                                int32_t iters, int32_t mode, int32_t chunk_bytes,
                                void *cuda_stream, float *ms_out, double *stats_out);

/* The FP8 quantisation of KIE_OPT_WEIGHT_FP8 applied to one matrix, for
 * tests and for callers that store FP8 weights: W[N][K] fp16 row-major
 * (device, 16-byte aligned, K a multiple of 16) to codes[N][K] (device,
 * E4M3, one byte each, 16-byte aligned) and scales[N] (device, fp32), with
 * s_r = max_c |W_rc| / 448 (1 for a zero row) and codes E4M3(W_rc / s_r),
 * round to nearest even, saturated.  The caller owns all three buffers.
 * Synchronous on `cuda_stream`.  KIE_ERR_INVALID_ARG for NULL or misaligned
 * pointers or bad sizes, KIE_ERR_CUDA for a failed launch. */
KIE_API kie_status kie_quantize_e4m3(const void *W, int32_t N, int32_t K, void *codes,
                                     float *scales, void *cuda_stream);

/* Largest fp16 weight matrix (N*K*2 bytes) kie_gemv_f16_noalloc takes. */
#define KIE_NOALLOC_MAX_WEIGHT_BYTES (16u * 1024u * 1024u)

/* The GEMV of kie_gemv_f16 (mode 1, one pass, 32 KB chunks) for callers
 * that cannot allocate device memory: a process that reserved all of the
 * GPU's memory for its own pool at start-up, where cudaMalloc would fail or
 * eat into that pool, or a latency-bound loop, where cudaMalloc and
 * cudaFree synchronise the device.  The pages describe no such entry point;
 * it exists for these callers only.
 *
 * y[N] = W[N][K] x[K]: W fp16 row-major, x and y fp32, all device pointers
 * (W and x 16-byte aligned), K a multiple of 256, N >= 1, and
 * N*K*2 <= KIE_NOALLOC_MAX_WEIGHT_BYTES, else KIE_ERR_TOO_LARGE.  The caller
 * owns W, x and y.  All device scratch (the streamed copy of W, the row
 * split, the status word) lives in one fixed array compiled into the
 * library, of KIE_NOALLOC_MAX_WEIGHT_BYTES plus under 64 KB; every GPU that
 * loads the library holds it until the process exits.  The call allocates
 * no device memory.
 *
 * The first call on a device looks up the array's address on that device
 * (cudaGetSymbolAddress, which may load the library's device code there,
 * so the first call takes longer than the ones after it).  The address belongs to
 * the device's current driver context: after cudaDeviceReset, or with
 * another context made current, the next call looks it up again (so that
 * call is again a first call).  Another host thread's kie_gemv_f16 does not
 * disturb a call, but it is GPU work like any other: overlapping the two on
 * the GPU is fine, overlapping two calls of this entry point is not.  Every call clears the
 * parts of the array that must start at zero; all calls on a device share
 * the array, so calls that overlap on the GPU (two streams, two host
 * threads) race and give wrong results: serialise them.  Synchronous on
 * `cuda_stream`.  Errors: KIE_ERR_INVALID_ARG, KIE_ERR_TOO_LARGE,
 * KIE_ERR_CUDA, KIE_ERR_TIMEOUT (a bounded device wait gave up). */
KIE_API kie_status kie_gemv_f16_noalloc(const void *W, const float *x, float *y, int32_t N,
                                        int32_t K, void *cuda_stream);

/* Host-only planning query (no CUDA call): the unit range [begin, end) that
 * CTA `cta` of a `grid`-CTA launch owns in GEMV stage `stage` (0 QKV, 1 O,
 * 2 gate/up, 3 down, 4 LM head).  Units are rows, except RoPE pairs of q/k
 * rows and gate/up row pairs, which count as one unit of two rows. */
KIE_API kie_status kie_plan_units(const kie_model_desc *desc, int32_t grid, int32_t stage,
                          int32_t cta, int32_t *begin, int32_t *end);

/* Host-only planning query (no CUDA call): how CTA `cta` of a `grid`-CTA
 * decode launch splits its GEMV work in stage `stage` for KIE_OPT_CHUNK_BYTES
 * = chunk_bytes (>= 8192, multiple of 512) and fp16 (fp8 = 0) or FP8 (1)
 * weights -- the same computation the decode kernel and its weight repack
 * make.  The CTA's rows are cut into blocks of nr <= 4 rows and each row's
 * 256-weight pieces into S parts; a block's part is one work unit (one bulk
 * copy, computed by one consumer warp).  out[6] (caller-owned) receives
 * {rows, pieces per row, nr, S, blocks, result slots reserved per CTA}.
 * Errors: KIE_ERR_INVALID_ARG, or the descriptor checks of kie_check_desc. */
KIE_API kie_status kie_plan_gemv_work(const kie_model_desc *desc, int32_t grid, int32_t stage,
                                      int32_t cta, int32_t chunk_bytes, int32_t fp8,
                                      int32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* KIE_H */
