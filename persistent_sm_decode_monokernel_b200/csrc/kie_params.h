// Parameters shared by the host side (kie_host.cu) and the persistent
// decode kernel (kie_kernel.cu).  Plain data only.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace kie {

// GEMV stages of one decoder layer plus the LM head.  The attention stage
// has no weight stream and is not listed here.
enum Stage : int { ST_QKV = 0, ST_O = 1, ST_GU = 2, ST_DOWN = 3, ST_LM = 4, N_STAGES = 5 };

constexpr int kConsumerWarps = 8;            // warps that compute (8 or 16)
constexpr int kConsumerThreads = kConsumerWarps * 32;
// + one producer warpgroup (only its first lane works): warpgroup-granular
// register split.  The launch gives every thread kRegsLaunch registers
// (all warps of the CTA fit one SM); the producer warpgroup then gives
// registers back down to kRegsProducer and the consumer warpgroups take
// kRegsConsumer, within the launch's total.
constexpr int kThreads = kConsumerThreads + 128;
constexpr int kRegsLaunch = kConsumerWarps == 16 ? 96 : 168;
constexpr int kRegsConsumer = kConsumerWarps == 16 ? 112 : 216;
constexpr int kRegsProducer = kConsumerWarps == 16 ? 24 : 56;
static_assert(kConsumerWarps * kRegsConsumer + 4 * kRegsProducer <=
                  (kConsumerWarps + 4) * kRegsLaunch,
              "register split exceeds the launch's registers");
static_assert((kConsumerWarps + 4) * 32 * kRegsLaunch <= 65536, "launch registers");
constexpr int kPieceElems = 256;             // one warp pass: 32 lanes x 8 weights
constexpr int kPieceBytes = kPieceElems * 2;   // an fp16 piece (16 bytes a lane)
// Bytes of a piece in the packed stream: fp16 weights, or fp8 E4M3 (8 bytes
// a lane).
__host__ __device__ constexpr int piece_bytes(int w8) { return w8 ? kPieceElems : kPieceBytes; }
constexpr int kRingBars = 32;                // mbarrier pairs of the byte ring (power of 2)
// Tensor-memory columns (32-bit, of its own 32 lanes) each consumer warp
// parks weight chunks in: 8 warps x 32 lanes x 256 columns = all 256 KB.
constexpr int kParkCols = 256;
static_assert(kConsumerWarps == 8 && kParkCols * 2 == 512, "tensor-memory split");
constexpr int kMaxGroup = 8;                 // heads per KV head handled by one CTA
constexpr int kAttnBlock = 256;              // positions per attention block
constexpr int kMaxSplitCombine = 96;         // most attention splits of one KV head
// per-CTA counters: loop cycles, sync-wait cycles, stream-wait cycles,
// producer slot-wait cycles, steps done, spare
constexpr int kStatsPerCta = 8;
// stage-trace stamps per layer (the LM head adds 4 per step)
constexpr int kTracePerLayer = 24;
// KV cache rows carry kKvPad unused fp16 elements after the hd values, so a
// run of rows lands in shared memory (one bulk copy) at a stride whose 8
// consecutive rows fall in 8 different bank groups.
constexpr int kKvPad = 8;
// Bytes of the attention combine's scratch per query head of a group (the
// (m, l) of up to kMaxSplitCombine splits and their o/l slices): 96 * 24.
constexpr int kCombineBytesPerHead = 2304;
// Shared-memory scratch words before the residual rows: per-warp partial
// sums and reductions, flags (kMiscHead floats).  The standalone GEMV
// engine's scratch (no residual rows) adds the per-stage GEMV plans.
constexpr int kMiscHead = 192;
constexpr int kEngineMisc = 1152;
// Most ids of the set that ends a decode (end-of-sequence ids).
constexpr int kMaxEosIds = 8;
// Top-k / top-p sampling: largest k, and how many entries of every CTA's
// local top-k list each CTA copies to shared memory for the merge (deeper
// entries are fetched from global memory when a merge reaches them).
constexpr int kMaxTopK = 64;
constexpr int kFilterHeads = 8;
// Shared-memory bytes of the top-k / top-p selection for a CTA with `rows`
// vocabulary rows in a grid of `grid` CTAs (it reuses the GEMV input area).
constexpr int filter_smem_bytes(int rows, int grid) {
  return 8 * (rows + 2 * kMaxTopK + grid * kFilterHeads + 2);
}

// Device status word block (library scratch, zeroed before each launch).
struct DevStatus {
  unsigned int code;   // 0 ok, 1 timeout, 2 protocol
  int cta, step, layer, stage, where;
  int n_done;          // forward passes finished (written by CTA 0)
  int pad;
};
enum : unsigned int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_PROTOCOL = 2 };

struct LayerW {
  const __half *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *wg, *wu, *wd;
};

// Shared-memory carve-up of one CTA (byte offsets from the dynamic base).
struct SmemLayout {
  int ring_off, bar_off, xs_off, rowacc_off, misc_off, total;
  int xs_bytes, rowacc_rows, resid_rows;
};

struct MonoParams {
  // model
  int L, d, H, KV, hd, F, V, G;
  float eps;
  int max_seq;
  int n_eos;               // a picked id equal to one of eos_ids[0 .. n_eos) ends the decode
  int eos_ids[kMaxEosIds];
  // token selection: greedy argmax (sample == 0), or the argmax of
  // logit * inv_temp + Gumbel noise from Philox4x64-10 keyed by seed
  int sample;
  double inv_temp;
  unsigned long long seed;
  // restriction of the draw (sample != 0): the top_k largest logits (0 =
  // none), then of those the shortest prefix by probability whose mass
  // reaches top_p (1 = none; top_p < 1 needs top_k >= 1)
  int top_k;
  double top_p;
  unsigned long long* cands;  // [grid][kMaxTopK][2] tagged words: every CTA's local top-k keys
  // weight format of the packed stream: 0 fp16; 1 fp8 E4M3 with one fp32
  // scale per row (weight = scale * value(code))
  int w8;
  const float* wscale;                    // row scales, each CTA's in its stream order
  const unsigned long long* wscale_off;   // [grid] offset (in floats) of each CTA's scales
  // weights (device)
  const LayerW* layers;
  const __half* tok_emb;
  const __half* final_norm;
  const __half* lm_head;
  __half* kv;              // [L][2][KV][max_seq][hd]
  const float2* rope;      // [max_seq][hd/2] (cos, sin)
  // plan
  const int2* ranges;      // [N_STAGES][grid] unit range per CTA
  int grid;
  int ring_bytes, chunk_bytes;   // byte ring size; largest chunk (one bulk copy)
  const unsigned char* packed;   // library copy of the weight matrices in stream order
  const unsigned long long* packed_off;  // [grid] byte offset of each CTA's stream
  int max_split, min_split_len;
  SmemLayout sm;
  // scratch (tagged 64-bit words: high 32 bits = epoch tag, low = fp32 bits)
  unsigned long long *x_attn, *x_ffn, *hbuf, *qbuf, *kvnew, *obuf, *slots;
  unsigned long long* partials;  // [grid][G][2 + hd/2] tagged words: m, l, o/l as fp16 pairs
  // run
  int n_steps, pos0, first_tok;
  const int* forced;       // [n_steps] or null
  int lm_from;
  unsigned int e0;
  float* capture;
  int capture_rows;
  int* out_ids;
  DevStatus* status;
  unsigned long long* cta_stats;  // [grid][kStatsPerCta]
  long long timeout_ns;
  unsigned poll_ns;        // sleep between re-polls of tagged words
  long long l2_prefetch;   // weight-stream bytes kept requested into L2 ahead of the copies
  int tmem_park;           // 1: waiting consumer warps park landed GEMV chunks in tensor memory
  unsigned long long* trace;  // stage timestamps of CTA trace_cta, or null
  int trace_cta, trace_steps;
  int trace_clock;         // 1: stamps are SM cycles (clock64), 0: %globaltimer ns
  int fault_cta, fault_step, fault_layer, fault_stage;
};

}  // namespace kie
