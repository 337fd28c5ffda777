// The persistent batch-1 decode kernel ("monokernel").
//
// One CTA per SM stays resident for a whole prefill or decode call and runs
// every layer of every token step: RMSNorm, QKV GEMV + RoPE + KV append,
// split-K attention over the fp16 KV cache, O projection + residual,
// gate/up GEMV + SwiGLU, down GEMV + residual, final RMSNorm + LM-head GEMV,
// argmax and the EOS test, with no launch per op and no host round-trip
// (revietech.ru, "Kog выжимает максимум из GPU: 3000 токенов/с", section
// "Что такое monokernel").  The projections are GEMVs on the FP32 pipes,
// not tensor cores: at batch 1 there is one activation column, so a tensor
// core tile would sit mostly idle (same page, "Архитектура и особенности",
// "GEMV вместо GEMM").
//
// B200 design
//  * Warp specialisation.  Warpgroup 2 is the producer (one lane works; the
//    group gives its registers to the consumers with setmaxnreg): it walks
//    the CTA's static weight schedule for the whole call and streams it
//    with cp.async.bulk into a byte ring of shared memory completed by
//    mbarriers.  The schedule does not depend on activations, so the
//    producer runs ahead across every stage boundary and keeps HBM busy
//    while the consumers wait for other CTAs.  Warps 0-7 consume: each
//    16-byte lane load of fp16 weights meets the fp16 activations held in
//    shared memory, fp16 x fp16 products accumulate in fp32, warp-shuffle
//    reductions.  Attention uses warp-level mma on fp16 tiles.
//  * Intra-kernel sync by tagged data.  Every vector a stage publishes is
//    written as 64-bit words {epoch tag, fp32 value}, stored relaxed at gpu
//    scope; consumers poll the words themselves until the tag of the
//    expected (step, layer) appears.  The data is the flag: no arrival
//    counter, no fence on the hot path, and no re-arming (tags only grow).
//    This replaces the pages' NaN-initialised buffers, which a consumer
//    polls until real data appears, in place of atomic arrival counters
//    (same page, "Что такое monokernel").  Once per step a fenced publish
//    (the argmax slots) orders the plain KV-cache stores for later steps.
//  * Every wait is bounded (%globaltimer); on expiry the CTA records the
//    error, all CTAs unwind at their next stage boundary, and the producer
//    drains its in-flight copies before exiting.
#include <cfloat>
#include <climits>
#include <cuda_runtime.h>
#include <type_traits>

#include "kie_device.cuh"
#include "kie_kernel.h"
#include "kie_params.h"
#include "kie_units.h"

namespace kie {

using u64 = unsigned long long;

namespace {

enum : int { F_ABORT = 0, F_STOP = 1, F_KVSTEP = 3 };

// The dynamic shared-memory block.  Pointers derived from it directly keep
// their address space, so the compiler emits shared-memory loads for them.
extern __shared__ __align__(128) unsigned char kie_smem[];

// The kernel's parameter block, copied to shared memory when a kernel starts:
// every function reads it with shared-memory loads, including the
// non-inlined stage functions, which could not know that a reference to the
// kernel parameter points at constant memory.
__shared__ MonoParams kie_p;
// Consumer thread 0's counters: cycles waiting for other CTAs' outputs,
// cycles waiting for the weight stream, and the ns the current stage waited
// for the stream (stage trace).
__shared__ long long kie_ctr[3];
// Ring cursors of the consumer warps, the same in every consumer thread:
// next chunk to wait for, next chunk to release (chunks are released in
// order), ring read position (mirrors the producer's placement).  Every
// consumer thread reads them at the start of a stage, after a barrier;
// consumer thread 0 writes them back after the stage's last barrier, and the
// next stage reads them only after another barrier.
__shared__ uint32_t kie_cur[3];
// (step, layer, stage) of the consumer warps, written by consumer thread 0
// only: exact for thread 0 (the stage trace), and for the other threads the
// position an error report names (possibly one stage behind).
__shared__ int kie_at[3];
// Ring read position after the last GEMV unit of a stage (written by the
// warp that computed that unit, read by thread 0 after the stage's barrier).
__shared__ uint32_t kie_ring_end;
// Tensor memory of the consumer warps (all 512 columns, allocated by warp 0
// when parking is on) and, per warp, how many of its units of the stage
// whose first chunk is kie_park_ci[w] it has parked there.
__shared__ uint32_t kie_tmem;
__shared__ int kie_park_n[kConsumerWarps];
__shared__ uint32_t kie_park_ci[kConsumerWarps];
// This CTA's row scales of an fp8 weight stream (set by setup_plans).
__shared__ const float* kie_wsc;

// Views of the dynamic shared memory, always derived from the __shared__
// symbol so that every access compiles to a shared-memory instruction.
__device__ __forceinline__ float* sm_xs(const MonoParams& p) {
  return reinterpret_cast<float*>(kie_smem + p.sm.xs_off);
}
__device__ __forceinline__ float* sm_rowacc(const MonoParams& p) {
  return reinterpret_cast<float*>(kie_smem + p.sm.rowacc_off);
}
__device__ __forceinline__ float* sm_misc(const MonoParams& p) {
  return reinterpret_cast<float*>(kie_smem + p.sm.misc_off);
}
// per-warp scratch words, kConsumerWarps each (<= 16; words 0-15 unused):
// two reductions with their indices; then flags
__device__ __forceinline__ float* sm_red(const MonoParams& p) { return sm_misc(p) + 16; }
__device__ __forceinline__ float* sm_red2(const MonoParams& p) { return sm_misc(p) + 32; }
__device__ __forceinline__ int* sm_redi(const MonoParams& p) {
  return reinterpret_cast<int*>(sm_misc(p) + 48);
}
__device__ __forceinline__ int* sm_redi2(const MonoParams& p) {
  return reinterpret_cast<int*>(sm_misc(p) + 64);
}
__device__ __forceinline__ volatile int* sm_flags(const MonoParams& p) {
  return reinterpret_cast<volatile int*>(sm_misc(p) + 80);
}
// monotonic start of the chunk on each ring barrier pair (producer only)
__device__ __forceinline__ uint32_t* sm_starts(const MonoParams& p) {
  return reinterpret_cast<uint32_t*>(sm_misc(p) + 96);
}
// ring offset of the chunk on each barrier pair, written by the producer
// before it arms the chunk's full barrier, so that a consumer that waited
// for the chunk reads it without following the placement of the chunks
// before it
__device__ __forceinline__ volatile uint32_t* sm_offs(const MonoParams& p) {
  return reinterpret_cast<volatile uint32_t*>(sm_misc(p) + 96 + kRingBars);
}
static_assert(kConsumerWarps <= 16 && 96 + 2 * kRingBars <= kMiscHead, "scratch words");
// residual stream rows this CTA owns (O / down stages)
__device__ __forceinline__ float* sm_res_attn(const MonoParams& p) { return sm_misc(p) + kMiscHead; }
__device__ __forceinline__ float* sm_res_ffn(const MonoParams& p) {
  return sm_misc(p) + kMiscHead + p.sm.resid_rows;
}

__device__ __forceinline__ StagePlan* sm_plan(const MonoParams& p) {
  return reinterpret_cast<StagePlan*>(sm_misc(p) + kMiscHead + 2 * p.sm.resid_rows);
}
__device__ __forceinline__ const unsigned char* sm_ring(const MonoParams& p) {
  return kie_smem + p.sm.ring_off;
}
// Writable view of the ring, for the consumers' fills of attention tiles
// they own (after the tile's copies have landed).
__device__ __forceinline__ unsigned char* sm_ring_w(const MonoParams& p) {
  return kie_smem + p.sm.ring_off;
}
__device__ __forceinline__ uint32_t sm_ring_s(const MonoParams& p) {
  return dev::smem_u32(kie_smem + p.sm.ring_off);
}
__device__ __forceinline__ uint32_t sm_full_s(const MonoParams& p) {
  return dev::smem_u32(kie_smem + p.sm.bar_off);
}
__device__ __forceinline__ uint32_t sm_empty_s(const MonoParams& p) {
  return sm_full_s(p) + 8 * kRingBars;
}

// ------------------------------------------------------------ stage geometry

__device__ __forceinline__ int stage_k(const MonoParams& p, int st) {
  switch (st) {
    case ST_O: return p.H * p.hd;
    case ST_DOWN: return p.F;
    default: return p.d;
  }
}

__device__ __forceinline__ int qkv_pair_units(const MonoParams& p) {
  return (p.H + p.KV) * (p.hd >> 1);
}

// pair units (RoPE pairs) inside [ub, ue) of the QKV stage
__device__ __forceinline__ int qkv_pairs_in(const MonoParams& p, int ub, int ue) {
  const int np = min(ue, qkv_pair_units(p)) - ub;
  return np > 0 ? np : 0;
}

__device__ __forceinline__ int range_rows(const MonoParams& p, int st, int ub, int ue) {
  if (st == ST_QKV) {
    const int np = qkv_pairs_in(p, ub, ue);
    return 2 * np + (ue - ub - np);
  }
  if (st == ST_GU) return 2 * (ue - ub);
  return ue - ub;
}

// Row j (0-based, in the CTA's stream order) of the CTA's share of a stage.
__device__ __forceinline__ const __half* row_ptr(const MonoParams& p, int st, const LayerW& w,
                                                 int ub, int ue, int j) {
  switch (st) {
    case ST_QKV: {
      const int half = p.hd >> 1;
      const int nqp = p.H * half;
      const int np = qkv_pairs_in(p, ub, ue);
      if (j < 2 * np) {
        int u = ub + (j >> 1);
        const int hi = j & 1;
        if (u < nqp) {
          const int h = u / half, i = u - h * half;
          return w.wq + (size_t)(h * p.hd + i + hi * half) * p.d;
        }
        u -= nqp;
        const int h = u / half, i = u - h * half;
        return w.wk + (size_t)(h * p.hd + i + hi * half) * p.d;
      }
      const int u = ub + np + (j - 2 * np);
      return w.wv + (size_t)(u - qkv_pair_units(p)) * p.d;
    }
    case ST_O: return w.wo + (size_t)(ub + j) * (p.H * p.hd);
    case ST_GU: return ((j & 1) ? w.wu : w.wg) + (size_t)(ub + (j >> 1)) * p.d;
    case ST_DOWN: return w.wd + (size_t)(ub + j) * p.F;
    default: return p.lm_head + (size_t)(ub + j) * p.d;
  }
}

// The rows and unit shape of CTA blockIdx.x's share of stage st.
__device__ __forceinline__ StagePlan stage_plan(const MonoParams& p, int st) {
  const int2 r = p.ranges[st * p.grid + blockIdx.x];
  StagePlan pl{};
  pl.rows = range_rows(p, st, r.x, r.y);
  pl.kp = stage_k(p, st) / kPieceElems;
  plan_units(pl, p.chunk_bytes, piece_bytes(p.w8), p.sm.rowacc_rows);
  return pl;
}

// The stream order of a stage's units (shared by the weight repack, the
// producer and the consumers): f(u, b, s, rows, n) receives each unit's
// index, block, part, row count and piece count; returning false stops the
// walk.
template <class F>
__device__ __forceinline__ bool for_each_unit(const StagePlan& pl, F&& f) {
  int u = 0;
  for (int b = 0; b < pl.nb; ++b) {
    const int rows = pl.block_rows(b);
    for (int s = 0; s < pl.S; ++s, ++u)
      if (!f(u, b, s, rows, pl.count(s))) return false;
  }
  return true;
}

// Fills the stage plans in shared memory (threads 0..N_STAGES-1; the caller
// synchronises) and thread 0 the fp8 row-scale pointer.
__device__ __forceinline__ void setup_plans(const MonoParams& p) {
  const int tid = (int)threadIdx.x;
  if (tid < N_STAGES) {
    const int st = tid;
    StagePlan pl = stage_plan(p, st);
    // row-scale positions of an fp8 stream (per layer: QKV, O, gate/up,
    // down rows; then the LM head after all layers)
    int before = 0, layer_rows = 0;
    for (int s2 = ST_QKV; s2 <= ST_DOWN; ++s2) {
      const int2 r2 = p.ranges[s2 * p.grid + blockIdx.x];
      const int n2 = range_rows(p, s2, r2.x, r2.y);
      if (s2 < st) before += n2;
      layer_rows += n2;
    }
    pl.rows_layer = layer_rows;
    pl.sbase = st == ST_LM ? p.L * layer_rows : before;
    sm_plan(p)[st] = pl;
  }
  if (tid == 0) kie_wsc = p.w8 ? p.wscale + p.wscale_off[blockIdx.x] : nullptr;
}

// Whether waiting consumer warps park GEMV chunks in tensor memory.
__device__ __forceinline__ bool parking(const MonoParams& p) { return p.tmem_park && !p.w8; }

// Byte ring placement shared by producer and consumers: a chunk goes right
// after the previous one, or back to offset 0 when it would not fit.
__device__ __forceinline__ uint32_t ring_place(uint32_t& wend, uint32_t sz, uint32_t ring_bytes) {
  const uint32_t off = (wend + sz <= ring_bytes) ? wend : 0u;
  wend = off + sz;
  return off;
}

// This CTA's attention work item at position pos: KV head j, positions
// [t0, t1) of 0..pos.  Items are (KV head, split) pairs, item = CTA index.
struct AttnItem {
  int j, s, t0, t1, nsplit;   // KV head, split index, positions [t0, t1), splits of head j
  bool valid;
};
__device__ __forceinline__ AttnItem attn_item(const MonoParams& p, int pos) {
  const int n_pos = pos + 1;
  int nsplit = (n_pos + p.min_split_len - 1) / p.min_split_len;
  if (nsplit > p.max_split) nsplit = p.max_split;
  AttnItem a;
  a.nsplit = nsplit;
  const int it = blockIdx.x;
  a.valid = it < p.KV * nsplit;
  a.j = it / nsplit;
  const int s = it - a.j * nsplit;
  a.s = s;
  a.t0 = (int)(((long long)s * n_pos) / nsplit);
  a.t1 = (int)(((long long)(s + 1) * n_pos) / nsplit);
  return a;
}
// Attention K/V tiles in the ring: rows of hd fp16 at the cache's padded
// stride of hd + kKvPad elements, so that the 8 rows an mma fragment load
// touches fall in 8 different bank groups.
__device__ __forceinline__ int attn_row_stride(const MonoParams& p) { return (p.hd + kKvPad) * 2; }
// Positions per attention block (one K tile and one V tile in the ring), a
// multiple of 16.
__device__ __forceinline__ int attn_block(const MonoParams& p) {
  return max(16, min(kAttnBlock, p.chunk_bytes / attn_row_stride(p)) & ~15);
}
__device__ __forceinline__ const __half* kv_rows(const MonoParams& p, int layer, int kv, int j) {
  return p.kv + (((size_t)layer * 2 + kv) * p.KV + j) * (size_t)p.max_seq * (p.hd + kKvPad);
}

__device__ __forceinline__ unsigned epoch_of(const MonoParams& p, int step, int layer) {
  return p.e0 + (unsigned)step * (unsigned)(p.L + 1) + (unsigned)layer + 1u;
}

__device__ __forceinline__ void raise_error(const MonoParams& p, unsigned code, int step,
                                            int layer, int stage, int where) {
  if (atomicCAS(&p.status->code, 0u, code) == 0u) {
    p.status->cta = blockIdx.x;
    p.status->step = step;
    p.status->layer = layer;
    p.status->stage = stage;
    p.status->where = where;
  }
}

__device__ __forceinline__ bool global_error(const MonoParams& p) {
  return dev::ld_relaxed_u32(&p.status->code) != 0u;
}

// ----------------------------------------------------------------- producer

// Runs inlined in the kernel body (no stack object): `p` is the kernel
// parameter itself, whose fields compile to constant-bank operands.
struct Producer {
  const MonoParams& p;
  uint64_t pol;
  uint32_t idx;    // chunks issued
  uint32_t cons;   // chunks known to be consumed
  uint32_t wend;   // ring write position (offset)
  // Monotonic write position: bytes placed so far plus the bytes skipped at
  // each wrap, so chunk i occupies the monotonic range [s_i, e_i) and its ring
  // bytes are that range modulo the ring size (32-bit, compared by signed
  // difference: a live span is far below 2^31).  s_i is kept in shared memory
  // per barrier pair (sm_starts).
  uint32_t head;
  long long t_wait;  // cycles spent waiting for ring space
  // L2 prefetch of the weight stream (p.l2_prefetch > 0): the bytes from
  // the copy cursor to p.l2_prefetch beyond it are kept requested into L2,
  // across stage and step boundaries, so HBM keeps streaming while the ring
  // is full and later copies hit L2.
  const unsigned char* wbase;
  long long len_layers, len_lm;  // bytes of the CTA's per-step stream
  long long pf_ahead;            // bytes requested beyond the copy cursor
  long long pf_off;              // prefetch cursor: offset within step pf_step
  int pf_step;

  __device__ explicit Producer(const MonoParams& pp)
      : p(pp), pol(dev::policy_evict_first()), idx(0), cons(0), wend(0), head(0), t_wait(0),
        wbase(nullptr), len_layers(0), len_lm(0), pf_ahead(0), pf_off(0), pf_step(0) {}

  __device__ long long stage_len(int st) const {
    const int2 r = p.ranges[st * p.grid + blockIdx.x];
    return (long long)range_rows(p, st, r.x, r.y) * stage_k(p, st) * piece_bytes(p.w8) / kPieceElems;
  }

  // Tops the prefetch up to `next` + p.l2_prefetch bytes beyond the copy cursor.
  __device__ void prefetch(uint32_t next) {
    const long long want = (long long)next + p.l2_prefetch;
    while (pf_ahead < want && pf_step < p.n_steps) {
      const long long rem = len_layers + (pf_step >= p.lm_from ? len_lm : 0) - pf_off;
      if (rem <= 0) {
        ++pf_step;
        pf_off = 0;
        continue;
      }
      const long long g = min(min(rem, 65536ll), want - pf_ahead);
      dev::bulk_prefetch_l2(wbase + pf_off, (uint32_t)g);
      pf_off += g;
      pf_ahead += g;
    }
  }

  // Waits until chunk i has been consumed; false = stop.
  __device__ bool wait_consumed(uint32_t i) {
    const uint32_t bar = sm_empty_s(p) + 8 * (i & (kRingBars - 1));
    const uint32_t par = (i / kRingBars) & 1u;
    if (dev::mbar_test_wait(bar, par)) return true;
    const long long c0 = clock64();
    const long long t0 = dev::globaltimer();
    bool ok = true;
    for (unsigned it = 1;; ++it) {
      if (sm_flags(p)[F_STOP]) {
        ok = false;
        break;
      }
      if (dev::mbar_try_wait(bar, par)) break;
      if ((it & 15u) == 0u && dev::globaltimer() - t0 > p.timeout_ns) {
        raise_error(p, DEV_TIMEOUT, -1, -1, -1, 1);
        ok = false;
        break;
      }
    }
    t_wait += clock64() - c0;
    return ok;
  }

  // Places the next chunk of sz bytes: its ring offset (the consumers'
  // ring_place) and its monotonic start.
  __device__ __forceinline__ uint32_t place(uint32_t sz, uint32_t& start) {
    const uint32_t ring = (uint32_t)p.ring_bytes;
    uint32_t off = wend;
    if (wend + sz > ring) {
      head += ring - wend;   // the bytes skipped at the wrap
      off = 0;
    }
    start = head;
    head += sz;
    wend = off + sz;
    return off;
  }

  // Frees the ring bytes of a chunk ending at monotonic position `end` and a
  // barrier pair for it.  The live chunks lie in [oldest start, new start);
  // once the oldest starts at or after end - ring they all lie in
  // [end - ring, new start), which shares no ring byte with the new chunk.
  // Chunks are released in order, so wait oldest first: one comparison per
  // released chunk.
  __device__ __forceinline__ bool acquire(uint32_t end) {
    const uint32_t bound = end - (uint32_t)p.ring_bytes;
    const uint32_t* starts = sm_starts(p);
    while (cons < idx) {
      if (idx - cons < (uint32_t)kRingBars &&
          (int)(starts[cons & (kRingBars - 1)] - bound) >= 0)
        break;
      if (!wait_consumed(cons)) return false;
      ++cons;
    }
    return true;
  }

  // One chunk = one bulk copy of the next `sz` bytes of the CTA's stream.
  __device__ bool chunk(const unsigned char*& src, uint32_t sz) {
    if (sm_flags(p)[F_STOP]) return false;
    uint32_t start;
    const uint32_t off = place(sz, start);
    if (!acquire(start + sz)) return false;
    const uint32_t b = idx & (kRingBars - 1);
    const uint32_t full = sm_full_s(p) + 8 * b;
    sm_offs(p)[b] = off;
    dev::mbar_arrive_expect_tx(full, sz);
    dev::bulk_g2s(sm_ring_s(p) + off, src, sz, full, pol);
    sm_starts(p)[b] = start;
    src += sz;
    ++idx;
    return true;
  }

  // One attention tile: `alloc` ring bytes, of which the first `bytes`
  // (whole padded cache rows) are copied from `src` in one bulk copy; the
  // consumers fill the remaining rows.
  __device__ bool tile(const unsigned char* src, uint32_t bytes, uint32_t alloc) {
    if (sm_flags(p)[F_STOP]) return false;
    uint32_t start;
    const uint32_t off = place(alloc, start);
    if (!acquire(start + alloc)) return false;
    const uint32_t b = idx & (kRingBars - 1);
    const uint32_t full = sm_full_s(p) + 8 * b;
    dev::mbar_arrive_expect_tx(full, bytes);
    if (bytes > 0) dev::bulk_g2s(sm_ring_s(p) + off, src, bytes, full, pol);
    sm_starts(p)[b] = start;
    ++idx;
    return true;
  }

  // Stage-trace stamp of the producer lane (slot ev of step i, layer l).
  __device__ __forceinline__ void trace(int i, int l, int ev) const {
    if (p.trace && (p.trace_cta < 0 || (int)blockIdx.x == p.trace_cta) && i < p.trace_steps) {
      const int per = p.L * kTracePerLayer + 4;
      const int row = p.trace_cta < 0 ? i * p.grid + (int)blockIdx.x : i;
      p.trace[row * per + l * kTracePerLayer + ev] = (unsigned long long)dev::globaltimer();
    }
  }

  // The stage's units in stream order, one chunk each (the plan is in
  // shared memory from the kernel's start).  One loop with a single issue
  // site keeps the producer's code small: it shares the SM's instruction
  // cache with the consumer warps.
  __device__ bool stage(int st, const unsigned char*& src) {
    const StagePlan& pl = sm_plan(p)[st];
    const int pb = piece_bytes(p.w8);
    const int nb = pl.nb, S = pl.S;
#pragma unroll 1
    for (int b = 0; b < nb; ++b) {
      const int rows = pl.block_rows(b);
#pragma unroll 1
      for (int s = 0; s < S; ++s) {
        const uint32_t sz = (uint32_t)(rows * pl.count(s) * pb);
        if (p.l2_prefetch > 0) prefetch(sz);
        if (!chunk(src, sz)) return false;
        pf_ahead -= sz;
      }
    }
    return true;
  }

  // K and V blocks of this CTA's attention item at step i, layer l, for the
  // positions before pos (the current position's k/v arrive as tagged
  // words).  The rows were written by other CTAs in earlier steps: before
  // the first such copy of step i the producer waits until its consumers
  // have passed step i-1's fenced publish, then orders that view before its
  // bulk copies with a proxy fence.
  __device__ bool attn(int i, int l) {
    const int pos = p.pos0 + i;
    const AttnItem it = attn_item(p, pos);
    if (!it.valid) return true;
    if (l == 0 && i > 0) {
      if (dev::ld_acquire_cta(sm_flags(p) + F_KVSTEP) < i) {
        const long long c0 = clock64();
        const long long t0 = dev::globaltimer();
        for (unsigned n = 1;; ++n) {
          if (sm_flags(p)[F_STOP]) return false;
          if (dev::ld_acquire_cta(sm_flags(p) + F_KVSTEP) >= i) break;
          if ((n & 63u) == 0u && dev::globaltimer() - t0 > p.timeout_ns) {
            raise_error(p, DEV_TIMEOUT, i, l, 5, 4);
            return false;
          }
        }
        t_wait += clock64() - c0;
      }
      dev::fence_proxy_async_global();
    }
    const int tb = attn_block(p);
    const unsigned char* K = reinterpret_cast<const unsigned char*>(kv_rows(p, l, 0, it.j));
    const unsigned char* V = reinterpret_cast<const unsigned char*>(kv_rows(p, l, 1, it.j));
    const uint32_t stride = (uint32_t)attn_row_stride(p);
    for (int b0 = it.t0; b0 < it.t1; b0 += tb) {
      const int nb = min(it.t1, b0 + tb) - b0;
      const int nc = max(0, min(b0 + nb, pos) - b0);   // rows already in the cache
      const uint32_t alloc = (uint32_t)((nb + 15) & ~15) * stride;
      if (!tile(K + (size_t)b0 * stride, (uint32_t)nc * stride, alloc) ||
          !tile(V + (size_t)b0 * stride, (uint32_t)nc * stride, alloc))
        return false;
    }
    return true;
  }

  // Asks L2 for the K and V rows this CTA's attention item of step i,
  // layer l will copy, when the layer's weight stream starts: the tiles are
  // copied into the ring only after the QKV chunks, and from L2 they land in
  // a fraction of a DRAM round trip under load.
  __device__ void prefetch_kv(int i, int l) {
    const int pos = p.pos0 + i;
    const AttnItem it = attn_item(p, pos);
    if (!it.valid) return;
    const int nc = max(0, min(it.t1, pos) - it.t0);
    if (nc == 0) return;
    const uint32_t stride = (uint32_t)attn_row_stride(p);
    for (int kv = 0; kv < 2; ++kv) {
      const unsigned char* src =
          reinterpret_cast<const unsigned char*>(kv_rows(p, l, kv, it.j)) + (size_t)it.t0 * stride;
      for (uint32_t o = 0, n = (uint32_t)nc * stride; o < n; o += 65536u)
        dev::bulk_prefetch_l2(src + o, min(65536u, n - o));
    }
  }

  // Waits until every copy this producer issued has landed (the last
  // kRingBars chunks; older ones were consumed before their barrier was
  // reused).
  __device__ void drain() {
    const long long t0 = dev::globaltimer();
    for (uint32_t i = idx > (uint32_t)kRingBars ? idx - kRingBars : 0u; i < idx; ++i) {
      const uint32_t bar = sm_full_s(p) + 8 * (i & (kRingBars - 1));
      const uint32_t par = (i / kRingBars) & 1u;
      while (!dev::mbar_try_wait(bar, par)) {
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, -1, -1, -1, 2);
          return;
        }
      }
    }
  }

  // The whole call's stream: per step the CTA's packed layers, then the LM
  // head on steps that pick an id.
  __device__ void run() {
    bool ok = true;
    const unsigned char* base = p.packed + p.packed_off[blockIdx.x];
    wbase = base;
    len_layers = p.L * (stage_len(ST_QKV) + stage_len(ST_O) + stage_len(ST_GU) + stage_len(ST_DOWN));
    len_lm = stage_len(ST_LM);
    for (int i = 0; i < p.n_steps && ok; ++i) {
      const unsigned char* src = base;
      // layers, then the LM head as a last pseudo-layer on steps that pick
      // an id; per layer QKV, the attention tiles, O, gate/up, down.  One
      // call site per kind of work (see stage).
      const int nl = p.L + (i >= p.lm_from ? 1 : 0);
#pragma unroll 1
      for (int l = 0; l < nl && ok; ++l) {
        const bool lm = l == p.L;
        if (!lm) {
          prefetch_kv(i, l);
          trace(i, l, 22);
        }
#pragma unroll 1
        for (int k = lm ? 4 : 0; k < 5 && ok; ++k) {
          if (k == 1) {
            trace(i, l, 23);
            ok = attn(i, l);
            trace(i, l, 20);
          } else {
            ok = stage(lm ? ST_LM : (k == 0 ? ST_QKV : k - 1), src);
          }
        }
      }
    }
    drain();
    p.cta_stats[kStatsPerCta * blockIdx.x + 3] = (unsigned long long)t_wait;
  }
};

// FP8 E4M3 weights with one fp32 scale per row: s = max |w| / 448 (1 for a
// zero row), codes E4M3(w / s) with fp32 division, round to nearest even,
// saturated at +-448.
__device__ __forceinline__ float e4m3_row_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}
// 16 fp16 weights (two 16-byte loads) to 16 codes
__device__ __forceinline__ uint4 quantize16(const uint4& a, const uint4& b, float s) {
  const uint32_t hw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&hw[2 * k]));
    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&hw[2 * k + 1]));
    o[k] = dev::f32x4_to_e4m3x4(__fdiv_rn(f0.x, s), __fdiv_rn(f0.y, s), __fdiv_rn(f1.x, s),
                                __fdiv_rn(f1.y, s));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Lays out CTA blockIdx.x's one-token weight stream in the order Producer
// streams it: per layer the QKV, O, gate/up and down units, then the LM
// head, each unit [row][piece][piece bytes].  fp16: a copy; fp8: every
// weight w of row r becomes the E4M3 code of w / s_r (fp32 division, round
// to nearest even, saturated at +-448), s_r the row's scale (rowscale_stage).
// Run once per model (and per change of the weight format or chunk size).
__device__ void repack_stage(const MonoParams& p, int st, const LayerW& w, unsigned char*& dst,
                             const float* scales) {
  const int2 r = p.ranges[st * p.grid + blockIdx.x];
  const int pb = piece_bytes(p.w8);
  const StagePlan pl = stage_plan(p, st);
  for_each_unit(pl, [&](int, int b, int s, int rows, int n) {
    const int n16 = n * pb / 16;   // 16-byte units of a row's part of the unit
    const int p0 = pl.first(s);
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int e = threadIdx.x; e < rows * n16; e += blockDim.x) {
      const int j = e / n16, q = e - j * n16;
      const int k = b * pl.nr + j;
      const __half* row = row_ptr(p, st, w, r.x, r.y, k) + (size_t)p0 * kPieceElems;
      if (!p.w8) {
        d[e] = reinterpret_cast<const uint4*>(row)[q];
      } else {   // 16 weights -> 16 codes
        d[e] = quantize16(reinterpret_cast<const uint4*>(row)[2 * q],
                          reinterpret_cast<const uint4*>(row)[2 * q + 1], scales[k]);
      }
    }
    dst += (size_t)rows * n * pb;
    return true;
  });
}

// Row scales of CTA blockIdx.x's rows of stage st, in stream order:
// s_r = max_c |w_rc| / 448 in fp32 (1 for a zero row).  One warp per row.
__device__ void rowscale_stage(const MonoParams& p, int st, const LayerW& w, float* out) {
  const int2 r = p.ranges[st * p.grid + blockIdx.x];
  const int R = range_rows(p, st, r.x, r.y);
  const int K = stage_k(p, st);
  const int lane = threadIdx.x & 31;
  for (int j = threadIdx.x >> 5; j < R; j += blockDim.x >> 5) {
    const __half2* row = reinterpret_cast<const __half2*>(row_ptr(p, st, w, r.x, r.y, j));
    float m = 0.f;
    for (int k = lane; k < K / 2; k += 32) {
      const float2 v = __half22float2(row[k]);
      m = fmaxf(m, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) out[j] = e4m3_row_scale(m);
  }
}

// ----------------------------------------------------------------- consumer

// Attention scratch in the activation area of shared memory: q as fp16 hi
// and lo tiles [kMaxGroup][HD + 8] (the mma's padding rows 8-15 are passed
// as zero registers, never stored), P tile [kMaxGroup][kAttnBlock + 8]
// fp16, scores [G][kAttnBlock] fp32 (tiles and scores together hold at
// least kCombineBytesPerHead * G bytes, the combine's scratch), the current
// position's k and v, the running output [G][HD] and per-head running max,
// sum and rescale factor.
template <int HD>
struct AttnSmem {
  static constexpr int kTiles = 2 * kMaxGroup * (HD + 8) * 2 + kMaxGroup * (kAttnBlock + 8) * 2;
  __half *qhi, *qlo, *ps;
  float *sc, *kn, *vn, *orun, *mrun, *lrun, *alpha;
  __device__ explicit AttnSmem(const MonoParams& p) {
    unsigned char* b = reinterpret_cast<unsigned char*>(sm_xs(p));
    qhi = reinterpret_cast<__half*>(b);
    b += kMaxGroup * (HD + 8) * 2;
    qlo = reinterpret_cast<__half*>(b);
    b += kMaxGroup * (HD + 8) * 2;
    ps = reinterpret_cast<__half*>(b);
    b += kMaxGroup * (kAttnBlock + 8) * 2;
    sc = reinterpret_cast<float*>(b);
    b += max(p.G * kAttnBlock * 4, kCombineBytesPerHead * p.G - kTiles);
    kn = reinterpret_cast<float*>(b);
    vn = kn + HD;
    orun = vn + HD;
    mrun = orun + p.G * HD;
    lrun = mrun + kMaxGroup;
    alpha = lrun + kMaxGroup;
  }
};

// The consumer warps' code.  It keeps no state in the object: a non-inlined
// member function reaches members through a pointer to the stack, and stack
// lines that miss the small L1 left beside the shared-memory carve-out cost
// an L2 round trip at every stage entry.  The parameter block is read from
// its shared-memory copy (kie_p), thread indices come from threadIdx, the
// ring cursors, the (step, layer, stage) position and thread 0's counters
// live in shared memory (kie_cur, kie_at, kie_ctr), and the stage functions
// get the layer and the fault-hook decision as arguments.
struct Consumer {
  __device__ Consumer() {}

  // Stage trace (measurement, tid 0 only): per step kTracePerLayer slots
  // per layer (stage boundaries, attention sub-steps, stream waits; the
  // layout is documented with kie_set_trace) + 4 for the LM head.
  __device__ __noinline__ void trace_put(int ev, unsigned long long v) const {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    if (p.trace && tid == 0 && (p.trace_cta < 0 || (int)blockIdx.x == p.trace_cta) &&
        kie_at[0] < p.trace_steps) {
      const int step = kie_at[0], layer = kie_at[1];
      const int per = p.L * kTracePerLayer + 4;
      const int row = p.trace_cta < 0 ? step * p.grid + (int)blockIdx.x : step;
      const int idx = row * per + (layer < p.L ? layer * kTracePerLayer : p.L * kTracePerLayer) + ev;
      p.trace[idx] = v;
    }
  }
  __device__ __forceinline__ void trace(int ev) const {
    const MonoParams& p = kie_p;
    if (p.trace)
      trace_put(ev, p.trace_clock ? (unsigned long long)clock64()
                                  : (unsigned long long)dev::globaltimer());
  }
  // Stream wait of the stage just finished (slots 16 + stage), then reset.
  __device__ __forceinline__ void trace_stream_wait(int st) {
    const MonoParams& p = kie_p;
    if (threadIdx.x == 0) {
      if (p.trace) trace_put(16 + st, (unsigned long long)kie_ctr[2]);
      kie_ctr[2] = 0;
    }
  }
  __device__ __forceinline__ void trace_loaded() const {
    switch (kie_at[2]) {
      case ST_QKV: trace(1); break;
      case ST_O: trace(4); break;
      case ST_GU: trace(6); break;
      case ST_DOWN: trace(8); break;
      default: trace(1); break;
    }
  }

  // Test hook: the stage whose publication this CTA withholds at (step i,
  // layer l), or -1.
  __device__ __forceinline__ static int fault_stage_at(int i, int l) {
    const MonoParams& p = kie_p;
    return (p.fault_cta == (int)blockIdx.x && p.fault_step == i && p.fault_layer == l)
               ? p.fault_stage
               : -1;
  }
  // Sets the stage of the position reported by errors and traces.
  __device__ __forceinline__ static void at_stage(int st) {
    if (threadIdx.x == 0) kie_at[2] = st;
  }

  // Slow path of a chunk wait: bounded spin on the full barrier.
  __device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t par) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    const long long c0 = clock64();
    const long long t0 = dev::globaltimer();
    bool ok = true;
    for (unsigned it = 1;; ++it) {
      if (dev::mbar_try_wait(bar, par)) break;
      if ((it & 15u) == 0u) {
        if (sm_flags(p)[F_ABORT]) {
          ok = false;
          break;
        }
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, kie_at[0], kie_at[1], kie_at[2], 3);
          sm_flags(p)[F_ABORT] = 1;
          ok = false;
          break;
        }
      }
    }
    if (tid == 0) {
      kie_ctr[1] += clock64() - c0;
      if (p.trace) kie_ctr[2] += dev::globaltimer() - t0;
    }
    return ok;
  }

  // ---- ring: waits for the next chunk (sz bytes) and returns its offset;
  // cidx / cend: the caller's copies of the wait and read-position cursors
  __device__ __forceinline__ bool wait_chunk(uint32_t sz, uint32_t& off, uint32_t& cidx,
                                             uint32_t& cend) {
    const MonoParams& p = kie_p;
    off = ring_place(cend, sz, (uint32_t)p.ring_bytes);
    const uint32_t bar = sm_full_s(p) + 8 * (cidx & (kRingBars - 1));
    const uint32_t par = (cidx / kRingBars) & 1u;
    ++cidx;
    if (dev::mbar_test_wait(bar, par)) return true;
    return wait_slow(bar, par);
  }
  // Releases the oldest chunk this warp waited for and has not released
  // (crel: the caller's copy of the release cursor).
  __device__ __forceinline__ void release_chunk(uint32_t& crel) {
    const MonoParams& p = kie_p;
    const int lane = (int)(threadIdx.x & 31);
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(sm_empty_s(p) + 8 * (crel & (kRingBars - 1)));
    ++crel;
  }

  // Polls NB pairs of tagged words (pair b at src + 2*k2[b], used when
  // k2[b] < n2) until every word carries `tag`.  All pending pairs are
  // re-read together, so a round costs one L2 round trip; rounds after the
  // first sleep p.poll_ns (0 by default: measured fastest) before the next.
  // Returns false on abort, timeout or a word that carries a newer tag
  // (protocol violation).
  template <int NB>
  __device__ __forceinline__ bool poll_pairs(const u64* src, const int (&k2)[NB], int n2,
                                             unsigned tag, ulonglong2 (&v)[NB], int where) {
    const MonoParams& p = kie_p;
    unsigned pend = 0;
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (k2[b] < n2) {
        v[b] = dev::ld_relaxed_v2_u64(src + 2 * k2[b]);
        pend |= 1u << b;
      }
    long long t0 = 0;
    for (unsigned it = 0;; ++it) {
      bool newer = false;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if ((pend >> b) & 1u) {
          const unsigned tx = (unsigned)(v[b].x >> 32), ty = (unsigned)(v[b].y >> 32);
          if (tx == tag && ty == tag) pend &= ~(1u << b);
          newer |= (tx != 0u && (int)(tx - tag) > 0) || (ty != 0u && (int)(ty - tag) > 0);
        }
      }
      if (!pend) return true;
      if (newer) {
        raise_error(p, DEV_PROTOCOL, kie_at[0], kie_at[1], kie_at[2], where);
        sm_flags(p)[F_ABORT] = 1;
        return false;
      }
      if (it == 0) {
        t0 = dev::globaltimer();
      } else if ((it & 7u) == 0u) {
        if (sm_flags(p)[F_ABORT] || global_error(p)) {
          sm_flags(p)[F_ABORT] = 1;
          return false;
        }
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, kie_at[0], kie_at[1], kie_at[2], where);
          sm_flags(p)[F_ABORT] = 1;
          return false;
        }
      }
      __nanosleep(p.poll_ns);
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if ((pend >> b) & 1u) v[b] = dev::ld_relaxed_v2_u64(src + 2 * k2[b]);
    }
  }

  // ---- GEMV input vector in shared memory: fp16, natural order (lane l of
  // piece q reads elements 256q + 8l .. +8 with one 16-byte load).
  __device__ __forceinline__ __half2* xs16() const {
    const MonoParams& p = kie_p;
    return reinterpret_cast<__half2*>(kie_smem + p.sm.xs_off);
  }

  // Stores elements 2*k2 and 2*k2+1 of a K-vector into xs as fp16 (times
  // the gain when given); adds the squares of the raw values to acc.
  __device__ __forceinline__ void store_pair(int k2, float a, float b, const __half* gain,
                                             float& acc) {
    acc = fmaf(a, a, acc);
    acc = fmaf(b, b, acc);
    if (gain) {
      const float2 g = __half22float2(reinterpret_cast<const __half2*>(gain)[k2]);
      a *= g.x;
      b *= g.y;
    }
    xs16()[k2] = __floats2half2_rn(a, b);
  }

  // Loads a K-vector into xs (times `gain` if given) and returns in `ss` the
  // sum of squares of the raw values.  Source: tagged words, or an fp16
  // embedding row.  The polls of one thread are issued in batches of 8
  // 16-byte loads (one batch for K <= 4096) so that their L2 round trips
  // overlap.  With parking on, each warp first parks the landed chunks of
  // stage park_st (the GEMV that reads this vector; -1: none).  Returns
  // false (uniformly) on abort.
  __device__ __noinline__ bool load_vec(const u64* src, unsigned tag, const __half* emb, int K,
                           const __half* gain, float& ss, int where, int park_st) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x, warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
    constexpr int NB = 8;
    const long long c0 = clock64();
    if (parking(p) && park_st >= 0) {
      // the previous stage's ring cursors are visible after this barrier
      dev::consumer_sync();
      park(park_st);
    }
    float acc = 0.f;
    bool bad = false;
    const int K2 = K >> 1;
    if (emb) {
      const __half2* e2 = reinterpret_cast<const __half2*>(emb);
      for (int k2 = tid; k2 < K2; k2 += kConsumerThreads) {
        const float2 v = __half22float2(e2[k2]);
        store_pair(k2, v.x, v.y, gain, acc);
      }
    } else {
      for (int base = tid; base < K2 && !bad; base += kConsumerThreads * NB) {
        ulonglong2 v[NB];
        int k2[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) k2[b] = base + b * kConsumerThreads;
        if (!poll_pairs<NB>(src, k2, K2, tag, v, where)) {
          bad = true;
          break;
        }
#pragma unroll
        for (int b = 0; b < NB; ++b)
          if (k2[b] < K2)
            store_pair(k2[b], __uint_as_float((unsigned)v[b].x), __uint_as_float((unsigned)v[b].y),
                       gain, acc);
      }
    }
    acc = dev::warp_sum(acc);
    if (lane == 0) sm_red(p)[warp] = acc;
    bad = dev::consumer_sync_or(bad);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) t += sm_red(p)[w];
    ss = t;
    if (tid == 0) kie_ctr[0] += clock64() - c0;
    trace_loaded();
    return !bad;
  }

  // Polls n2 pairs of tagged words into dst[0 .. 2*n2) (times `scale`).
  __device__ __noinline__ bool load_pairs(const u64* src, unsigned tag, int n2, float* dst,
                                          float scale, int where) {
    const int tid = (int)threadIdx.x;
    constexpr int NB = 4;
    for (int base = tid; base < n2; base += kConsumerThreads * NB) {
      ulonglong2 v[NB];
      int k2[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) k2[b] = base + b * kConsumerThreads;
      if (!poll_pairs<NB>(src, k2, n2, tag, v, where)) return false;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (k2[b] < n2) {
          dst[2 * k2[b]] = __uint_as_float((unsigned)v[b].x) * scale;
          dst[2 * k2[b] + 1] = __uint_as_float((unsigned)v[b].y) * scale;
        }
    }
    return true;
  }

  // ---- GEMV arithmetic: lane l of a 512-byte piece multiplies 8 fp16
  // weights by the 8 fp16 activations it shares with the other row.
  __device__ __forceinline__ static void dot_piece(const uint4& w, const uint4& x, float (&c)[8]) {
    dev::fma_f16x2_f32(c[0], c[1], w.x, x.x);
    dev::fma_f16x2_f32(c[2], c[3], w.y, x.y);
    dev::fma_f16x2_f32(c[4], c[5], w.z, x.z);
    dev::fma_f16x2_f32(c[6], c[7], w.w, x.w);
  }
  // fp8 weights: lane l's 8 E4M3 codes of a piece (elements 8l .. 8l+7)
  __device__ __forceinline__ static void dot_piece(const uint2& w, const uint4& x, float (&c)[8]) {
    dev::fma_f16x2_f32(c[0], c[1], dev::e4m3x2_to_f16x2((unsigned short)(w.x & 0xFFFFu)), x.x);
    dev::fma_f16x2_f32(c[2], c[3], dev::e4m3x2_to_f16x2((unsigned short)(w.x >> 16)), x.y);
    dev::fma_f16x2_f32(c[4], c[5], dev::e4m3x2_to_f16x2((unsigned short)(w.y & 0xFFFFu)), x.z);
    dev::fma_f16x2_f32(c[6], c[7], dev::e4m3x2_to_f16x2((unsigned short)(w.y >> 16)), x.w);
  }
  __device__ __forceinline__ static float sum8(const float (&c)[8]) {
    return ((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7]));
  }

  // Sums of NR rows' per-lane partial sums c[i][0..7] over the warp.  On
  // return lane l holds the sum of row l / (32 / NR') (NR' = NR rounded up
  // to a power of two; a fourth row of NR = 3 is zero): butterflies that
  // hand half of the rows to the other half-warp first need 4 + log2 NR'
  // exchanges for all rows instead of 5 per row.
  template <int NR>
  __device__ __forceinline__ static float reduce_rows(const float (&c)[NR][8], int lane) {
    if constexpr (NR == 1) {
      return dev::warp_sum(sum8(c[0]));
    } else if constexpr (NR == 2) {
      const bool up = (lane & 16) != 0;
      const float a = sum8(c[0]), b = sum8(c[1]);
      float t = (up ? b : a) + __shfl_xor_sync(0xffffffffu, up ? a : b, 16);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      return t;
    } else {
      const float v0 = sum8(c[0]), v1 = sum8(c[1]), v2 = sum8(c[2]);
      float v3 = 0.f;
      if constexpr (NR == 4) v3 = sum8(c[3]);
      // lanes 16-31 keep rows 2 and 3, lanes 0-15 rows 0 and 1
      const bool up = (lane & 16) != 0;
      const float t0 = (up ? v2 : v0) + __shfl_xor_sync(0xffffffffu, up ? v0 : v2, 16);
      const float t1 = (up ? v3 : v1) + __shfl_xor_sync(0xffffffffu, up ? v1 : v3, 16);
      // lanes with bit 3 set keep the odd row of their pair
      const bool mid = (lane & 8) != 0;
      float t = (mid ? t1 : t0) + __shfl_xor_sync(0xffffffffu, mid ? t0 : t1, 8);
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      return t;
    }
  }

  // Tensor-memory address of column 0 of warp w's parking columns: its own
  // 32 lanes, columns kParkCols * (w / 4) onward.
  __device__ __forceinline__ static uint32_t park_base(int w) {
    return kie_tmem + ((uint32_t)(32 * (w & 3)) << 16) + (uint32_t)(kParkCols * (w >> 2));
  }

  // Moves this warp's next units of stage st that have already landed in
  // the ring (in unit order, while they fit its kParkCols columns) into its
  // tensor memory, lane l keeping its 16 bytes of every piece of every row,
  // and releases their ring chunks, so that the producer streams further
  // ahead while the warp waits for other CTAs.  Called after a consumer
  // barrier that follows the previous stage (the ring cursors are current).
  // fp16 streams only.
  __device__ __noinline__ void park(int st) {
    const MonoParams& p = kie_p;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const StagePlan pl = sm_plan(p)[st];
    const uint32_t ci0 = kie_cur[0];
    const int S = pl.S, nu = pl.nb * S;
    const unsigned char* ring = sm_ring(p);
    const uint32_t full_s = sm_full_s(p), empty_s = sm_empty_s(p);
    const volatile uint32_t* offs = sm_offs(p);
    const uint32_t tb = park_base(warp);
    int b = warp / S, s = warp - (warp / S) * S;
    uint32_t col = 0;
    int parked = 0;
#pragma unroll 1
    for (int u = warp; u < nu; u += kConsumerWarps) {
      const int rows = pl.block_rows(b), n = pl.count(s);
      const int np = rows * n;   // piece rows: 16 bytes of each per lane, 4 columns
      if (col + 4u * (uint32_t)np > (uint32_t)kParkCols) break;
      const uint32_t chunk = ci0 + (uint32_t)u;
      const uint32_t bar = full_s + 8 * (chunk & (kRingBars - 1));
      // every lane must have seen the chunk land before reading it
      if (!__all_sync(0xffffffffu, dev::mbar_test_wait(bar, (chunk / kRingBars) & 1u))) break;
      const uint32_t off = offs[chunk & (kRingBars - 1)];
      if (u == nu - 1 && lane == 0) kie_ring_end = off + (uint32_t)(np * kPieceBytes);
      const uint4* src = reinterpret_cast<const uint4*>(ring + off) + lane;
      int j = 0;
#pragma unroll 1
      for (; j + 4 <= np; j += 4) {
        const uint4 v0 = src[(j + 0) * 32], v1 = src[(j + 1) * 32];
        const uint4 v2 = src[(j + 2) * 32], v3 = src[(j + 3) * 32];
        dev::tmem_st4(tb + col + 4 * j, v0);
        dev::tmem_st4(tb + col + 4 * j + 4, v1);
        dev::tmem_st4(tb + col + 4 * j + 8, v2);
        dev::tmem_st4(tb + col + 4 * j + 12, v3);
      }
#pragma unroll 1
      for (; j < np; ++j) dev::tmem_st4(tb + col + 4 * j, src[j * 32]);
      dev::tmem_wait_st();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive_n(empty_s + 8 * (chunk & (kRingBars - 1)), kConsumerWarps);
      col += 4u * (uint32_t)np;
      ++parked;
      s += kConsumerWarps;
      while (s >= S) {
        s -= S;
        ++b;
      }
    }
    if (lane == 0) {
      kie_park_n[warp] = parked;
      kie_park_ci[warp] = ci0;
    }
    __syncwarp();
  }

  // This warp's units of a stage whose blocks have NR rows (see StagePlan):
  // unit u belongs to warp u % kConsumerWarps and is the stage's chunk
  // ci0 + u.  For each of its units the warp waits for the chunk, reads its
  // ring offset (published by the producer before it armed the chunk's
  // barrier), multiplies the rows' pieces by the activation pieces (one
  // activation load serves all rows of the unit), releases the chunk with
  // one arrival worth all consumer warps, reduces the rows across the lanes
  // and writes each row's sum (part s of the row when the rows are split in
  // parts) times the row's scale.  The owner of the last unit records the
  // ring position after it.
  template <bool W8, int NR>
  __device__ __forceinline__ void gemv_units(const StagePlan& pl, const float* rsc, uint32_t ci0,
                                             bool& bad) {
    using WT = typename std::conditional<W8, uint2, uint4>::type;   // a lane's weights of a piece
    constexpr int PB = W8 ? kPieceElems : kPieceBytes;
    constexpr int kLanesPerRow = NR == 1 ? 32 : (NR == 2 ? 16 : 8);
    const MonoParams& p = kie_p;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned char* ring = sm_ring(p);
    const uint4* xv = reinterpret_cast<const uint4*>(kie_smem + p.sm.xs_off) + lane;
    float* rowacc = sm_rowacc(p);
    const uint32_t full_s = sm_full_s(p), empty_s = sm_empty_s(p);
    const volatile uint32_t* offs = sm_offs(p);
    const int my_i = lane / kLanesPerRow;          // the unit row whose sum this lane writes
    const bool writer = (lane & (kLanesPerRow - 1)) == 0;
    const int S = pl.S, nu = pl.nb * S;
    int b = warp / S, s = warp - (warp / S) * S;   // block and part of unit u
    // this warp's first units of the stage may be parked in tensor memory
    const int npark = (!W8 && kie_park_ci[warp] == ci0) ? kie_park_n[warp] : 0;
    const uint32_t tb = W8 ? 0u : park_base(warp);
    uint32_t pcol = 0;
    int kown = 0;
#pragma unroll 1
    for (int u = warp; u < nu; u += kConsumerWarps, ++kown) {
      const int rows = pl.block_rows(b), n = pl.count(s);
      const uint32_t chunk = ci0 + (uint32_t)u;
      const int k = b * NR + my_i;
      const bool mine = writer && my_i < rows;
      const float sc = (W8 && mine) ? __ldg(rsc + k) : 1.f;
      float c[NR][8];
#pragma unroll
      for (int i = 0; i < NR; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) c[i][j] = 0.f;
      if constexpr (!W8) {
        if (kown < npark) {
          // parked: the chunk was released when it was parked; rows past
          // the end of a short block read the block's last row again
          if (!bad) {
            const uint32_t rs = 4u * (uint32_t)n;   // columns per row
            const uint32_t a0 = tb + pcol, a1 = a0 + rs * (uint32_t)min(1, rows - 1);
            const uint32_t a2 = a0 + rs * (uint32_t)min(2, rows - 1);
            const uint32_t a3 = a0 + rs * (uint32_t)min(3, rows - 1);
            const uint4* x = xv + (size_t)pl.first(s) * 32;
#pragma unroll 1
            for (int q = 0; q < n; ++q) {
              uint4 wv[4];
              dev::tmem_ld4x4_wait(a0 + 4 * q, a1 + 4 * q, a2 + 4 * q, a3 + 4 * q, wv);
              const uint4 a = x[q * 32];
#pragma unroll
              for (int i = 0; i < NR; ++i) dot_piece(wv[i], a, c[i]);
            }
          }
          pcol += 4u * (uint32_t)(rows * n);
          const float t = reduce_rows<NR>(c, lane);
          if (mine) rowacc[S == 1 ? k : k * S + s] = t * sc;
          s += kConsumerWarps;
          while (s >= S) {
            s -= S;
            ++b;
          }
          continue;
        }
      }
      const uint32_t bar = full_s + 8 * (chunk & (kRingBars - 1));
      const uint32_t par = (chunk / kRingBars) & 1u;
      if (!dev::mbar_test_wait(bar, par) && !wait_slow(bar, par)) bad = true;
      const uint32_t off = offs[chunk & (kRingBars - 1)];
      if (u == nu - 1 && lane == 0) kie_ring_end = off + (uint32_t)(rows * n * PB);
      if (!bad) {
        // rows past the end of a short last block read the block's last
        // row again (their sums are not written), so that every load is
        // unconditional
        const WT* w[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i)
          w[i] = reinterpret_cast<const WT*>(ring + off) + (size_t)min(i, rows - 1) * n * 32 + lane;
        const uint4* x = xv + (size_t)pl.first(s) * 32;
#pragma unroll 2
        for (int q = 0; q < n; ++q) {
          const uint4 a = x[q * 32];
#pragma unroll
          for (int i = 0; i < NR; ++i) dot_piece(w[i][q * 32], a, c[i]);
        }
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive_n(empty_s + 8 * (chunk & (kRingBars - 1)), kConsumerWarps);
      const float t = reduce_rows<NR>(c, lane);
      if (mine) rowacc[S == 1 ? k : k * S + s] = t * sc;
      // the unit kConsumerWarps further on
      s += kConsumerWarps;
      while (s >= S) {
        s -= S;
        ++b;
      }
    }
  }

  // GEMV of this CTA's rows of stage st: dot products (times the rows'
  // scales when the stream is fp8), read back with row_result.  The stage's
  // chunks are the next nb * S of the ring; one barrier at the end, after
  // which thread 0 moves the ring cursors past them.  W8: pieces of fp8 E4M3 weights (8 bytes a lane), converted to fp16
  // pairs and multiplied like fp16 weights; rsc: the row scales of this
  // CTA's rows of the stage (unused for fp16).
  template <bool W8>
  __device__ __noinline__ bool gemv(int st, const float* rsc) {
    const StagePlan pl = sm_plan(kie_p)[st];
    const uint32_t ci0 = kie_cur[0];
    bool bad = false;
    switch (pl.nr) {
      case 1: gemv_units<W8, 1>(pl, rsc, ci0, bad); break;
      case 2: gemv_units<W8, 2>(pl, rsc, ci0, bad); break;
      case 3: gemv_units<W8, 3>(pl, rsc, ci0, bad); break;
      default: gemv_units<W8, 4>(pl, rsc, ci0, bad); break;
    }
    const bool any_bad = dev::consumer_sync_or(bad);
    if (threadIdx.x == 0 && pl.nb > 0) {
      // every chunk of the stage was released by the warp that computed it
      const uint32_t ci = ci0 + (uint32_t)(pl.nb * pl.S);
      kie_cur[0] = ci;
      kie_cur[1] = ci;
      kie_cur[2] = kie_ring_end;
    }
    return !any_bad;
  }

  // The GEMV of stage st of layer `layer` in the stream's weight format.
  __device__ __forceinline__ bool gemv_stage(int st, int layer) {
    const MonoParams& p = kie_p;
    if (!p.w8) return gemv<false>(st, nullptr);
    const StagePlan& pl = sm_plan(p)[st];
    return gemv<true>(st, kie_wsc + (st == ST_LM ? 0 : (size_t)layer * pl.rows_layer) + pl.sbase);
  }

  // Raw dot product of row k (0-based within the CTA's rows) of the last
  // gemv: the row's sum, or its parts' sums added in part order.
  __device__ __forceinline__ float row_result(const StagePlan& pl, int k) const {
    const float* a = sm_rowacc(kie_p);
    if (pl.S == 1) return a[k];
    float s = 0.f;
    for (int q = 0; q < pl.S; ++q) s += a[k * pl.S + q];
    return s;
  }

  __device__ __forceinline__ void put(u64* dst, unsigned tag, float v, bool skip) {
    if (!skip) dev::st_relaxed_u64(dst, dev::tag_word(tag, v));
  }

  // ---- stage bodies -------------------------------------------------------

  // RMSNorm + QKV GEMV + RoPE + KV append.
  __device__ __noinline__ bool stage_qkv(const LayerW& w, int layer, int tok, int pos, unsigned tag,
                                         bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    at_stage(ST_QKV);
    const int2 r = p.ranges[ST_QKV * p.grid + blockIdx.x];
    float ss;
    const __half* emb = layer == 0 ? p.tok_emb + (size_t)tok * p.d : nullptr;
    if (r.y <= r.x) return true;
    const int half = p.hd >> 1;
    const int nqp = p.H * half, np_all = qkv_pair_units(p);
    const float2* cs = p.rope + (size_t)pos * half;
    // this thread's first RoPE angle, fetched before the input wait and the
    // GEMV so that its global round trip is off the critical path
    float2 cs0 = make_float2(1.f, 0.f);
    {
      const int u = r.x + tid;
      if (u < r.y && u < np_all) cs0 = cs[(u < nqp ? u : u - nqp) % half];
    }
    if (!load_vec(p.x_attn, tag, emb, p.d, w.attn_norm, ss, 10, ST_QKV)) return false;
    if (!gemv_stage(ST_QKV, layer)) return false;
    const StagePlan pl = sm_plan(p)[ST_QKV];
    const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
    const int np = qkv_pairs_in(p, r.x, r.y);
    const int kvs = p.hd + kKvPad;                    // padded cache row
    __half* kbase = p.kv + (size_t)layer * 2 * p.KV * p.max_seq * kvs;
    __half* vbase = kbase + (size_t)p.KV * p.max_seq * kvs;
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      if (u < np_all) {
        const float a = row_result(pl, 2 * k) * rs, b = row_result(pl, 2 * k + 1) * rs;
        const bool isq = u < nqp;
        const int uu = isq ? u : u - nqp;
        const int h = uu / half, i = uu - h * half;
        const float2 c = u == r.x + tid ? cs0 : cs[i];
        const float lo = a * c.x - b * c.y;
        const float hi = b * c.x + a * c.y;
        if (isq) {
          put(p.qbuf + h * p.hd + i, tag, lo, skip);
          put(p.qbuf + h * p.hd + i + half, tag, hi, skip);
        } else {
          const __half klo = __float2half_rn(lo), khi = __float2half_rn(hi);
          __half* kd = kbase + ((size_t)h * p.max_seq + pos) * kvs;
          kd[i] = klo;
          kd[i + half] = khi;
          put(p.kvnew + h * p.hd + i, tag, __half2float(klo), skip);
          put(p.kvnew + h * p.hd + i + half, tag, __half2float(khi), skip);
        }
      } else {
        const int vr = u - np_all;
        const int lr = 2 * np + (k - np);
        const __half vh = __float2half_rn(row_result(pl, lr) * rs);
        const int h = vr / p.hd, e = vr - h * p.hd;
        vbase[((size_t)h * p.max_seq + pos) * kvs + e] = vh;
        put(p.kvnew + p.KV * p.hd + vr, tag, __half2float(vh), skip);
      }
    }
    return true;
  }

  // Combine of a KV head's partials, spread over the head's items: item s
  // owns output dims [d0, d1) (a multiple of 4 wide) of every one of the G
  // heads.  A partial row of (item, head) is [m, l, o/l as fp16 pairs] in
  // tagged words, so completeness is read from the tags: no fence and no
  // counter.  The item polls the (m, l) of every split and its dims of
  // every split's o/l in one batch, then with
  // w_s = exp(m_s - M) l_s / sum_s exp(m_s - M) l_s writes
  // o = sum_s w_s (o_s / l_s) for its dims.  Returns false (uniformly) on
  // abort.
  template <int HD>
  __device__ __noinline__ bool attn_combine(const AttnItem it, unsigned tag, bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    constexpr int ROW = 2 + HD / 2;          // tagged words per (item, head) row
    const int G = p.G, nsplit = it.nsplit, j = it.j;
    const int W = (((HD + nsplit - 1) / nsplit) + 3) & ~3;
    const int d0 = it.s * W, d1 = min(HD, d0 + W);
    if (d0 >= d1) return true;
    const int nd4 = (d1 - d0) / 4;           // o word pairs per row in this slice
    const u64* base = p.partials + (size_t)(j * nsplit) * G * ROW;
    const int n2 = nsplit * G * ROW / 2;     // pairs of the head's partial block
    const int nml = nsplit * G, ntot = nml + nml * nd4;
    // polled values go where q, P and the scores lived (free once the
    // blocks are done): (m, l) [nsplit * G], then o/l [nsplit * G][4 * nd4]
    // at a 16-byte boundary; with nsplit <= 96 at most
    // kCombineBytesPerHead * G bytes, which the tiles and scores span
    float2* ml = reinterpret_cast<float2*>(AttnSmem<HD>(p).qhi);
    float* os = reinterpret_cast<float*>(ml + ((nml + 1) & ~1));
    constexpr int NB = 4;
    bool bad = false;
    for (int q0 = tid; q0 < ntot && !bad; q0 += kConsumerThreads * NB) {
      int k2[NB];
      ulonglong2 v[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int q = q0 + b * kConsumerThreads;
        if (q < nml) {
          k2[b] = q * (ROW / 2);
        } else if (q < ntot) {
          const int r = (q - nml) / nd4, d4 = (q - nml) - r * nd4;
          k2[b] = (r * ROW + 2 + d0 / 2 + 2 * d4) / 2;
        } else {
          k2[b] = n2;
        }
      }
      if (!poll_pairs<NB>(base, k2, n2, tag, v, 23)) {
        bad = true;
        break;
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int q = q0 + b * kConsumerThreads;
        if (q < nml) {
          ml[q] = make_float2(__uint_as_float((unsigned)v[b].x), __uint_as_float((unsigned)v[b].y));
        } else if (q < ntot) {
          const int r = (q - nml) / nd4, d4 = (q - nml) - r * nd4;
          const unsigned lo = (unsigned)v[b].x, hi = (unsigned)v[b].y;
          const float2 x0 = __half22float2(*reinterpret_cast<const __half2*>(&lo));
          const float2 x1 = __half22float2(*reinterpret_cast<const __half2*>(&hi));
          *reinterpret_cast<float4*>(os + r * 4 * nd4 + 4 * d4) = make_float4(x0.x, x0.y, x1.x, x1.y);
        }
      }
    }
    if (dev::consumer_sync_or(bad)) return false;
    const int wd = d1 - d0;
    for (int e = tid; e < G * wd; e += kConsumerThreads) {
      const int g = e / wd, dd = e - g * wd;
      float M = -INFINITY;
      for (int q = 0; q < nsplit; ++q) M = fmaxf(M, ml[q * G + g].x);
      float L = 0.f, O = 0.f;
      for (int q = 0; q < nsplit; ++q) {
        const float2 v = ml[q * G + g];
        const float f = expf(v.x - M) * v.y;
        L += f;
        O = fmaf(f, os[(q * G + g) * 4 * nd4 + dd], O);
      }
      put(p.obuf + ((size_t)j * G + g) * HD + d0 + dd, tag, O / L, skip);
    }
    // the polled values live in the activation buffer, which the next
    // stage's input load overwrites
    dev::consumer_sync();
    trace(13);
    return true;
  }

  // Split-K attention over positions 0..pos for the G query heads of one
  // KV head; the head's items then share the combine (attn_combine).  K and V
  // tiles arrive through the ring (issued by the producer before q is
  // ready, rows at a padded stride); the current position's k and v come
  // from the tagged words and are written into the tiles here.  Both
  // contractions run on warp-level mma (m16n8k16, fp16 in, fp32 out):
  //   scores: S^T[head][t] = Q K^T, A = q (heads padded to 16 rows) split
  //           into fp16 hi + lo parts so that S keeps fp32 accuracy, B = the
  //           K tile; warps take 8-position column tiles in turn;
  //   softmax: warp g owns head g (online over the item's blocks); P is
  //           rounded to fp16 and its row sums use the rounded values;
  //   P.V:    O[head][dims] += P V, B fragments by transposed ldmatrix from
  //           the V tile; warp w owns HD/8 dims.
  template <int HD>
  __device__ __noinline__ bool stage_attn(int pos, unsigned tag, bool skip_combine) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x, warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
    at_stage(5);
    const AttnItem it = attn_item(p, pos);
    if (!it.valid) return true;
    constexpr int QS = HD + 8;                  // halfs per Q tile row
    constexpr int PSW = kAttnBlock + 8;         // halfs per P tile row
    constexpr int KT = HD / 16;                 // k-steps of the score mma
    // 8-dim output tiles per warp in P.V (warps past HD / 8 have none)
    constexpr int DTW = HD / 8 >= kConsumerWarps ? HD / 8 / kConsumerWarps : 1;
    const bool pv_warp = warp * DTW < HD / 8;
    const int G = p.G;
    const int j = it.j;
    const AttnSmem<HD> a(p);
    const float scale = 1.0f / sqrtf((float)HD);
    const long long c0 = clock64();
    bool bad = false;
    // Q rows >= G and the whole P tile start at zero (those rows stay zero)
    for (int e = tid; e < (kMaxGroup - G) * QS; e += kConsumerThreads) {
      a.qhi[G * QS + e] = __float2half_rn(0.f);
      a.qlo[G * QS + e] = __float2half_rn(0.f);
    }
    for (int e = tid; e < kMaxGroup * PSW / 2; e += kConsumerThreads)
      reinterpret_cast<uint32_t*>(a.ps)[e] = 0u;
    // q (tagged), scaled, as fp16 hi + lo
    {
      const u64* src = p.qbuf + (size_t)j * G * HD;
      const int n2 = G * HD / 2;
      constexpr int NB = 4;
      for (int base = tid; base < n2 && !bad; base += kConsumerThreads * NB) {
        ulonglong2 v[NB];
        int k2[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) k2[b] = base + b * kConsumerThreads;
        if (!poll_pairs<NB>(src, k2, n2, tag, v, 20)) {
          bad = true;
          break;
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (k2[b] < n2) {
            const int e = 2 * k2[b], g = e / HD, d = e - g * HD;
            const float x0 = __uint_as_float((unsigned)v[b].x) * scale;
            const float x1 = __uint_as_float((unsigned)v[b].y) * scale;
            const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
            *reinterpret_cast<__half2*>(a.qhi + g * QS + d) = __halves2half2(h0, h1);
            *reinterpret_cast<__half2*>(a.qlo + g * QS + d) = __halves2half2(
                __float2half_rn(x0 - __half2float(h0)), __float2half_rn(x1 - __half2float(h1)));
          }
        }
      }
    }
    if (it.t1 > pos && !bad) {
      bad = !load_pairs(p.kvnew + j * HD, tag, HD / 2, a.kn, 1.0f, 21) ||
            !load_pairs(p.kvnew + p.KV * HD + j * HD, tag, HD / 2, a.vn, 1.0f, 22);
    }
    if (tid < kMaxGroup) {
      a.mrun[tid] = -INFINITY;
      a.lrun[tid] = 0.f;
    }
    if (dev::consumer_sync_or(bad)) return false;
    if (tid == 0) kie_ctr[0] += clock64() - c0;
    trace(10);
    // ring cursors (read after the barrier above; written back after the last
    // barrier below)
    uint32_t ci = kie_cur[0], cr = kie_cur[1], ce = kie_cur[2];

    const int gid = lane >> 2, tig = lane & 3;
    // A fragments of q come from the hi / lo tiles (rows gid are heads,
    // rows gid + 8 zero padding)
    const __half* qh = a.qhi + gid * QS + tig * 2;
    const __half* ql = a.qlo + gid * QS + tig * 2;
    float oacc[DTW][4];
#pragma unroll
    for (int dt = 0; dt < DTW; ++dt) oacc[dt][0] = oacc[dt][1] = oacc[dt][2] = oacc[dt][3] = 0.f;

    const unsigned char* ring = sm_ring(p);
    const int RS = attn_row_stride(p);
    const int RSH = RS / 2;
    const int tb = attn_block(p);
    for (int b0 = it.t0; b0 < it.t1; b0 += tb) {
      const int nb = min(it.t1, b0 + tb) - b0;
      const int nc = max(0, min(b0 + nb, pos) - b0);   // rows that came through the ring
      const int nbp = (nb + 15) & ~15;
      const uint32_t sz = (uint32_t)(nbp * RS);
      uint32_t offk = 0, offv = 0;
      bool badc = !wait_chunk(sz, offk, ci, ce);
      badc = !wait_chunk(sz, offv, ci, ce) || badc;
      if (b0 == it.t0) trace(14);
      __half* Kt = reinterpret_cast<__half*>(sm_ring_w(p) + offk);
      __half* Vt = reinterpret_cast<__half*>(sm_ring_w(p) + offv);
      if (!badc) {
        // row nc: the current position (when in this block); rows up to nbp: zero
        for (int e = tid; e < (nbp - nc) * HD; e += kConsumerThreads) {
          const int r = nc + e / HD, d = e - (e / HD) * HD;
          const bool cur = r < nb;
          Kt[r * RSH + d] = __float2half_rn(cur ? a.kn[d] : 0.f);
          Vt[r * RSH + d] = __float2half_rn(cur ? a.vn[d] : 0.f);
        }
      }
      if (dev::consumer_sync_or(badc)) return false;
      // scores
      for (int nt = warp; nt < nbp / 8; nt += kConsumerWarps) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        const unsigned char* krow = ring + offk + (nt * 8 + gid) * RS + tig * 4;
#pragma unroll
        for (int ks = 0; ks < KT; ++ks) {
          const uint32_t kb0 = *reinterpret_cast<const uint32_t*>(krow + ks * 32);
          const uint32_t kb1 = *reinterpret_cast<const uint32_t*>(krow + ks * 32 + 16);
          dev::mma_16816(c, *reinterpret_cast<const uint32_t*>(qh + ks * 16), 0u,
                         *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 8), 0u, kb0, kb1);
          dev::mma_16816(c, *reinterpret_cast<const uint32_t*>(ql + ks * 16), 0u,
                         *reinterpret_cast<const uint32_t*>(ql + ks * 16 + 8), 0u, kb0, kb1);
        }
        if (gid < G) {
          const int t = nt * 8 + 2 * tig;
          a.sc[gid * kAttnBlock + t] = t < nb ? c[0] : -INFINITY;
          a.sc[gid * kAttnBlock + t + 1] = t + 1 < nb ? c[1] : -INFINITY;
        }
      }
      dev::consumer_sync();
      // online softmax over the block: warp g owns head g
      if (warp < G) {
        const float* row = a.sc + warp * kAttnBlock;
        __half* prow = a.ps + warp * PSW;
        float mx = -INFINITY;
        for (int t = lane; t < nbp; t += 32) mx = fmaxf(mx, row[t]);
        mx = dev::warp_max(mx);
        const float mold = a.mrun[warp];
        const float mnew = fmaxf(mold, mx);
        float sum = 0.f;
        for (int t = lane; t < nbp; t += 32) {
          const __half e = __float2half_rn(expf(row[t] - mnew));
          prow[t] = e;
          sum += __half2float(e);
        }
        sum = dev::warp_sum(sum);
        if (lane == 0) {
          const float al = expf(mold - mnew);
          a.alpha[warp] = al;
          a.lrun[warp] = a.lrun[warp] * al + sum;
          a.mrun[warp] = mnew;
        }
      }
      dev::consumer_sync();
      if (b0 == it.t0) trace(15);
      // P.V into the running output (rows gid < G are heads)
      if (pv_warp) {
        const float al = gid < G ? a.alpha[gid] : 0.f;
#pragma unroll
        for (int dt = 0; dt < DTW; ++dt) {
          oacc[dt][0] *= al;
          oacc[dt][1] *= al;
        }
        const int d0 = warp * 8 * DTW;
        const int m = lane >> 3, r8 = lane & 7;
        const uint32_t vrow = sm_ring_s(p) + offv + (uint32_t)(((m & 1) * 8 + r8) * RS) +
                              (uint32_t)((d0 + (m >> 1) * 8) * 2);
        for (int kk = 0; kk < nbp / 16; ++kk) {
          const __half* pr = a.ps + gid * PSW + kk * 16 + tig * 2;
          const uint32_t pa0 = *reinterpret_cast<const uint32_t*>(pr);
          const uint32_t pa2 = *reinterpret_cast<const uint32_t*>(pr + 8);
          const uint32_t va = vrow + (uint32_t)(kk * 16 * RS);
          if constexpr (DTW == 2) {
            uint32_t v0, v1, v2, v3;
            dev::ldmatrix_x4_trans(va, v0, v1, v2, v3);
            dev::mma_16816(oacc[0], pa0, 0u, pa2, 0u, v0, v1);
            dev::mma_16816(oacc[DTW - 1], pa0, 0u, pa2, 0u, v2, v3);
          } else {
            uint32_t v0, v1;
            dev::ldmatrix_x2_trans(va, v0, v1);
            dev::mma_16816(oacc[0], pa0, 0u, pa2, 0u, v0, v1);
          }
        }
      }
      dev::consumer_sync();
      release_chunk(cr);
      release_chunk(cr);
    }
    // running output of heads gid < G to shared memory
    if (gid < G && pv_warp) {
#pragma unroll
      for (int dt = 0; dt < DTW; ++dt) {
        const int d = warp * 8 * DTW + dt * 8 + 2 * tig;
        a.orun[gid * HD + d] = oacc[dt][0];
        a.orun[gid * HD + d + 1] = oacc[dt][1];
      }
    }
    dev::consumer_sync();
    if (tid == 0) {
      kie_cur[0] = ci;
      kie_cur[1] = cr;
      kie_cur[2] = ce;
    }
    trace(11);
    // publish this item's partial as tagged words: per head [m, l, then
    // o / l as fp16 pairs]
    constexpr int ROW = 2 + HD / 2;
    u64* part = p.partials + (size_t)blockIdx.x * G * ROW;
    for (int e = tid; e < G * HD / 2; e += kConsumerThreads) {
      const int g = e / (HD / 2), i = e - g * (HD / 2);
      const float inv = 1.0f / a.lrun[g];
      const __half2 h =
          __floats2half2_rn(a.orun[g * HD + 2 * i] * inv, a.orun[g * HD + 2 * i + 1] * inv);
      dev::st_relaxed_u64(part + g * ROW + 2 + i,
                          (static_cast<u64>(tag) << 32) | *reinterpret_cast<const unsigned*>(&h));
    }
    if (tid < G) {
      dev::st_relaxed_u64(part + tid * ROW, dev::tag_word(tag, a.mrun[tid]));
      dev::st_relaxed_u64(part + tid * ROW + 1, dev::tag_word(tag, a.lrun[tid]));
    }
    trace(12);
    return attn_combine<HD>(it, tag, skip_combine);
  }

  // O projection + residual -> x_ffn.
  __device__ bool stage_o(const LayerW& w, int layer, int tok, unsigned tag, bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    at_stage(ST_O);
    const int2 r = p.ranges[ST_O * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    // O's chunks are not parked (measured 0.5% faster on the 2.2B model:
    // the whole O stage fits the ring and is read right after the wait)
    if (!load_vec(p.obuf, tag, nullptr, p.H * p.hd, nullptr, ss, 30, -1)) return false;
    if (!gemv_stage(ST_O, layer)) return false;
    const StagePlan pl = sm_plan(p)[ST_O];
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      const float res = layer == 0 ? __half2float(p.tok_emb[(size_t)tok * p.d + u]) : sm_res_attn(p)[k];
      const float v = res + row_result(pl, k);
      sm_res_ffn(p)[k] = v;
      put(p.x_ffn + u, tag, v, skip);
    }
    return true;
  }

  // RMSNorm + gate/up GEMV + SwiGLU -> h.
  __device__ bool stage_gu(const LayerW& w, int layer, unsigned tag, bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    at_stage(ST_GU);
    const int2 r = p.ranges[ST_GU * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    if (!load_vec(p.x_ffn, tag, nullptr, p.d, w.ffn_norm, ss, 40, ST_GU)) return false;
    if (!gemv_stage(ST_GU, layer)) return false;
    const StagePlan pl = sm_plan(p)[ST_GU];
    const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      const float g = row_result(pl, 2 * k) * rs, up = row_result(pl, 2 * k + 1) * rs;
      const float sg = g / (1.0f + expf(-g));
      put(p.hbuf + u, tag, sg * up, skip);
    }
    return true;
  }

  // Down GEMV + residual -> x_attn (input of the next layer).
  __device__ bool stage_down(const LayerW& w, int layer, unsigned tag, unsigned tag_next, bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    at_stage(ST_DOWN);
    const int2 r = p.ranges[ST_DOWN * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    if (!load_vec(p.hbuf, tag, nullptr, p.F, nullptr, ss, 50, ST_DOWN)) return false;
    if (!gemv_stage(ST_DOWN, layer)) return false;
    const StagePlan pl = sm_plan(p)[ST_DOWN];
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      const float v = sm_res_ffn(p)[k] + row_result(pl, k);
      sm_res_attn(p)[k] = v;
      put(p.x_attn + u, tag_next, v, skip);
    }
    return true;
  }

  __device__ __forceinline__ static bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
  }
  __device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      if (better(v2, i2, v, i)) {
        v = v2;
        i = i2;
      }
    }
  }

  // Score of vocabulary entry u whose logit is v, at position pos: the
  // logit itself (greedy), or v / T + G with G = -log(-log(U)) standard
  // Gumbel noise, U from word u % 4 of Philox4x64-10 block (u / 4, pos)
  // under key (seed, 0), mapped to the open interval (0, 1).  The argmax of
  // the noisy scores is a draw from softmax(logits / T).
  __device__ __forceinline__ float pick_score(float v, int u, int pos) const {
    const MonoParams& p = kie_p;
    if (!p.sample) return v;
    const unsigned long long w =
        dev::philox4x64_10_word((unsigned long long)(u >> 2), (unsigned long long)pos, p.seed, u & 3);
    const double uu = ((double)(w >> 11) + 0.5) * 0x1p-53;
    return (float)((double)v * p.inv_temp - log(-log(uu)));
  }
  __device__ __forceinline__ bool is_eos(int t) const {
    const MonoParams& p = kie_p;
    for (int k = 0; k < p.n_eos; ++k)
      if (t == p.eos_ids[k]) return true;
    return false;
  }

  // ---- top-k / top-p restriction of the draw
  // Sort key of vocabulary entry u with logit v: unsigned order is the
  // order "larger logit first, then the lower index" (the fp32 bits made
  // monotone in the high half, the complemented index in the low half).
  // Keys are unique and never 0, so 0 marks "no entry".
  __device__ __forceinline__ static u64 vocab_key(float v, int u) {
    const unsigned b = __float_as_uint(v);
    const unsigned ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return (static_cast<u64>(ord) << 32) | (0xFFFFFFFFu - (unsigned)u);
  }
  __device__ __forceinline__ static float key_value(u64 k) {
    const unsigned ord = (unsigned)(k >> 32);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
  }
  __device__ __forceinline__ static u64 shfl_xor_u64(u64 v, int o) {
    const unsigned lo = __shfl_xor_sync(0xffffffffu, (unsigned)v, o);
    const unsigned hi = __shfl_xor_sync(0xffffffffu, (unsigned)(v >> 32), o);
    return (static_cast<u64>(hi) << 32) | lo;
  }

  // The smallest key of the kept set: the top_k largest logits of the
  // whole vocabulary (ties by the lower index), then of those the shortest
  // prefix, largest probability first, whose mass under softmax(logits / T)
  // restricted to them reaches top_p.  Every CTA ranks its own rows and
  // publishes its sorted top_k keys as tagged words; every CTA then copies
  // the first kFilterHeads keys of all the CTAs' lists and pops the global
  // top_k with one warp (a lane holds the heads of grid / 32 lists; a list
  // popped past its copied keys is read on from global memory), so every
  // CTA finds the same threshold and no further exchange is needed.
  // Called by all consumer threads; returns ~0 on abort.
  __device__ __noinline__ u64 filter_threshold(int2 r, float rs, unsigned tag) {
    const MonoParams& p = kie_p;
    const StagePlan pl = sm_plan(p)[ST_LM];
    const int tid = (int)threadIdx.x, warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
    constexpr u64 kAbort = ~0ull;
    const int n = r.y - r.x, kf = p.top_k, m = min(kf, kFilterHeads);
    u64* K = reinterpret_cast<u64*>(kie_smem + p.sm.xs_off);   // this CTA's keys [n]
    u64* Ls = K + n;                                            // its top kf, sorted
    u64* S = Ls + kMaxTopK;                                     // [grid][kFilterHeads]
    u64* P = S + p.grid * kFilterHeads;                         // global top kf, popped
    u64* tau_s = P + kMaxTopK;
    for (int i = tid; i < n; i += kConsumerThreads)
      K[i] = vocab_key(row_result(pl, i) * rs, r.x + i);
    for (int i = tid; i < kf; i += kConsumerThreads) Ls[i] = 0ull;
    dev::consumer_sync();
    for (int i = tid; i < n; i += kConsumerThreads) {
      const u64 k = K[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) rank += K[j] > k ? 1 : 0;
      if (rank < kf) Ls[rank] = k;
    }
    dev::consumer_sync();
    // publish: pair (2i, 2i+1) = high and low half of key i, tagged
    u64* mine = p.cands + (size_t)blockIdx.x * kMaxTopK * 2;
    for (int i = tid; i < kf; i += kConsumerThreads) {
      dev::st_relaxed_u64(mine + 2 * i, (static_cast<u64>(tag) << 32) | (unsigned)(Ls[i] >> 32));
      dev::st_relaxed_u64(mine + 2 * i + 1, (static_cast<u64>(tag) << 32) | (unsigned)Ls[i]);
    }
    // gather the first m keys of every list
    constexpr int NB = 4;
    const int ntot = p.grid * m, n2 = p.grid * kMaxTopK;
    bool bad = false;
    for (int base = tid; base < ntot && !bad; base += kConsumerThreads * NB) {
      int k2[NB];
      ulonglong2 v[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int q = base + b * kConsumerThreads;
        const int c = q / m, j = q - (q / m) * m;
        k2[b] = q < ntot ? c * kMaxTopK + j : n2;
      }
      if (!poll_pairs<NB>(p.cands, k2, n2, tag, v, 62)) {
        bad = true;
        break;
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int q = base + b * kConsumerThreads;
        if (q < ntot) {
          const int c = q / m, j = q - (q / m) * m;
          S[c * kFilterHeads + j] = (v[b].x << 32) | (v[b].y & 0xFFFFFFFFull);
        }
      }
    }
    if (dev::consumer_sync_or(bad)) return kAbort;
    if (warp == 0) {
      constexpr int Q = (160 + 31) / 32;   // lists per lane (grid <= 160)
      int ptr[Q];
      u64 h[Q];
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        const int c = lane + 32 * q;
        ptr[q] = 0;
        h[q] = c < p.grid ? S[c * kFilterHeads] : 0ull;
      }
      // (every lane runs every round: the shuffles need the whole warp)
      for (int t = 0; t < kf; ++t) {
        u64 best = 0ull;
        int bq = 0;
#pragma unroll
        for (int q = 0; q < Q; ++q)
          if (h[q] > best) {
            best = h[q];
            bq = q;
          }
        u64 wb = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const u64 x = shfl_xor_u64(wb, o);
          wb = x > wb ? x : wb;
        }
        if (lane == 0) P[t] = wb;
        if (wb != 0ull && best == wb) {
#pragma unroll
          for (int q = 0; q < Q; ++q)
            if (q == bq) {
              const int c = lane + 32 * q;
              ++ptr[q];
              if (ptr[q] >= kf) {
                h[q] = 0ull;
              } else if (ptr[q] < m) {
                h[q] = S[c * kFilterHeads + ptr[q]];
              } else {   // past the copied keys: read the list on
                const int k2[1] = {c * kMaxTopK + ptr[q]};
                ulonglong2 v[1];
                if (!poll_pairs<1>(p.cands, k2, n2, tag, v, 63)) bad = true;
                h[q] = bad ? 0ull : (v[0].x << 32) | (v[0].y & 0xFFFFFFFFull);
              }
            }
        }
      }
      bad = __any_sync(0xffffffffu, bad);
      __syncwarp();
      // the kept prefix: all kf (or fewer if the vocabulary is smaller), cut
      // at the first entry where the probability mass reaches top_p
      int nk = 0;
      for (int i = lane; i < kf; i += 32) nk += P[i] != 0ull ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nk += __shfl_xor_sync(0xffffffffu, nk, o);
      int cut = nk;   // entries kept
      if (p.top_p < 1.0 && nk > 0) {
        const double z0 = (double)key_value(P[0]) * p.inv_temp;
        const double e0 = lane < nk ? exp((double)key_value(P[lane]) * p.inv_temp - z0) : 0.0;
        const double e1 = lane + 32 < nk ? exp((double)key_value(P[lane + 32]) * p.inv_temp - z0) : 0.0;
        // inclusive prefix sums of both halves
        double c0 = e0, c1 = e1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double a0 = __shfl_up_sync(0xffffffffu, c0, o);
          const double a1 = __shfl_up_sync(0xffffffffu, c1, o);
          if (lane >= o) {
            c0 += a0;
            c1 += a1;
          }
        }
        const double half0 = __shfl_sync(0xffffffffu, c0, 31);
        c1 += half0;
        const double total = __shfl_sync(0xffffffffu, c1, 31);
        const unsigned b0 = __ballot_sync(0xffffffffu, lane < nk && c0 / total >= p.top_p);
        const unsigned b1 = __ballot_sync(0xffffffffu, lane + 32 < nk && c1 / total >= p.top_p);
        cut = b0 ? __ffs(b0) : (b1 ? 32 + __ffs(b1) : nk);
      }
      if (lane == 0) *tau_s = cut > 0 ? P[cut - 1] : 0ull;
    }
    if (dev::consumer_sync_or(bad)) return kAbort;
    return *tau_s;
  }

  // Final RMSNorm + LM head + token pick (argmax of pick_score); or, on
  // steps that pick no id, only the per-step fenced publish.  Returns the
  // picked id (uniform across the grid), or -1 on abort.
  __device__ __noinline__ int stage_lm(bool pick, int step, int step_row, unsigned tag, int pos,
                                       bool skip) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x, warp = (int)(threadIdx.x >> 5), lane = (int)(threadIdx.x & 31);
    at_stage(ST_LM);
    float best = -INFINITY;
    int bi = INT_MAX;
    const int2 r = p.ranges[ST_LM * p.grid + blockIdx.x];
    if (pick && r.y > r.x) {
      float ss;
      if (!load_vec(p.x_attn, tag, nullptr, p.d, p.final_norm, ss, 60, ST_LM)) return -1;
      if (!gemv_stage(ST_LM, 0)) return -1;
      const StagePlan pl = sm_plan(p)[ST_LM];
      trace(2);
      const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
      float* cap = (p.capture && step_row < p.capture_rows)
                       ? p.capture + (size_t)step_row * p.V
                       : nullptr;
      // rows below the top-k / top-p threshold key take no part in the draw
      u64 tau = 0ull;
      if (p.sample && p.top_k > 0) {
        tau = filter_threshold(r, rs, tag);
        if (tau == ~0ull) return -1;
      }
      for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
        const float v = row_result(pl, u - r.x) * rs;
        if (cap) cap[u] = v;
        if (vocab_key(v, u) < tau) continue;
        const float sc = pick_score(v, u, pos);
        if (better(sc, u, best, bi)) {
          best = sc;
          bi = u;
        }
      }
    }
    warp_argmax(best, bi);
    if (lane == 0) {
      sm_red(p)[warp] = best;
      sm_redi(p)[warp] = bi;
    }
    dev::consumer_sync();
    if (tid == 0) {
      float b = sm_red(p)[0];
      int ib = sm_redi(p)[0];
      for (int w = 1; w < kConsumerWarps; ++w)
        if (better(sm_red(p)[w], sm_redi(p)[w], b, ib)) {
          b = sm_red(p)[w];
          ib = sm_redi(p)[w];
        }
      // release: every plain store this CTA made in this step (KV cache,
      // logits) happens-before any CTA that reads these slots.
      dev::fence_acq_rel_gpu();
      if (!skip) {
        dev::st_relaxed_u64(p.slots + 2 * blockIdx.x, dev::tag_word(tag, b));
        dev::st_relaxed_u64(p.slots + 2 * blockIdx.x + 1,
                            (static_cast<u64>(tag) << 32) | (unsigned)ib);
      }
    }
    // gather every CTA's pick
    const long long c0 = clock64();
    bool bad = false;
    float gb = -INFINITY;
    int gi = INT_MAX;
    for (int c = tid; c < p.grid; c += kConsumerThreads) {
      ulonglong2 w2[1];
      const int k2[1] = {c};
      if (!poll_pairs<1>(p.slots, k2, p.grid, tag, w2, 61)) {
        bad = true;
        break;
      }
      const unsigned vb = (unsigned)w2[0].x, ib = (unsigned)w2[0].y;
      if (better(__uint_as_float(vb), (int)ib, gb, gi)) {
        gb = __uint_as_float(vb);
        gi = (int)ib;
      }
    }
    // acquire: later loads of KV entries written by other CTAs see them
    dev::fence_acq_rel_gpu();
    warp_argmax(gb, gi);
    if (lane == 0) {
      sm_red2(p)[warp] = gb;
      sm_redi2(p)[warp] = gi;
    }
    if (dev::consumer_sync_or(bad)) return -1;
    float b = sm_red2(p)[0];
    int ib = sm_redi2(p)[0];
    for (int w = 1; w < kConsumerWarps; ++w)
      if (better(sm_red2(p)[w], sm_redi2(p)[w], b, ib)) {
        b = sm_red2(p)[w];
        ib = sm_redi2(p)[w];
      }
    if (tid == 0) {
      kie_ctr[0] += clock64() - c0;
      // this step's KV writes of every CTA are now visible to this CTA:
      // the producer may copy them for the next step
      dev::st_release_cta(sm_flags(p) + F_KVSTEP, step + 1);
    }
    return ib;
  }

  // Walks a stage's chunk sequence without computing (stream-only timing).
  __device__ __noinline__ bool skip_stage(int st) {
    const MonoParams& p = kie_p;
    const StagePlan pl = sm_plan(p)[st];
    bool bad = false;
    uint32_t ci = kie_cur[0], cr = kie_cur[1], ce = kie_cur[2];
    const int pb = piece_bytes(p.w8);
    for_each_unit(pl, [&](int, int, int, int rows, int n) {
      uint32_t off;
      if (!wait_chunk((uint32_t)(rows * n * pb), off, ci, ce)) bad = true;
      release_chunk(cr);
      return true;
    });
    const bool any_bad = dev::consumer_sync_or(bad);
    if (threadIdx.x == 0) {
      kie_cur[0] = ci;
      kie_cur[1] = cr;
      kie_cur[2] = ce;
    }
    return !any_bad;
  }

  // Standalone GEMV engine run: y = W x over the LM-head stage's rows,
  // `iters` times (mode 0: stream the weights only, mode 1: full GEMV).
  __device__ void gemv_bench(int mode, const float* x, float* y, int iters) {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    const int2 r = p.ranges[ST_LM * p.grid + blockIdx.x];
    const int K = p.d;
    float acc = 0.f;
    for (int k2 = tid; k2 < K / 2; k2 += kConsumerThreads) {
      const float2 v = reinterpret_cast<const float2*>(x)[k2];
      store_pair(k2, v.x, v.y, nullptr, acc);
    }
    dev::consumer_sync();
    bool ok = true;
    for (int it = 0; it < iters && ok; ++it) {
      dev::consumer_sync();   // the ring cursors thread 0 wrote back are visible
      ok = mode == 0 ? skip_stage(ST_LM) : gemv_stage(ST_LM, 0);
    }
    if (ok && mode == 1)
      for (int u = r.x + tid; u < r.y; u += kConsumerThreads) y[u] = row_result(sm_plan(p)[ST_LM], u - r.x);
    if (tid == 0) {
      sm_flags(p)[F_STOP] = 1;
      u64* st = p.cta_stats + kStatsPerCta * blockIdx.x;
      st[2] = (u64)kie_ctr[1];
    }
  }

  template <int HD>
  __device__ void run() {
    const MonoParams& p = kie_p;
    const int tid = (int)threadIdx.x;
    const bool tmem = parking(p);
    if (tmem && (tid >> 5) == 0) dev::tmem_alloc(dev::smem_u32(&kie_tmem), 2 * kParkCols);
    dev::tmem_fence_before_sync();
    dev::consumer_sync();
    dev::tmem_fence_after_sync();
    const long long c_begin = clock64();
    int tok = p.forced ? p.forced[0] : p.first_tok;
    int done = 0;
    bool ok = true;
    for (int i = 0; i < p.n_steps && ok; ++i) {
      if (tid == 0) kie_at[0] = i;
      const int pos = p.pos0 + i;
      for (int l = 0; l < p.L && ok; ++l) {
        if (tid == 0) kie_at[1] = l;
        const LayerW& w = p.layers[l];
        const unsigned tag = epoch_of(p, i, l);
        const int fst = fault_stage_at(i, l);
        trace(0);
        ok = stage_qkv(w, l, tok, pos, tag, fst == ST_QKV);
        trace(2);
        trace_stream_wait(ST_QKV);
        ok = ok && stage_attn<HD>(pos, tag, fst == ST_O);
        trace(3);
        trace_stream_wait(5);
        ok = ok && stage_o(w, l, tok, tag, fst == ST_O);
        trace(5);
        trace_stream_wait(ST_O);
        ok = ok && stage_gu(w, l, tag, fst == ST_GU);
        trace(7);
        trace_stream_wait(ST_GU);
        ok = ok && stage_down(w, l, tag, tag + 1u, fst == ST_DOWN);
        trace(9);
        trace_stream_wait(ST_DOWN);
      }
      if (!ok) break;
      if (tid == 0) kie_at[1] = p.L;
      const bool pick = i >= p.lm_from;
      trace(0);
      const int next = stage_lm(pick, i, i - p.lm_from, epoch_of(p, i, p.L), pos,
                                fault_stage_at(i, p.L) == ST_LM);
      trace(3);
      if (tid == 0) kie_ctr[2] = 0;
      if (next < 0) {
        ok = false;
        break;
      }
      done = i + 1;
      if (pick && blockIdx.x == 0 && tid == 0) p.out_ids[i] = next;
      if (pick && is_eos(next)) break;
      if (p.forced && i + 1 < p.n_steps) tok = p.forced[i + 1];
      else tok = next;
    }
    if (tid == 0) sm_flags(p)[F_STOP] = 1;
    if (tmem) {
      // every warp's tensor-memory accesses are done before warp 0 frees it
      dev::tmem_fence_before_sync();
      dev::consumer_sync();
      dev::tmem_fence_after_sync();
      if ((tid >> 5) == 0) dev::tmem_dealloc(kie_tmem, 2 * kParkCols);
    }
    if (blockIdx.x == 0 && tid == 0) p.status->n_done = done;
    if (tid == 0) {
      u64* st = p.cta_stats + kStatsPerCta * blockIdx.x;
      st[0] = (u64)(clock64() - c_begin);
      st[1] = (u64)kie_ctr[0];
      st[2] = (u64)kie_ctr[1];
      st[4] = (u64)done;
    }
  }
};

// Common start of the persistent kernels: the parameter block's shared copy,
// the ring barriers, the flags and thread 0's counters.
__device__ __forceinline__ void kernel_setup(const MonoParams& p) {
  static_assert(sizeof(MonoParams) % 4 == 0, "parameter block copy");
  const unsigned* src = reinterpret_cast<const unsigned*>(&p);
  unsigned* dst = reinterpret_cast<unsigned*>(&kie_p);
  for (int i = threadIdx.x; i < (int)(sizeof(MonoParams) / 4); i += blockDim.x) dst[i] = src[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRingBars; ++s) {
      dev::mbar_init(sm_full_s(p) + 8 * s, 1);
      dev::mbar_init(sm_empty_s(p) + 8 * s, kConsumerWarps);
    }
    sm_flags(p)[F_ABORT] = 0;
    sm_flags(p)[F_STOP] = 0;
    sm_flags(p)[F_KVSTEP] = 0;
    kie_ctr[0] = kie_ctr[1] = kie_ctr[2] = 0;
    kie_cur[0] = kie_cur[1] = kie_cur[2] = 0u;
    kie_at[0] = kie_at[1] = kie_at[2] = 0;
    for (int w = 0; w < kConsumerWarps; ++w) kie_park_n[w] = 0;
    dev::mbar_fence_init();
  }
  setup_plans(p);
  __syncthreads();
}

}  // namespace

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) kie_monokernel(const __grid_constant__ MonoParams p) {
  kernel_setup(p);
  if (threadIdx.x >= kConsumerThreads) {
    dev::regs_dec<kRegsProducer>();
    if (threadIdx.x == kConsumerThreads) {
      Producer prod(p);
      prod.run();
    }
    return;
  }
  dev::regs_inc<kRegsConsumer>();
  Consumer c;
  c.run<HD>();
}

__global__ void __launch_bounds__(kThreads, 1)
    kie_gemv_kernel(const __grid_constant__ MonoParams p, int mode, const float* x, float* y,
                    int iters) {
  kernel_setup(p);
  if (threadIdx.x >= kConsumerThreads) {
    dev::regs_dec<kRegsProducer>();
    if (threadIdx.x == kConsumerThreads) {
      Producer prod(p);
      bool ok = true;
      for (int it = 0; it < iters && ok; ++it) {
        const unsigned char* src = p.packed + p.packed_off[blockIdx.x];
        ok = prod.stage(ST_LM, src);
      }
      prod.drain();
      p.cta_stats[kStatsPerCta * blockIdx.x + 3] = (unsigned long long)prod.t_wait;
    }
    return;
  }
  dev::regs_inc<kRegsConsumer>();
  Consumer c;
  c.gemv_bench(mode, x, y, iters);
}

__global__ void __launch_bounds__(256) kie_rowscale_kernel(const __grid_constant__ MonoParams p) {
  float* out = const_cast<float*>(p.wscale) + p.wscale_off[blockIdx.x];
  for (int l = 0; l < p.L; ++l) {
    const LayerW& w = p.layers[l];
    for (int st = ST_QKV; st <= ST_DOWN; ++st) {
      rowscale_stage(p, st, w, out);
      const int2 r = p.ranges[st * p.grid + blockIdx.x];
      out += range_rows(p, st, r.x, r.y);
    }
  }
  rowscale_stage(p, ST_LM, p.layers[0], out);
}

__global__ void __launch_bounds__(256) kie_repack_kernel(const __grid_constant__ MonoParams p,
                                                         unsigned char* packed) {
  unsigned char* dst = packed + p.packed_off[blockIdx.x];
  const float* sc = p.w8 ? p.wscale + p.wscale_off[blockIdx.x] : nullptr;
  for (int l = 0; l < p.L; ++l) {
    const LayerW& w = p.layers[l];
    for (int st = ST_QKV; st <= ST_DOWN; ++st) {
      repack_stage(p, st, w, dst, sc);
      if (sc) {
        const int2 r = p.ranges[st * p.grid + blockIdx.x];
        sc += range_rows(p, st, r.x, r.y);
      }
    }
  }
  repack_stage(p, ST_LM, p.layers[0], dst, sc);
}

// One matrix W[N][K] (fp16, row-major) to E4M3 codes[N][K] and scales[N]:
// a warp per row.
__global__ void __launch_bounds__(256) kie_quantize_kernel(const __half* W, int N, int K,
                                                           unsigned char* codes, float* scales) {
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * 8 + (int)(threadIdx.x >> 5); r < N; r += gridDim.x * 8) {
    const uint4* row = reinterpret_cast<const uint4*>(W + (size_t)r * K);
    float m = 0.f;
    for (int k = lane; k < K / 8; k += 32) {
      const uint4 v = row[k];
      const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[h]));
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sr = e4m3_row_scale(m);
    if (lane == 0) scales[r] = sr;
    uint4* out = reinterpret_cast<uint4*>(codes + (size_t)r * K);
    for (int q = lane; q < K / 16; q += 32) out[q] = quantize16(row[2 * q], row[2 * q + 1], sr);
  }
}

cudaError_t quantize_launch(const __half* W, int N, int K, unsigned char* codes, float* scales,
                            cudaStream_t s) {
  const int blocks = (N + 7) / 8 < 1184 ? (N + 7) / 8 : 1184;
  kie_quantize_kernel<<<blocks, 256, 0, s>>>(W, N, K, codes, scales);
  return cudaGetLastError();
}

cudaError_t repack_launch(const MonoParams& p, unsigned char* packed, cudaStream_t s) {
  if (p.w8) {
    kie_rowscale_kernel<<<p.grid, 256, 0, s>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  kie_repack_kernel<<<p.grid, 256, 0, s>>>(p, packed);
  return cudaGetLastError();
}

cudaError_t dynamic_smem_limit(int* out) {
  int dev = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  size_t stat = 0;
  for (const void* fn : {(const void*)kie_monokernel<64>, (const void*)kie_monokernel<128>,
                         (const void*)kie_gemv_kernel}) {
    cudaFuncAttributes a{};
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&a, fn);
    stat = a.sharedSizeBytes > stat ? a.sharedSizeBytes : stat;
  }
  if (e != cudaSuccess) return e;
  *out = optin - (int)stat;
  return cudaSuccess;
}

// Lets kie_gemv_kernel use all the dynamic shared memory it may have on the
// current device.  Always the same value, so calls from several host
// threads (the allocating and the no-allocation GEMV entry points) cannot
// undo each other's setting between configure and launch.
cudaError_t gemv_configure() {
  int limit = 0;
  cudaError_t e = dynamic_smem_limit(&limit);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute((const void*)kie_gemv_kernel,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
}

cudaError_t gemv_launch(const MonoParams& p, int mode, const float* x, float* y, int iters,
                        int grid, int smem_bytes, cudaStream_t s) {
  kie_gemv_kernel<<<grid, kThreads, smem_bytes, s>>>(p, mode, x, y, iters);
  return cudaGetLastError();
}

cudaError_t mono_configure(int hd, int smem_bytes, int* blocks_per_sm) {
  const void* fn = hd == 64 ? (const void*)kie_monokernel<64> : (const void*)kie_monokernel<128>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fn, kThreads, smem_bytes);
}

cudaError_t mono_launch(const MonoParams& p, int hd, int grid, int smem_bytes, cudaStream_t s) {
  const void* fn = hd == 64 ? (const void*)kie_monokernel<64> : (const void*)kie_monokernel<128>;
  void* args[] = {const_cast<MonoParams*>(&p)};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), args, (size_t)smem_bytes, s);
}

}  // namespace kie
