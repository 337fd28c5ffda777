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
//  * Warp specialisation.  Warp 8 is a producer: one lane walks the CTA's
//    static weight schedule for the whole call and streams it with
//    cp.async.bulk into a ring of shared-memory slots completed by
//    mbarriers.  The schedule does not depend on activations, so the
//    producer runs ahead across every stage boundary and keeps HBM busy
//    while the consumers wait for other CTAs.  Warps 0-7 consume: each
//    16-byte lane load of fp16 weights meets fp32 activations held in shared
//    memory, FMA in fp32, warp-shuffle reductions.
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

#include "kie_device.cuh"
#include "kie_kernel.h"
#include "kie_params.h"

namespace kie {

using u64 = unsigned long long;

namespace {

enum : int { F_ABORT = 0, F_STOP = 1, F_LAST = 2 };

struct Smem {
  unsigned char* ring;
  uint32_t ring_s;
  uint32_t full_s, empty_s;
  float* xs;
  float* rowacc;
  float* part;        // [8] tail-group partial sums
  float* red;         // [8] reduction scratch
  float* red2;        // [8]
  int* redi;          // [8]
  int* redi2;         // [8]
  volatile int* flags;
};

__device__ __forceinline__ Smem carve(const MonoParams& p, unsigned char* base) {
  Smem S;
  S.ring = base + p.sm.ring_off;
  S.ring_s = dev::smem_u32(S.ring);
  S.full_s = dev::smem_u32(base + p.sm.bar_off);
  S.empty_s = S.full_s + 8 * kMaxSlots;
  S.xs = reinterpret_cast<float*>(base + p.sm.xs_off);
  S.rowacc = reinterpret_cast<float*>(base + p.sm.rowacc_off);
  float* m = reinterpret_cast<float*>(base + p.sm.misc_off);
  S.part = m;
  S.red = m + 8;
  S.red2 = m + 16;
  S.redi = reinterpret_cast<int*>(m + 24);
  S.redi2 = reinterpret_cast<int*>(m + 32);
  S.flags = reinterpret_cast<volatile int*>(m + 40);
  return S;
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

// k-chunking of one group of rg (<= 8) rows with kp pieces per row: chunk kc
// covers pieces [first(kc), first(kc+1)) of every row of the group.
struct Chunking {
  int kp, nk;
  __device__ __forceinline__ int first(int kc) const {
    return (int)(((long long)kc * kp) / nk);
  }
};
__device__ __forceinline__ Chunking chunking(int rg, int kp, int slot_bytes) {
  int mp = slot_bytes / (rg * kPieceBytes);
  if (mp < 1) mp = 1;
  Chunking c;
  c.kp = kp;
  c.nk = (kp + mp - 1) / mp;
  return c;
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

struct Producer {
  const MonoParams& p;
  const Smem& S;
  uint64_t pol;
  int slot;
  unsigned round;
  unsigned used_mask, par_mask;

  __device__ Producer(const MonoParams& pp, const Smem& ss)
      : p(pp), S(ss), pol(dev::policy_evict_first()), slot(0), round(0), used_mask(0),
        par_mask(0) {}

  // Waits for the consumers to free the current slot; false = stop.
  __device__ bool wait_free() {
    if (round == 0) return true;
    const uint32_t bar = S.empty_s + 8 * slot;
    const uint32_t par = (round - 1) & 1u;
    if (dev::mbar_try_wait(bar, par)) return true;
    const long long t0 = dev::globaltimer();
    for (unsigned it = 1;; ++it) {
      if (S.flags[F_STOP]) return false;
      if (dev::mbar_try_wait(bar, par)) return true;
      if ((it & 15u) == 0u && dev::globaltimer() - t0 > p.timeout_ns) {
        raise_error(p, DEV_TIMEOUT, -1, -1, -1, 1);
        return false;
      }
    }
  }

  __device__ bool stage(int st, int layer) {
    const LayerW& w = p.layers[layer];
    const int2 r = p.ranges[st * p.grid + blockIdx.x];
    const int R = range_rows(p, st, r.x, r.y);
    const int K = stage_k(p, st);
    const int kp = K / kPieceElems;
    for (int g0 = 0; g0 < R; g0 += 8) {
      const int rg = min(8, R - g0);
      const Chunking ch = chunking(rg, kp, p.slot_bytes);
      for (int kc = 0; kc < ch.nk; ++kc) {
        if (S.flags[F_STOP]) return false;
        if (!wait_free()) return false;
        const int p0 = ch.first(kc), n = ch.first(kc + 1) - p0;
        const uint32_t bytes = (uint32_t)(n * kPieceBytes);
        const uint32_t full = S.full_s + 8 * slot;
        dev::mbar_arrive_expect_tx(full, bytes * rg);
        const uint32_t dst = S.ring_s + (uint32_t)slot * (uint32_t)p.slot_bytes;
        for (int j = 0; j < rg; ++j) {
          const __half* src = row_ptr(p, st, w, r.x, r.y, g0 + j) + (size_t)p0 * kPieceElems;
          dev::bulk_g2s(dst + (uint32_t)j * bytes, src, bytes, full, pol);
        }
        used_mask |= 1u << slot;
        par_mask = (par_mask & ~(1u << slot)) | ((round & 1u) << slot);
        if (++slot == p.ring_slots) {
          slot = 0;
          ++round;
        }
      }
    }
    return true;
  }

  // Waits until every copy this producer issued has landed.
  __device__ void drain() {
    const long long t0 = dev::globaltimer();
    for (int s = 0; s < p.ring_slots; ++s) {
      if (!((used_mask >> s) & 1u)) continue;
      const uint32_t bar = S.full_s + 8 * s;
      const uint32_t par = (par_mask >> s) & 1u;
      while (!dev::mbar_try_wait(bar, par)) {
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, -1, -1, -1, 2);
          return;
        }
      }
    }
  }

  __device__ void run() {
    for (int i = 0; i < p.n_steps; ++i) {
      for (int l = 0; l < p.L; ++l) {
        if (!stage(ST_QKV, l) || !stage(ST_O, l) || !stage(ST_GU, l) || !stage(ST_DOWN, l)) {
          drain();
          return;
        }
      }
      if (i >= p.lm_from && !stage(ST_LM, 0)) {
        drain();
        return;
      }
    }
    drain();
  }
};

// ----------------------------------------------------------------- consumer

struct Consumer {
  const MonoParams& p;
  const Smem& S;
  int tid, warp, lane;
  int slot;
  unsigned round;
  long long t_sync, t_stream;
  int step, layer, stage;  // for error reports

  __device__ Consumer(const MonoParams& pp, const Smem& ss)
      : p(pp), S(ss), slot(0), round(0), t_sync(0), t_stream(0), step(0), layer(0), stage(0) {
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
  }

  __device__ __forceinline__ bool fault_here(int st) const {
    return p.fault_cta == (int)blockIdx.x && p.fault_step == step && p.fault_layer == layer &&
           p.fault_stage == st;
  }

  // ---- tagged-word polling
  __device__ __noinline__ bool wait_tag_slow(const u64* a, unsigned tag, unsigned& out,
                                             int where) {
    const long long t0 = dev::globaltimer();
    for (unsigned it = 1;; ++it) {
      const u64 v = dev::ld_relaxed_u64(a);
      const unsigned tg = (unsigned)(v >> 32);
      if (tg == tag) {
        out = (unsigned)v;
        return true;
      }
      if (tg != 0u && (int)(tg - tag) > 0) {
        raise_error(p, DEV_PROTOCOL, step, layer, stage, where);
        S.flags[F_ABORT] = 1;
        return false;
      }
      if ((it & 31u) == 0u) {
        if (S.flags[F_ABORT] || global_error(p)) {
          S.flags[F_ABORT] = 1;
          return false;
        }
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, step, layer, stage, where);
          S.flags[F_ABORT] = 1;
          return false;
        }
      }
    }
  }
  __device__ __forceinline__ bool wait_tag(const u64* a, unsigned tag, unsigned& out, int where) {
    const u64 v = dev::ld_relaxed_u64(a);
    if ((unsigned)(v >> 32) == tag) {
      out = (unsigned)v;
      return true;
    }
    return wait_tag_slow(a, tag, out, where);
  }
  __device__ __forceinline__ bool wait_f(const u64* a, unsigned tag, float& out, int where) {
    unsigned u;
    const bool ok = wait_tag(a, tag, u, where);
    out = __uint_as_float(u);
    return ok;
  }

  // ---- ring
  __device__ __forceinline__ bool wait_full() {
    const uint32_t bar = S.full_s + 8 * slot;
    const uint32_t par = round & 1u;
    if (dev::mbar_try_wait(bar, par)) return true;
    const long long c0 = clock64();
    const long long t0 = dev::globaltimer();
    bool ok = true;
    for (unsigned it = 1;; ++it) {
      if (dev::mbar_try_wait(bar, par)) break;
      if ((it & 15u) == 0u) {
        if (S.flags[F_ABORT]) {
          ok = false;
          break;
        }
        if (dev::globaltimer() - t0 > p.timeout_ns) {
          raise_error(p, DEV_TIMEOUT, step, layer, stage, 3);
          S.flags[F_ABORT] = 1;
          ok = false;
          break;
        }
      }
    }
    if (tid == 0) t_stream += clock64() - c0;
    return ok;
  }
  __device__ __forceinline__ void release_slot() {
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(S.empty_s + 8 * slot);
    if (++slot == p.ring_slots) {
      slot = 0;
      ++round;
    }
  }

  // ---- permuted activation layout: element k of a K-vector sits where
  // lane (k%256)/8 of piece k/256 reads it with two conflict-free 16-byte
  // loads (elements 0-3 of the lane's 8 in the low half, 4-7 in the high).
  __device__ __forceinline__ int perm(int k, int K) const {
    const int piece = k >> 8, w = k & 255, ln = w >> 3, e = w & 7;
    return (e < 4 ? 0 : (K >> 1)) + ((piece * 32 + ln) << 2) + (e & 3);
  }

  // Loads a K-vector into xs (times `gain` if given) and returns in `ss` the
  // sum of squares of the raw values.  Source: tagged words, or an fp16
  // embedding row.  Returns false (uniformly) on abort.
  __device__ bool load_vec(const u64* src, unsigned tag, const __half* emb, int K,
                           const __half* gain, float& ss, int where) {
    const long long c0 = clock64();
    float acc = 0.f;
    bool bad = false;
    for (int k = tid; k < K; k += kConsumerThreads) {
      float v;
      if (emb) {
        v = __half2float(emb[k]);
      } else if (!wait_f(src + k, tag, v, where)) {
        bad = true;
        break;
      }
      acc = fmaf(v, v, acc);
      S.xs[perm(k, K)] = gain ? v * __half2float(gain[k]) : v;
    }
    acc = dev::warp_sum(acc);
    if (lane == 0) S.red[warp] = acc;
    bad = dev::consumer_sync_or(bad);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) t += S.red[w];
    ss = t;
    if (tid == 0) t_sync += clock64() - c0;
    return !bad;
  }

  // ---- GEMV of this CTA's rows of a stage into rowacc (raw dot products).
  __device__ bool gemv(int st, const LayerW& w, int ub, int ue) {
    const int R = range_rows(p, st, ub, ue);
    const int K = stage_k(p, st);
    const int kp = K / kPieceElems;
    const float4* xlo = reinterpret_cast<const float4*>(S.xs);
    const float4* xhi = reinterpret_cast<const float4*>(S.xs + (K >> 1));
    bool bad = false;
    for (int g0 = 0; g0 < R; g0 += 8) {
      const int rg = min(8, R - g0);
      const Chunking ch = chunking(rg, kp, p.slot_bytes);
      const int wpr = kConsumerWarps / rg;
      const bool active = warp < rg * wpr;
      const int r = warp / wpr, part = warp - (warp / wpr) * wpr;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int kc = 0; kc < ch.nk; ++kc) {
        if (!bad && !wait_full()) bad = true;
        if (active && !bad) {
          const int p0 = ch.first(kc), n = ch.first(kc + 1) - p0;
          const int pa = (part * n) / wpr, pb = ((part + 1) * n) / wpr;
          const uint4* wrow = reinterpret_cast<const uint4*>(
                                  S.ring + (size_t)slot * p.slot_bytes + (size_t)r * n * kPieceBytes) +
                              lane;
          const float4* xl = xlo + (size_t)p0 * 32 + lane;
          const float4* xh = xhi + (size_t)p0 * 32 + lane;
#pragma unroll 2
          for (int q = pa; q < pb; ++q) {
            const uint4 wv = wrow[q * 32];
            const float4 xa = xl[q * 32];
            const float4 xb = xh[q * 32];
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&wv.x));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&wv.y));
            const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&wv.z));
            const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&wv.w));
            a0 = fmaf(f0.x, xa.x, a0);
            a1 = fmaf(f0.y, xa.y, a1);
            a2 = fmaf(f1.x, xa.z, a2);
            a3 = fmaf(f1.y, xa.w, a3);
            a0 = fmaf(f2.x, xb.x, a0);
            a1 = fmaf(f2.y, xb.y, a1);
            a2 = fmaf(f3.x, xb.z, a2);
            a3 = fmaf(f3.y, xb.w, a3);
          }
        }
        release_slot();
      }
      if (active) {
        const float s = dev::warp_sum((a0 + a1) + (a2 + a3));
        if (lane == 0) {
          if (wpr == 1) S.rowacc[g0 + r] = s;
          else S.part[warp] = s;
        }
      }
      if (wpr > 1) {
        dev::consumer_sync();
        if (tid < rg) {
          float s = 0.f;
          for (int q = 0; q < wpr; ++q) s += S.part[tid * wpr + q];
          S.rowacc[g0 + tid] = s;
        }
      }
    }
    return !dev::consumer_sync_or(bad);
  }

  __device__ __forceinline__ void put(u64* dst, unsigned tag, float v, bool skip) {
    if (!skip) dev::st_relaxed_u64(dst, dev::tag_word(tag, v));
  }

  // ---- stage bodies -------------------------------------------------------

  // RMSNorm + QKV GEMV + RoPE + KV append.
  __device__ bool stage_qkv(const LayerW& w, int tok, int pos, unsigned tag) {
    stage = ST_QKV;
    const int2 r = p.ranges[ST_QKV * p.grid + blockIdx.x];
    float ss;
    const __half* emb = layer == 0 ? p.tok_emb + (size_t)tok * p.d : nullptr;
    if (r.y > r.x) {
      if (!load_vec(p.x_attn, tag, emb, p.d, w.attn_norm, ss, 10)) return false;
      if (!gemv(ST_QKV, w, r.x, r.y)) return false;
    } else {
      return true;
    }
    const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
    const int half = p.hd >> 1;
    const int nqp = p.H * half, np_all = qkv_pair_units(p);
    const int np = qkv_pairs_in(p, r.x, r.y);
    const float2* cs = p.rope + (size_t)pos * half;
    const bool skip = fault_here(ST_QKV);
    __half* kbase = p.kv + (size_t)layer * 2 * p.KV * p.max_seq * p.hd;
    __half* vbase = kbase + (size_t)p.KV * p.max_seq * p.hd;
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      if (u < np_all) {
        const float a = S.rowacc[2 * k] * rs, b = S.rowacc[2 * k + 1] * rs;
        const bool isq = u < nqp;
        const int uu = isq ? u : u - nqp;
        const int h = uu / half, i = uu - h * half;
        const float2 c = cs[i];
        const float lo = a * c.x - b * c.y;
        const float hi = b * c.x + a * c.y;
        if (isq) {
          put(p.qbuf + h * p.hd + i, tag, lo, skip);
          put(p.qbuf + h * p.hd + i + half, tag, hi, skip);
        } else {
          const __half klo = __float2half_rn(lo), khi = __float2half_rn(hi);
          __half* kd = kbase + ((size_t)h * p.max_seq + pos) * p.hd;
          kd[i] = klo;
          kd[i + half] = khi;
          put(p.kvnew + h * p.hd + i, tag, __half2float(klo), skip);
          put(p.kvnew + h * p.hd + i + half, tag, __half2float(khi), skip);
        }
      } else {
        const int vr = u - np_all;
        const int lr = 2 * np + (k - np);
        const __half vh = __float2half_rn(S.rowacc[lr] * rs);
        const int h = vr / p.hd, e = vr - h * p.hd;
        vbase[((size_t)h * p.max_seq + pos) * p.hd + e] = vh;
        put(p.kvnew + p.KV * p.hd + vr, tag, __half2float(vh), skip);
      }
    }
    return true;
  }

  // Split-K attention over positions 0..pos, GQA group of one KV head per
  // work item; the last item of a KV head combines the partials.
  template <int HD>
  __device__ bool stage_attn(int pos, unsigned tag) {
    stage = 5;
    const int n_pos = pos + 1;
    int nsplit = (n_pos + p.min_split_len - 1) / p.min_split_len;
    if (nsplit > p.max_split) nsplit = p.max_split;
    const int items = p.KV * nsplit;
    const int it = blockIdx.x;
    if (it >= items) return true;
    const int G = p.G;
    const int j = it / nsplit, s = it - (it / nsplit) * nsplit;
    const int t0 = (int)(((long long)s * n_pos) / nsplit);
    const int t1 = (int)(((long long)(s + 1) * n_pos) / nsplit);
    constexpr int NGRP = kConsumerThreads / (HD / 2);
    float* qs = S.xs;
    float* sc = qs + G * HD;
    float* kn = sc + G * kAttnBlock;
    float* vn = kn + HD;
    float* red = vn + HD;
    float* orun = red + NGRP * G * HD;
    float* mrun = orun + G * HD;
    float* lrun = mrun + kMaxGroup;
    float* alpha = lrun + kMaxGroup;
    const float scale = 1.0f / sqrtf((float)HD);
    const long long c0 = clock64();
    bool bad = false;
    for (int e = tid; e < G * HD && !bad; e += kConsumerThreads) {
      float v;
      if (!wait_f(p.qbuf + (size_t)j * G * HD + e, tag, v, 20)) bad = true;
      qs[e] = v * scale;
      orun[e] = 0.f;
    }
    if (t1 > pos) {
      for (int e = tid; e < 2 * HD && !bad; e += kConsumerThreads) {
        float v;
        const u64* src = e < HD ? p.kvnew + j * HD + e : p.kvnew + p.KV * HD + j * HD + (e - HD);
        if (!wait_f(src, tag, v, 21)) bad = true;
        if (e < HD) kn[e] = v;
        else vn[e - HD] = v;
      }
    }
    if (tid < kMaxGroup) {
      mrun[tid] = -INFINITY;
      lrun[tid] = 0.f;
    }
    if (dev::consumer_sync_or(bad)) return false;
    if (tid == 0) t_sync += clock64() - c0;

    const __half* Kc = p.kv + (((size_t)layer * 2 + 0) * p.KV + j) * (size_t)p.max_seq * HD;
    const __half* Vc = p.kv + (((size_t)layer * 2 + 1) * p.KV + j) * (size_t)p.max_seq * HD;
    for (int b0 = t0; b0 < t1; b0 += kAttnBlock) {
      const int nb = min(kAttnBlock, t1 - b0);
      // scores of the block: one thread per position, all G heads
      if (tid < nb) {
        const int u = b0 + tid;
        float sg[kMaxGroup];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) sg[g] = 0.f;
        const uint4* krow = reinterpret_cast<const uint4*>(Kc + (size_t)u * HD);
#pragma unroll 4
        for (int c = 0; c < HD / 8; ++c) {
          float kf[8];
          if (u == pos) {
#pragma unroll
            for (int e = 0; e < 8; ++e) kf[e] = kn[c * 8 + e];
          } else {
            const uint4 kv = krow[c];
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&kv.x));
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&kv.y));
            const float2 cc = __half22float2(*reinterpret_cast<const __half2*>(&kv.z));
            const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&kv.w));
            kf[0] = a.x; kf[1] = a.y; kf[2] = b.x; kf[3] = b.y;
            kf[4] = cc.x; kf[5] = cc.y; kf[6] = d.x; kf[7] = d.y;
          }
#pragma unroll
          for (int g = 0; g < kMaxGroup; ++g) {
            if (g < G) {
              const float4 qa = *reinterpret_cast<const float4*>(qs + g * HD + c * 8);
              const float4 qb = *reinterpret_cast<const float4*>(qs + g * HD + c * 8 + 4);
              float t = sg[g];
              t = fmaf(qa.x, kf[0], t); t = fmaf(qa.y, kf[1], t);
              t = fmaf(qa.z, kf[2], t); t = fmaf(qa.w, kf[3], t);
              t = fmaf(qb.x, kf[4], t); t = fmaf(qb.y, kf[5], t);
              t = fmaf(qb.z, kf[6], t); t = fmaf(qb.w, kf[7], t);
              sg[g] = t;
            }
          }
        }
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g)
          if (g < G) sc[g * kAttnBlock + tid] = sg[g];
      }
      dev::consumer_sync();
      // online softmax: warp g owns head g
      if (warp < G) {
        float* row = sc + warp * kAttnBlock;
        float mx = -INFINITY;
        for (int t = lane; t < nb; t += 32) mx = fmaxf(mx, row[t]);
        mx = dev::warp_max(mx);
        const float mold = mrun[warp];
        const float mnew = fmaxf(mold, mx);
        float sum = 0.f;
        for (int t = lane; t < nb; t += 32) {
          const float e = expf(row[t] - mnew);
          row[t] = e;
          sum += e;
        }
        sum = dev::warp_sum(sum);
        if (lane == 0) {
          const float a = expf(mold - mnew);
          alpha[warp] = a;
          lrun[warp] = lrun[warp] * a + sum;
          mrun[warp] = mnew;
        }
      }
      dev::consumer_sync();
      // P.V: thread (dim pair dp, position group tg)
      {
        const int dp = tid % (HD / 2), tg = tid / (HD / 2);
        float2 acc[kMaxGroup];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) acc[g] = make_float2(0.f, 0.f);
        for (int t = tg; t < nb; t += NGRP) {
          const int u = b0 + t;
          float2 v;
          if (u == pos) v = make_float2(vn[2 * dp], vn[2 * dp + 1]);
          else v = __half22float2(reinterpret_cast<const __half2*>(Vc + (size_t)u * HD)[dp]);
#pragma unroll
          for (int g = 0; g < kMaxGroup; ++g) {
            if (g < G) {
              const float pr = sc[g * kAttnBlock + t];
              acc[g].x = fmaf(pr, v.x, acc[g].x);
              acc[g].y = fmaf(pr, v.y, acc[g].y);
            }
          }
        }
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
          if (g < G) {
            red[(tg * G + g) * HD + 2 * dp] = acc[g].x;
            red[(tg * G + g) * HD + 2 * dp + 1] = acc[g].y;
          }
        }
      }
      dev::consumer_sync();
      for (int e = tid; e < G * HD; e += kConsumerThreads) {
        const int g = e / HD, dd = e - g * HD;
        float sum = 0.f;
        for (int q = 0; q < NGRP; ++q) sum += red[(q * G + g) * HD + dd];
        orun[e] = orun[e] * alpha[g] + sum;
      }
      dev::consumer_sync();
    }
    // publish this item's partial (m, l, unnormalised o)
    float* part = p.partials + (size_t)it * G * (HD + 2);
    for (int e = tid; e < G * HD; e += kConsumerThreads) {
      const int g = e / HD, dd = e - g * HD;
      part[g * (HD + 2) + 2 + dd] = orun[e];
    }
    if (tid < G) {
      part[tid * (HD + 2)] = mrun[tid];
      part[tid * (HD + 2) + 1] = lrun[tid];
    }
    dev::consumer_sync();
    if (tid == 0) {
      dev::fence_acq_rel_gpu();
      const unsigned old = atomicAdd(p.att_ctr + layer * p.KV + j, 1u);
      S.flags[F_LAST] = (old == (unsigned)(nsplit - 1)) ? 1 : 0;
    }
    dev::consumer_sync();
    if (S.flags[F_LAST]) {
      dev::fence_acq_rel_gpu();
      const float* base = p.partials + (size_t)(j * nsplit) * G * (HD + 2);
      const bool skip = fault_here(1);
      for (int e = tid; e < G * HD; e += kConsumerThreads) {
        const int g = e / HD, dd = e - g * HD;
        float M = -INFINITY;
        for (int q = 0; q < nsplit; ++q) M = fmaxf(M, base[((size_t)q * G + g) * (HD + 2)]);
        float Lsum = 0.f, O = 0.f;
        for (int q = 0; q < nsplit; ++q) {
          const float* pq = base + ((size_t)q * G + g) * (HD + 2);
          const float f = expf(pq[0] - M);
          Lsum = fmaf(f, pq[1], Lsum);
          O = fmaf(f, pq[2 + dd], O);
        }
        put(p.obuf + ((size_t)j * G + g) * HD + dd, tag, O / Lsum, skip);
      }
      if (tid == 0) p.att_ctr[layer * p.KV + j] = 0u;
    }
    return true;
  }

  // O projection + residual -> x_ffn.
  __device__ bool stage_o(const LayerW& w, int tok, unsigned tag) {
    stage = ST_O;
    const int2 r = p.ranges[ST_O * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    if (!load_vec(p.obuf, tag, nullptr, p.H * p.hd, nullptr, ss, 30)) return false;
    if (!gemv(ST_O, w, r.x, r.y)) return false;
    const bool skip = fault_here(ST_O);
    bool bad = false;
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      float res;
      if (layer == 0) res = __half2float(p.tok_emb[(size_t)tok * p.d + u]);
      else if (!wait_f(p.x_attn + u, tag, res, 31)) { bad = true; break; }
      put(p.x_ffn + u, tag, res + S.rowacc[u - r.x], skip);
    }
    return !dev::consumer_sync_or(bad);
  }

  // RMSNorm + gate/up GEMV + SwiGLU -> h.
  __device__ bool stage_gu(const LayerW& w, unsigned tag) {
    stage = ST_GU;
    const int2 r = p.ranges[ST_GU * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    if (!load_vec(p.x_ffn, tag, nullptr, p.d, w.ffn_norm, ss, 40)) return false;
    if (!gemv(ST_GU, w, r.x, r.y)) return false;
    const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
    const bool skip = fault_here(ST_GU);
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      const int k = u - r.x;
      const float g = S.rowacc[2 * k] * rs, up = S.rowacc[2 * k + 1] * rs;
      const float sg = g / (1.0f + expf(-g));
      put(p.hbuf + u, tag, sg * up, skip);
    }
    return true;
  }

  // Down GEMV + residual -> x_attn (input of the next layer).
  __device__ bool stage_down(const LayerW& w, unsigned tag, unsigned tag_next) {
    stage = ST_DOWN;
    const int2 r = p.ranges[ST_DOWN * p.grid + blockIdx.x];
    if (r.y <= r.x) return true;
    float ss;
    if (!load_vec(p.hbuf, tag, nullptr, p.F, nullptr, ss, 50)) return false;
    if (!gemv(ST_DOWN, w, r.x, r.y)) return false;
    const bool skip = fault_here(ST_DOWN);
    bool bad = false;
    for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
      float res;
      if (!wait_f(p.x_ffn + u, tag, res, 51)) { bad = true; break; }
      put(p.x_attn + u, tag_next, res + S.rowacc[u - r.x], skip);
    }
    return !dev::consumer_sync_or(bad);
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

  // Final RMSNorm + LM head + argmax; or, on steps that pick no id, only
  // the per-step fenced publish.  Returns false on abort; *tok_out gets the
  // greedy id (uniform across the grid).
  __device__ bool stage_lm(bool pick, int step_row, unsigned tag, int* tok_out) {
    stage = ST_LM;
    float best = -INFINITY;
    int bi = INT_MAX;
    const int2 r = p.ranges[ST_LM * p.grid + blockIdx.x];
    if (pick && r.y > r.x) {
      float ss;
      if (!load_vec(p.x_attn, tag, nullptr, p.d, p.final_norm, ss, 60)) return false;
      if (!gemv(ST_LM, p.layers[0], r.x, r.y)) return false;
      const float rs = 1.0f / sqrtf(ss / (float)p.d + p.eps);
      float* cap = (p.capture && step_row < p.capture_rows)
                       ? p.capture + (size_t)step_row * p.V
                       : nullptr;
      for (int u = r.x + tid; u < r.y; u += kConsumerThreads) {
        const float v = S.rowacc[u - r.x] * rs;
        if (cap) cap[u] = v;
        if (better(v, u, best, bi)) {
          best = v;
          bi = u;
        }
      }
    }
    warp_argmax(best, bi);
    if (lane == 0) {
      S.red[warp] = best;
      S.redi[warp] = bi;
    }
    dev::consumer_sync();
    const bool skip = fault_here(ST_LM);
    if (tid == 0) {
      float b = S.red[0];
      int ib = S.redi[0];
      for (int w = 1; w < kConsumerWarps; ++w)
        if (better(S.red[w], S.redi[w], b, ib)) {
          b = S.red[w];
          ib = S.redi[w];
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
      unsigned vb, ib;
      if (!wait_tag(p.slots + 2 * c, tag, vb, 61) || !wait_tag(p.slots + 2 * c + 1, tag, ib, 62)) {
        bad = true;
        break;
      }
      if (better(__uint_as_float(vb), (int)ib, gb, gi)) {
        gb = __uint_as_float(vb);
        gi = (int)ib;
      }
    }
    // acquire: later loads of KV entries written by other CTAs see them
    dev::fence_acq_rel_gpu();
    warp_argmax(gb, gi);
    if (lane == 0) {
      S.red2[warp] = gb;
      S.redi2[warp] = gi;
    }
    if (dev::consumer_sync_or(bad)) return false;
    float b = S.red2[0];
    int ib = S.redi2[0];
    for (int w = 1; w < kConsumerWarps; ++w)
      if (better(S.red2[w], S.redi2[w], b, ib)) {
        b = S.red2[w];
        ib = S.redi2[w];
      }
    *tok_out = ib;
    if (tid == 0) t_sync += clock64() - c0;
    return true;
  }

  template <int HD>
  __device__ void run() {
    const long long c_begin = clock64();
    int tok = p.forced ? p.forced[0] : p.first_tok;
    int done = 0;
    bool ok = true;
    for (int i = 0; i < p.n_steps && ok; ++i) {
      step = i;
      const int pos = p.pos0 + i;
      for (int l = 0; l < p.L && ok; ++l) {
        layer = l;
        const LayerW& w = p.layers[l];
        const unsigned tag = epoch_of(p, i, l);
        ok = stage_qkv(w, tok, pos, tag) && stage_attn<HD>(pos, tag) && stage_o(w, tok, tag) &&
             stage_gu(w, tag) && stage_down(w, tag, tag + 1u);
      }
      if (!ok) break;
      layer = p.L;
      const bool pick = i >= p.lm_from;
      int next = 0;
      if (!stage_lm(pick, i - p.lm_from, epoch_of(p, i, p.L), &next)) {
        ok = false;
        break;
      }
      done = i + 1;
      if (pick && blockIdx.x == 0 && tid == 0) p.out_ids[i] = next;
      if (pick && p.eos >= 0 && next == p.eos) break;
      if (p.forced && i + 1 < p.n_steps) tok = p.forced[i + 1];
      else tok = next;
    }
    if (tid == 0) S.flags[F_STOP] = 1;
    if (blockIdx.x == 0 && tid == 0) p.status->n_done = done;
    if (tid == 0) {
      u64* st = p.cta_stats + 4 * blockIdx.x;
      st[0] = (u64)(clock64() - c_begin);
      st[1] = (u64)t_sync;
      st[2] = (u64)t_stream;
      st[3] = (u64)done;
    }
  }
};

}  // namespace

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) kie_monokernel(const __grid_constant__ MonoParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const Smem S = carve(p, smem);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.ring_slots; ++s) {
      dev::mbar_init(S.full_s + 8 * s, 1);
      dev::mbar_init(S.empty_s + 8 * s, kConsumerWarps);
    }
    S.flags[F_ABORT] = 0;
    S.flags[F_STOP] = 0;
    S.flags[F_LAST] = 0;
    dev::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) {
      Producer prod(p, S);
      prod.run();
    }
    return;
  }
  Consumer c(p, S);
  c.run<HD>();
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
