#include "kie_plan.h"

#include <algorithm>

namespace kie {

int stage_units(const Shape& s, int stage) {
  switch (stage) {
    case ST_QKV: return s.H * s.hd / 2 + s.KV * s.hd / 2 + s.KV * s.hd;
    case ST_O: return s.d;
    case ST_GU: return s.F;
    case ST_DOWN: return s.d;
    case ST_LM: return s.V;
  }
  return 0;
}

int stage_rows(const Shape& s, int stage) {
  switch (stage) {
    case ST_QKV: return (s.H + 2 * s.KV) * s.hd;
    case ST_GU: return 2 * s.F;
    default: return stage_units(s, stage);
  }
}

int stage_k(const Shape& s, int stage) {
  switch (stage) {
    case ST_QKV: return s.d;
    case ST_O: return s.H * s.hd;
    case ST_GU: return s.d;
    case ST_DOWN: return s.F;
    case ST_LM: return s.d;
  }
  return 0;
}

// rows held by units [0, u)
static long long cum_rows(const Shape& s, int stage, long long u) {
  if (stage == ST_QKV) {
    const long long np = (long long)(s.H + s.KV) * s.hd / 2;
    return u <= np ? 2 * u : 2 * np + (u - np);
  }
  if (stage == ST_GU) return 2 * u;
  return u;
}

// unit boundary whose cumulative row count is nearest to `rows`
// (ties to the lower boundary)
static int unit_at_rows(const Shape& s, int stage, long long rows) {
  if (stage == ST_QKV) {
    const long long np = (long long)(s.H + s.KV) * s.hd / 2;
    if (rows <= 2 * np) return (int)(rows / 2);
    return (int)(np + (rows - 2 * np));
  }
  if (stage == ST_GU) return (int)(rows / 2);
  return (int)rows;
}

int rows_in_range(const Shape& s, int stage, int ub, int ue) {
  return (int)(cum_rows(s, stage, ue) - cum_rows(s, stage, ub));
}

std::vector<int2> partition(const Shape& s, int grid, int stage) {
  const long long R = stage_rows(s, stage);
  std::vector<int> bound(grid + 1);
  for (int v = 0; v <= grid; ++v) {
    long long target = (R * v + grid / 2) / grid;
    bound[v] = unit_at_rows(s, stage, target);
  }
  bound[grid] = stage_units(s, stage);
  // O and down share one partition: the CTA that owns residual row r in the
  // O stage owns it in the down stage too, so the residual stream of its
  // rows never leaves the CTA.
  const int rot = ((stage == ST_DOWN ? ST_O : stage) * 41) % grid;
  std::vector<int2> r(grid);
  for (int c = 0; c < grid; ++c) {
    const int v = (c + rot) % grid;
    r[c] = make_int2(bound[v], bound[v + 1]);
  }
  return r;
}

int attn_smem_bytes(int G, int hd) {
  const int tiles = 2 * kMaxGroup * (hd + 8) * 2 +   // q as fp16 hi and lo tiles
                    kMaxGroup * (kAttnBlock + 8) * 2;  // P tile, fp16
  int b = tiles;
  // scores; the combine's scratch reuses the tiles and the scores
  b += std::max(G * kAttnBlock * 4, kCombineBytesPerHead * G - tiles);
  b += 2 * hd * 4;                   // current position's k and v
  b += G * hd * 4;                   // running output
  b += 4 * kMaxGroup * 4;            // running max, sum, rescale, spare
  return b;
}

static int align_up(int x, int a) { return (x + a - 1) / a * a; }

int result_slots(int rows, int kp, int chunk_bytes) {
  const int per_chunk = std::max(1, chunk_bytes / kPieceBytes);
  const int parts = (kp + per_chunk - 1) / per_chunk;
  return std::max(256, rows * parts);
}

int gemv_slots(const Shape& s, const std::vector<std::vector<int2>>& ranges, int grid,
               int chunk_bytes) {
  int slots = 0;
  for (int st = 0; st < N_STAGES; ++st)
    for (int c = 0; c < grid; ++c)
      slots = std::max(slots, result_slots(rows_in_range(s, st, ranges[st][c].x, ranges[st][c].y),
                                           stage_k(s, st) / kPieceElems, chunk_bytes));
  return slots;
}

bool plan_smem(const Shape& s, int grid, int chunk_bytes, int smem_limit,
               const std::vector<std::vector<int2>>& ranges, SmemLayout* out, int* ring_bytes) {
  const int G = s.H / s.KV;
  const int kmax = std::max(std::max(s.d, s.H * s.hd), s.F);
  SmemLayout L{};
  int maxrows = 0;
  for (int st = 0; st < N_STAGES; ++st)
    for (int c = 0; c < grid; ++c)
      maxrows = std::max(maxrows, rows_in_range(s, st, ranges[st][c].x, ranges[st][c].y));
  const int slots = gemv_slots(s, ranges, grid, chunk_bytes);
  // fp16 input vector; the area also holds the attention scratch and the
  // top-k / top-p selection of the LM-head pick
  L.xs_bytes = align_up(std::max(std::max(kmax * 2, attn_smem_bytes(G, s.hd)),
                                 filter_smem_bytes(maxrows, grid)),
                        128);
  L.rowacc_rows = slots;
  int maxres = 0;
  for (int c = 0; c < grid; ++c)
    maxres = std::max(maxres, rows_in_range(s, ST_O, ranges[ST_O][c].x, ranges[ST_O][c].y));
  L.resid_rows = maxres;
  const int bars = 2 * kRingBars * 8;
  const int misc = align_up(kMiscHead * 4 + 2 * maxres * 4 + N_STAGES * 64, 128);  // + stage plans
  const int fixed = align_up(bars, 128) + L.xs_bytes + align_up(slots * 4, 128) + misc;
  const int ring = (smem_limit - fixed) / 512 * 512;
  if (ring < 2 * chunk_bytes) return false;
  L.ring_off = 0;
  L.bar_off = ring;
  L.xs_off = L.bar_off + align_up(bars, 128);
  L.rowacc_off = L.xs_off + L.xs_bytes;
  L.misc_off = L.rowacc_off + align_up(slots * 4, 128);
  L.total = L.misc_off + misc;
  *out = L;
  *ring_bytes = ring;
  return L.total <= smem_limit;
}

size_t stream_bytes(const Shape& s, const std::vector<std::vector<int2>>& ranges, int cta,
                    int elem_bytes) {
  size_t layer = 0;
  for (int st = ST_QKV; st <= ST_DOWN; ++st)
    layer += (size_t)rows_in_range(s, st, ranges[st][cta].x, ranges[st][cta].y) * stage_k(s, st) *
             elem_bytes;
  const size_t lm =
      (size_t)rows_in_range(s, ST_LM, ranges[ST_LM][cta].x, ranges[ST_LM][cta].y) * s.d * elem_bytes;
  return (size_t)s.L * layer + lm;
}

size_t stream_rows(const Shape& s, const std::vector<std::vector<int2>>& ranges, int cta) {
  size_t layer = 0;
  for (int st = ST_QKV; st <= ST_DOWN; ++st)
    layer += (size_t)rows_in_range(s, st, ranges[st][cta].x, ranges[st][cta].y);
  return (size_t)s.L * layer +
         (size_t)rows_in_range(s, ST_LM, ranges[ST_LM][cta].x, ranges[ST_LM][cta].y);
}

}  // namespace kie
