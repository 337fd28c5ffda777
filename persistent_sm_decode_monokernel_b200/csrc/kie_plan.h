// Host-side planning of the persistent decode kernel: which rows of each
// weight matrix every CTA streams, and how its shared memory is carved.
#pragma once

#include <cstdint>
#include <vector>

#include "kie_params.h"

namespace kie {

struct Shape {
  int L, d, H, KV, hd, F, V;
};

// Units of a GEMV stage.  A unit is the smallest piece of work a CTA owns:
//   QKV:  H*hd/2 q RoPE pairs, then KV*hd/2 k RoPE pairs (2 rows each),
//         then KV*hd v rows (1 row each);
//   O:    d rows of Wo;      GU: F (gate row, up row) pairs;
//   DOWN: d rows of Wd;      LM: V rows of the LM head.
int stage_units(const Shape& s, int stage);
int stage_rows(const Shape& s, int stage);
int stage_k(const Shape& s, int stage);
// Rows held by units [ub, ue) of a stage.
int rows_in_range(const Shape& s, int stage, int ub, int ue);

// Contiguous unit ranges for `grid` CTAs, balanced by rows (at most one
// unit apart); the assignment is rotated by a stage-dependent offset so
// that the CTAs holding an extra unit differ from stage to stage.
std::vector<int2> partition(const Shape& s, int grid, int stage);

// Attention shared-memory bytes for group size G and head_dim hd.
int attn_smem_bytes(int G, int hd);

// GEMV result words a CTA with `rows` rows of `kp` pieces needs: one per
// row, and one per row and part when chunks of `chunk_bytes` hold less than
// a row (a row then spans several work units); at least 256, so that the
// kernel's unit planner may split the rows of small shares into parts.
int result_slots(int rows, int kp, int chunk_bytes);
// The result words every CTA of the plan reserves: result_slots of the
// largest need over all stages and CTAs.
int gemv_slots(const Shape& s, const std::vector<std::vector<int2>>& ranges, int grid,
               int chunk_bytes);

// Shared memory carve-up: fixed regions first, the rest (rounded down to
// 512 B) is the weight ring.  Returns false if the ring would be smaller
// than two chunks of `chunk_bytes`.
bool plan_smem(const Shape& s, int grid, int chunk_bytes, int smem_limit,
               const std::vector<std::vector<int2>>& ranges, SmemLayout* out, int* ring_bytes);

// Bytes of CTA `cta`'s one-token weight stream (all layers + LM head) with
// `elem_bytes` bytes per weight (2: fp16, 1: fp8).
size_t stream_bytes(const Shape& s, const std::vector<std::vector<int2>>& ranges, int cta,
                    int elem_bytes = 2);
// Rows of CTA `cta`'s one-token stream (all layers + LM head): the number of
// row scales of an fp8 stream.
size_t stream_rows(const Shape& s, const std::vector<std::vector<int2>>& ranges, int cta);

}  // namespace kie
