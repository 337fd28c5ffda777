// The work units of a GEMV stage on one CTA (shared by the decode kernel,
// its weight repack and the host-side planning query).  Plain data and
// arithmetic only; included by CUDA translation units (min is CUDA's
// host and device overload).
#pragma once

#include "kie_params.h"

namespace kie {

// This CTA's GEMV work in one stage, computed once per launch (plan_units).
// The rows are cut into blocks of nr rows (the last block may be shorter)
// and the kp pieces of a block's rows into S parts (part s: count(s)
// pieces from piece first(s)).  Unit u = (block u / S, part u % S) is one
// ring chunk, stored [row][piece][piece bytes], and warp u % kConsumerWarps
// alone computes it.  With S > 1 a row's S partial sums go to S result
// slots, which row_result adds in part order.
struct StagePlan {
  int rows, kp;          // rows of the CTA in the stage, pieces per row
  int nr, S;             // rows per block, parts per row
  int base, rem;         // part s has base + (s < rem ? 1 : 0) pieces
  int nb;                // blocks: ceil(rows / nr)
  // fp8 streams: index of the stage's first row scale among the CTA's scales
  // of one layer (LM head: of the whole stream), and the scales of a layer
  int sbase, rows_layer;
  int pad[7];
  __host__ __device__ __forceinline__ int first(int s) const { return s * base + min(s, rem); }
  __host__ __device__ __forceinline__ int count(int s) const { return base + (s < rem ? 1 : 0); }
  __host__ __device__ __forceinline__ int block_rows(int b) const { return min(nr, rows - b * nr); }
};
static_assert(sizeof(StagePlan) == 64, "stage plan slot");
// Unit shape of a stage plan's rows x kp pieces: the (rows per block,
// parts) pair with the least estimated time of the busiest warp among those
// whose units fit a chunk of chunk_bytes and whose partial sums fit `slots`
// result words.  A warp runs its units one after another; a unit costs
// (rows x pieces) piece-rows of weights, 0.3 piece-rows per piece for the
// activation load its rows share and 6 for its wait, release and row
// reductions.  Units of one row and one piece always fit (the host keeps
// chunk_bytes >= pb and slots >= rows x ceil(kp / (chunk_bytes / pb))).
__host__ __device__ __forceinline__ void plan_units(StagePlan& pl, int chunk_bytes, int pb,
                                                    int slots) {
  const int R = pl.rows, kp = pl.kp, m = chunk_bytes / pb;
  int best = 0x7fffffff;
  pl.nr = 1;
  pl.S = (kp + m - 1) / m;
  for (int nr = 1; nr <= 4 && (nr == 1 || nr <= R); ++nr) {
    const int nb = (R + nr - 1) / nr;
    for (int S = 1; S <= min(kp, 16); ++S) {
      const int nmax = (kp + S - 1) / S;
      if (nr * nmax > m) continue;
      if (S > 1 && R * S > slots) break;
      const int per_warp = (nb * S + kConsumerWarps - 1) / kConsumerWarps;
      const int cost = per_warp * (10 * nr * nmax + 3 * nmax + 60);
      if (cost < best) {
        best = cost;
        pl.nr = nr;
        pl.S = S;
      }
    }
  }
  pl.base = kp / pl.S;
  pl.rem = kp - pl.base * pl.S;
  pl.nb = (R + pl.nr - 1) / pl.nr;
}

}  // namespace kie
