// The ragged tile list of the grouped expert GEMMs (expert_gemm.cu, expert_gemm_mx.cu): tile w of the
// list is (group g, weight-row tile m, token chunk c), groups 0..E-1 the routed experts on their rows
// offsets[g] .. offsets[g+1] of the permuted activations and group E the shared expert on all T
// tokens; chunk_prefix[g] counts the token chunks of the groups before g.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {

struct TileInfo {
  int g;        // group (E = shared expert)
  int a_row;    // first weight row in the stacked [(E+1) * M_total, K] weight matrix
  int b_row;    // first token row in the B tensor map
  int out_row;  // first output row (in out_routed, or in out_shared for the shared expert)
  int n;        // valid token rows (1..bn)
  int m;        // weight-row tile index
};

// Token (row of x) of routed row r, clamped into [0, T) so that a gathered load stays in bounds.
__device__ __forceinline__ int gather_row(const GemmParams& p, int r) {
  const int v = __ldg(p.gather_rows + r);
  return v < 0 ? 0 : (v >= p.T ? p.T - 1 : v);
}

__device__ __forceinline__ TileInfo decode_tile(int w, const int* prefix, const int* offsets, const GemmParams& p) {
  // largest g in [0, E] with m_tiles * prefix[g] <= w
  int lo = 0, hi = p.E;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.m_tiles * prefix[mid] <= w) lo = mid; else hi = mid - 1;
  }
  TileInfo t;
  t.g = lo;
  const int chunks = prefix[lo + 1] - prefix[lo];
  const int local = w - p.m_tiles * prefix[lo];
  t.m = local / chunks;
  const int c = local - t.m * chunks;
  int rows, first;
  if (lo < p.E) {
    first = offsets[lo];
    rows = offsets[lo + 1] - first;
    t.b_row = first + c * p.bn;
    t.out_row = first + c * p.bn;
  } else {
    rows = p.T;
    t.b_row = p.shared_b_row + c * p.bn;
    t.out_row = c * p.bn;
  }
  t.n = min(p.bn, rows - c * p.bn);
  t.a_row = lo * p.M_total + t.m * p.m_rows;
  return t;
}

}  // namespace moe
