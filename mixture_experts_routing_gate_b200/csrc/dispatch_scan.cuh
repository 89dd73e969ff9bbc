// The last step of dispatch's counting: per-block expert histograms hist[nblk][E] (block b covering
// slots [b*C, (b+1)*C)) turned into the per-block bases base[b][e] (slots of e in the blocks before b),
// the counts and the exclusive prefix over the experts (offsets, offsets[E] = S).  Run by the one
// block of a grid that took the last ticket of an atomic counter (every other block fenced its row
// before taking its ticket); it re-arms the counter.  Used by the histogram kernel (dispatch.cu) and
// by the cluster router's epilogue when the forward fuses the histogram into it (router.cu).
#pragma once

#include "common.cuh"

namespace moe {

// blockDim.x >= E and a multiple of 32; warp_sums: shared memory of blockDim.x / 32 ints.
__device__ __forceinline__ void dispatch_finish_scan(const int32_t* hist, int nblk, int E, int S, int32_t* base,
                                                     int32_t* counts, int32_t* offsets, int* ticket, int* warp_sums) {
  __threadfence();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    constexpr int kBatch = 64;   // up to 64 rows' loads in flight per thread
    for (int b0 = 0; b0 < nblk; b0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) v[i] = b0 + i < nblk ? __ldcg(hist + (size_t)(b0 + i) * E + e) : 0;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (b0 + i < nblk) base[(size_t)(b0 + i) * E + e] = total;
        total += v[i];
      }
    }
    counts[e] = total;
  }
  // exclusive prefix of the counts over the experts
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    if (lane < (int)(blockDim.x >> 5)) warp_sums[lane] = w;   // inclusive prefix of the warp totals
  }
  __syncthreads();
  if (e < E) offsets[e] = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e == 0) {
    offsets[E] = S;
    *ticket = 0;   // every block has taken its ticket: re-armed for the next call
  }
}

}  // namespace moe
