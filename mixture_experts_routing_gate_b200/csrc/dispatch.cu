// Dispatch: "DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt (bincount of the chosen
// experts, then x[idx] per expert), done as a stable counting sort with no host round trip.
//
//   count   : each block histograms 128 slots in shared memory and writes its row of hist[blk][E];
//   scan    : one block turns the histogram into counts, offsets (exclusive prefix over experts) and
//             the first row of every (block, expert) pair -- stable across blocks;
//   scatter : each block ranks its slots in slot order with warp match/popc (stable within the
//             block), writes row_of_slot / tok_of_row, then copies the token rows of x into x_perm
//             with 16-byte vector loads and streaming stores.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void dispatch_count_kernel(const int32_t* __restrict__ indices, int S, int E, int32_t* __restrict__ hist,
                                      ErrorWord* ew) {
  extern __shared__ int sh_hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh_hist[e] = 0;
  __syncthreads();
  const int s = blockIdx.x * kDispatchSlotsPerBlock + threadIdx.x;
  if (threadIdx.x < kDispatchSlotsPerBlock && s < S) {
    int e = indices[s];
    if (e < 0 || e >= E) {
      record_error(ew, MOE_ERR_DEVICE, e);
      e = e < 0 ? 0 : E - 1;
    }
    atomicAdd(&sh_hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = sh_hist[e];
}

// One block of 1024 threads; thread e owns expert e (E <= 1024).
__global__ void dispatch_scan_kernel(const int32_t* __restrict__ hist, int nblk, int E, int S,
                                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                     int32_t* __restrict__ base) {
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) total += hist[(size_t)b * E + e];
  }
  // block-wide exclusive scan of `total` over e
  const int lane = e & 31, warp = e >> 5;
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    warp_sums[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e < E) {
    counts[e] = total;
    offsets[e] = excl;
    int run = excl;
#pragma unroll 8
    for (int b = 0; b < nblk; ++b) {
      base[(size_t)b * E + e] = run;
      run += hist[(size_t)b * E + e];
    }
  }
  if (e == 0) offsets[E] = S;
}

__global__ void __launch_bounds__(256) dispatch_scatter_kernel(
    const int32_t* __restrict__ indices, int S, int k, int E, const int32_t* __restrict__ base,
    const __nv_bfloat16* __restrict__ x, int d, int32_t* __restrict__ row_of_slot, int32_t* __restrict__ tok_of_row,
    __nv_bfloat16* __restrict__ x_perm) {
  extern __shared__ int sh[];
  int* cursor = sh;                       // [E]
  int* rows = sh + E;                     // [kDispatchSlotsPerBlock]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s0 = blockIdx.x * kDispatchSlotsPerBlock;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] = 0;
  __syncthreads();
  if (warp == 0) {
    for (int c = 0; c < kDispatchSlotsPerBlock / 32; ++c) {
      const int s = s0 + c * 32 + lane;
      int e = -1;
      if (s < S) {
        e = indices[s];
        e = e < 0 ? 0 : (e >= E ? E - 1 : e);  // out-of-range ids were recorded by the count kernel
      }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      int before = 0;
      if (e >= 0) before = cursor[e];
      __syncwarp();
      if (e >= 0 && lane == leader) cursor[e] = before + __popc(peers);
      __syncwarp();
      int row = -1;
      if (e >= 0) {
        row = base[(size_t)blockIdx.x * E + e] + before + rank;
        row_of_slot[s] = row;
        tok_of_row[row] = s / k;
      }
      rows[c * 32 + lane] = row;
    }
  }
  __syncthreads();
  // copy the token rows: one warp per slot, 16-byte vectors, eight loads in flight per lane
  const int nvec = d / 8;
  const int nwarps = blockDim.x >> 5;
  for (int i = warp; i < kDispatchSlotsPerBlock; i += nwarps) {
    const int row = rows[i];
    if (row < 0) continue;
    const int t = (s0 + i) / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * d);
    int v = lane;
    for (; v + 7 * 32 < nvec; v += 8 * 32) {
      uint4 r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) r[u] = __ldg(src + v + u * 32);
#pragma unroll
      for (int u = 0; u < 8; ++u) __stcs(dst + v + u * 32, r[u]);
    }
    for (; v < nvec; v += 32) __stcs(dst + v, __ldg(src + v));
  }
}

cudaError_t launch_dispatch(const int32_t* indices, int S, int k, int E, const __nv_bfloat16* x, int d,
                            int32_t* hist, int32_t* base, int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                            int32_t* tok_of_row, __nv_bfloat16* x_perm, ErrorWord* ew, cudaStream_t stream) {
  const int nblk = dispatch_blocks(S);
  dispatch_count_kernel<<<nblk, kDispatchSlotsPerBlock, E * sizeof(int), stream>>>(indices, S, E, hist, ew);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dispatch_scan_kernel<<<1, 1024, 0, stream>>>(hist, nblk, E, S, counts, offsets, base);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dispatch_scatter_kernel<<<nblk, 256, (E + kDispatchSlotsPerBlock) * sizeof(int), stream>>>(
      indices, S, k, E, base, x, d, row_of_slot, tok_of_row, x_perm);
  return cudaGetLastError();
}

}  // namespace moe
