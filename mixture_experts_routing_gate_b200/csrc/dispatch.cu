// Dispatch: "DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt (bincount of the chosen
// experts, then x[idx] per expert), done as a stable counting sort with no host round trip.
//
//   count   : each block histograms 128 slots in shared memory and writes its row of hist[blk][E];
//   colscan : per expert, the total (counts) and the prefix over blocks (base) -- stable across blocks;
//   offsets : exclusive prefix of the counts over the experts;
//   rank    : each block ranks its slots in slot order with warp match/popc (stable within the
//             block) and writes row_of_slot / tok_of_row (and the permuted weights when asked);
//   gather  : x_perm[row_of_slot[s]] = x[s / k], each token's row read once and stored to its k rows
//             with 16-byte vectors and streaming stores, spread evenly over a grid sized to the SM count.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void dispatch_count_kernel(const int32_t* __restrict__ indices, int S, int E, int32_t* __restrict__ hist,
                                      ErrorWord* ew) {
  pdl_begin();
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

// Per-expert column pass over the histogram: block j owns experts 32j .. 32j+31 (one per lane) and
// its 32 warps split the histogram's blocks into contiguous ranges.  Writes counts[e] and
// base[b][e] = the number of slots of expert e in blocks before b (the row offset of block b inside
// expert e's rows, before the expert's own offset is added).
__global__ void __launch_bounds__(1024) dispatch_colscan_kernel(const int32_t* __restrict__ hist, int nblk, int E,
                                                                int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ base) {
  pdl_begin();
  __shared__ int part[32][33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const int per = (nblk + 31) / 32;
  const int b0 = warp * per, b1 = min(nblk, b0 + per);
  int sum = 0;
  if (e < E) {
#pragma unroll 4
    for (int b = b0; b < b1; ++b) sum += hist[(size_t)b * E + e];
  }
  part[warp][lane] = sum;
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int v = part[w][lane];
      part[w][lane] = run;  // exclusive prefix over the warps' ranges
      run += v;
    }
    if (e < E) counts[e] = run;
  }
  __syncthreads();
  if (e < E) {
    int run = part[warp][lane];
#pragma unroll 4
    for (int b = b0; b < b1; ++b) {
      base[(size_t)b * E + e] = run;
      run += hist[(size_t)b * E + e];
    }
  }
}

// Exclusive prefix over the experts' counts (one block of 1024 threads, E <= 1024).
__global__ void __launch_bounds__(1024) dispatch_offsets_kernel(const int32_t* __restrict__ counts, int E, int S,
                                                                int32_t* __restrict__ offsets) {
  pdl_begin();
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  const int total = e < E ? counts[e] : 0;
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
  if (e < E) offsets[e] = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (e == 0) offsets[E] = S;
}

// Ranks 128 slots per block (one warp, 32 slots at a time, in slot order): match_any groups the
// lanes of one expert, popc of the lower lanes gives the rank, and a shared cursor per expert carries
// the count across the four rounds.
__global__ void __launch_bounds__(32) dispatch_rank_kernel(
    const int32_t* __restrict__ indices, int S, int k, int E, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ base, int32_t* __restrict__ row_of_slot, int32_t* __restrict__ tok_of_row,
    const float* __restrict__ weights, float* __restrict__ w_perm) {
  pdl_begin();
  extern __shared__ int cursor[];  // [E]
  const int lane = threadIdx.x;
  const int s0 = blockIdx.x * kDispatchSlotsPerBlock;
  for (int e = lane; e < E; e += 32) cursor[e] = 0;
  __syncwarp();
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
    if (e >= 0) {
      const int row = offsets[e] + base[(size_t)blockIdx.x * E + e] + before + rank;
      row_of_slot[s] = row;
      tok_of_row[row] = s / k;
      if (w_perm != nullptr) w_perm[row] = weights[s];
    }
  }
}

// x_perm[row_of_slot[t*k + j]] = x[t] for j < k.  A unit of work is one token and one 4 KB block of
// its row: a warp loads the block once (eight 16-byte loads in flight per lane) and stores it to the
// token's k rows with streaming stores, so every row of x is read from memory once.  Units are
// strided over a grid sized to the SM count.
__global__ void __launch_bounds__(256) dispatch_gather_kernel(const int32_t* __restrict__ row_of_slot, int T, int k,
                                                              const __nv_bfloat16* __restrict__ x, int d,
                                                              __nv_bfloat16* __restrict__ x_perm) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
  const int nvec = d / 8;                   // 16-byte vectors per row
  const int nblk = (nvec + 255) / 256;      // 4 KB blocks per row
  const long units = (long)T * nblk;
  for (long u = blockIdx.x * (long)(blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += nwarps) {
    const int t = (int)(u / nblk), cb = (int)(u - (long)t * nblk);
    const int my_row = lane < k ? row_of_slot[(size_t)t * k + lane] : 0;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
    const int v0 = cb * 256 + lane;
    uint4 r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (v0 + 32 * i < nvec) r[i] = __ldg(src + v0 + 32 * i);
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xffffffffu, my_row, j);
      uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)row * d);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (v0 + 32 * i < nvec) __stcs(dst + v0 + 32 * i, r[i]);
    }
  }
}

cudaError_t launch_dispatch(const int32_t* indices, int S, int k, int E, const __nv_bfloat16* x, int d,
                            int32_t* hist, int32_t* base, int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                            int32_t* tok_of_row, __nv_bfloat16* x_perm, ErrorWord* ew, cudaStream_t stream,
                            const float* weights, float* w_perm) {
  const int nblk = dispatch_blocks(S);
  cudaError_t err = launch_pdl(dispatch_count_kernel, dim3(nblk), dim3(kDispatchSlotsPerBlock), E * sizeof(int),
                               stream, indices, S, E, hist, ew);
  if (err != cudaSuccess) return err;
  err = launch_pdl(dispatch_colscan_kernel, dim3((E + 31) / 32), dim3(1024), 0, stream, hist, nblk, E, counts, base);
  if (err != cudaSuccess) return err;
  err = launch_pdl(dispatch_offsets_kernel, dim3(1), dim3(1024), 0, stream, counts, E, S, offsets);
  if (err != cudaSuccess) return err;
  err = launch_pdl(dispatch_rank_kernel, dim3(nblk), dim3(32), E * sizeof(int), stream, indices, S, k, E, offsets, base,
                   row_of_slot, tok_of_row, weights, w_perm);
  if (err != cudaSuccess) return err;
  if (x_perm == nullptr) return cudaSuccess;  // the expert GEMM gathers the rows of x itself
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long units = (long)(S / k) * ((d / 8 + 255) / 256);
  const long want = (units + 7) / 8;  // blocks of eight warps
  const int grid = (int)(want < 4L * sms ? want : 4L * sms);
  return launch_pdl(dispatch_gather_kernel, dim3(grid), dim3(256), 0, stream, row_of_slot, S / k, k, x, d, x_perm);
}

}  // namespace moe
