// Dispatch: "DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt (bincount of the chosen
// experts, then x[idx] per expert), done as a stable counting sort in two launches with no host
// round trip and no waiting between blocks.
//
//   histogram : the slots are cut into at most ~64 coarse blocks; each block histograms its slots in
//               shared memory with warp-aggregated atomics (the lanes of one expert, found by
//               match_any, add their number once) and writes its row of hist[blk][E].  The block
//               that finishes last (an atomic ticket) turns the rows into the per-block bases
//               (base[b][e] = slots of e in blocks before b), the counts and the exclusive prefix
//               over the experts (offsets), and re-arms the ticket;
//   scatter   : a fine block of F tokens counts, per expert, the slots of its coarse block that come
//               before its own, ranks its own slots in slot order (match_any / popc, a shared cursor
//               per expert), so that row = offsets[e] + base[c][e] + earlier slots of e (stable
//               across and inside blocks), writes row_of_slot / tok_of_row (and the permuted
//               weights when asked), then copies its tokens' rows of x to their k rows of x_perm:
//               each 4 KB piece of a row is read once and stored k times with 16-byte streaming stores.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kHistThreads = 512;     // >= the largest E (512): the last block scans one expert per thread
constexpr int kScatterThreads = 256;

__device__ __forceinline__ int clamp_expert(int e, int E) { return e < 0 ? 0 : (e >= E ? E - 1 : e); }

__global__ void __launch_bounds__(kHistThreads) dispatch_histogram_kernel(
    const int32_t* __restrict__ indices, int S, int E, int C, int32_t* __restrict__ hist, int32_t* __restrict__ base,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int* ticket, ErrorWord* ew) {
  pdl_begin();
  extern __shared__ int sh_hist[];  // [E]
  __shared__ int s_last;
  __shared__ int warp_sums[kHistThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh_hist[e] = 0;
  __syncthreads();
  const long s_begin = (long)blockIdx.x * C;
  const long s_end = min((long)S, s_begin + C);
  for (long s0 = s_begin; s0 < s_end; s0 += blockDim.x) {   // the same trip count in every lane
    const long s = s0 + threadIdx.x;
    int e = -1;
    if (s < s_end) {
      e = indices[s];
      if (e < 0 || e >= E) {
        record_error(ew, MOE_ERR_DEVICE, e);
        e = clamp_expert(e, E);
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh_hist[e], __popc(peers));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = sh_hist[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;

  // The last block: every other block's row is visible (each fenced its writes before taking its
  // ticket).  Column prefix per expert, eight rows in flight per thread.
  __threadfence();
  const int nblk = gridDim.x;
  const int e = threadIdx.x;   // blockDim.x >= E
  int total = 0;
  if (e < E) {
    int b = 0;
    for (; b + 8 <= nblk; b += 8) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldcg(hist + (size_t)(b + i) * E + e);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        base[(size_t)(b + i) * E + e] = total;
        total += v[i];
      }
    }
    for (; b < nblk; ++b) {
      const int v = __ldcg(hist + (size_t)b * E + e);
      base[(size_t)b * E + e] = total;
      total += v;
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

__global__ void __launch_bounds__(kScatterThreads) dispatch_scatter_kernel(
    const int32_t* __restrict__ indices, int T, int k, int E, int C, int F, const int32_t* __restrict__ base,
    const int32_t* __restrict__ offsets, int32_t* __restrict__ row_of_slot, int32_t* __restrict__ tok_of_row,
    const float* __restrict__ weights, float* __restrict__ w_perm, const __nv_bfloat16* __restrict__ x, int d,
    __nv_bfloat16* __restrict__ x_perm) {
  pdl_begin();
  extern __shared__ int sm[];
  int* cursor = sm;       // [E]: slots of each expert before the one being ranked, from the coarse block's start
  int* rows = sm + E;     // [F * k]: the rows of this block's slots, for the copy
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = T * k;
  const int t0 = blockIdx.x * F, t1 = min(T, t0 + F);
  const int s0 = t0 * k, s1 = t1 * k;
  const int c0 = s0 / C;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] = 0;
  __syncthreads();
  // slots of the coarse block c0 that precede this block's own
  for (int p0 = c0 * C; p0 < s0; p0 += blockDim.x) {
    const int p = p0 + threadIdx.x;
    const int e = p < s0 ? clamp_expert(indices[p], E) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cursor[e], __popc(peers));
  }
  __syncthreads();
  // this block's slots, ranked in slot order by one warp (out-of-range ids were recorded by the
  // histogram kernel and are clamped the same way here)
  if (warp == 0) {
    const int* base_c = base + (size_t)c0 * E;
    for (int sb = s0; sb < s1; sb += 32) {
      const int s = sb + lane;
      const int e = s < s1 ? clamp_expert(indices[s], E) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int before = e >= 0 ? cursor[e] : 0;
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) cursor[e] = before + __popc(peers);
      __syncwarp();
      if (e >= 0) {
        int row = offsets[e] + base_c[e] + before + rank;
        row = row < 0 ? 0 : (row >= S ? S - 1 : row);   // never leaves the buffers, whatever the inputs
        row_of_slot[s] = row;
        tok_of_row[row] = s / k;
        if (w_perm != nullptr) w_perm[row] = weights[s];
        rows[s - s0] = row;
      }
    }
  }
  __syncthreads();
  if (x_perm == nullptr) return;   // the expert GEMM gathers the rows of x itself
  // x_perm[rows[t*k + j]] = x[t]: units of (token, 4 KB piece of its row), one warp per unit, eight
  // 16-byte loads in flight per lane, then k streaming stores of each vector
  const int nvec = d / 8;
  const int npiece = (nvec + 255) / 256;
  const int units = (t1 - t0) * npiece;
  for (int u = warp; u < units; u += blockDim.x >> 5) {
    const int tt = u / npiece, piece = u - tt * npiece;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(t0 + tt) * d);
    const int v0 = piece * 256 + lane;
    uint4 r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (v0 + 32 * i < nvec) r[i] = __ldg(src + v0 + 32 * i);
    for (int j = 0; j < k; ++j) {
      uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)rows[tt * k + j] * d);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (v0 + 32 * i < nvec) __stcs(dst + v0 + 32 * i, r[i]);
    }
  }
}

DispatchPlan dispatch_plan(long S, int k, int num_sms) {
  DispatchPlan p;
  // coarse blocks: about 64 of them (at least 1024 slots each, at most 8192, multiples of 256)
  long c = (S + 63) / 64;
  c = (c + 255) / 256 * 256;
  p.coarse = (int)(c < 1024 ? 1024 : (c > 8192 ? 8192 : c));
  p.n_coarse = (int)((S + p.coarse - 1) / p.coarse);
  // fine blocks: about two per SM, 1 to 16 tokens each
  const long T = S / k;
  long f = (T + 2L * num_sms - 1) / (2L * num_sms);
  p.fine_tokens = (int)(f < 1 ? 1 : (f > 16 ? 16 : f));
  p.n_fine = (int)((T + p.fine_tokens - 1) / p.fine_tokens);
  return p;
}

cudaError_t launch_dispatch(const int32_t* indices, int S, int k, int E, const __nv_bfloat16* x, int d,
                            int32_t* hist, int32_t* base, int* ticket, int32_t* counts, int32_t* offsets,
                            int32_t* row_of_slot, int32_t* tok_of_row, __nv_bfloat16* x_perm, ErrorWord* ew,
                            cudaStream_t stream, const float* weights, float* w_perm) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const DispatchPlan p = dispatch_plan(S, k, sms);
  cudaError_t err = launch_pdl(dispatch_histogram_kernel, dim3(p.n_coarse), dim3(kHistThreads), E * sizeof(int),
                               stream, indices, S, E, p.coarse, hist, base, counts, offsets, ticket, ew);
  if (err != cudaSuccess) return err;
  const size_t smem = (size_t)(E + p.fine_tokens * k) * sizeof(int);
  return launch_pdl(dispatch_scatter_kernel, dim3(p.n_fine), dim3(kScatterThreads), smem, stream, indices, S / k, k,
                    E, p.coarse, p.fine_tokens, base, offsets, row_of_slot, tok_of_row, weights, w_perm, x, d,
                    x_perm);
}

}  // namespace moe
