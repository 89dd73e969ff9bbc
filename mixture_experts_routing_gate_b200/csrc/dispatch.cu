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
//               each row is read once into shared memory and stored k times by the copy engine.
#include "common.cuh"
#include "dispatch_scan.cuh"
#include "kernels.h"

namespace moe {

constexpr int kHistThreads = 512;     // >= the largest E (512): the last block scans one expert per thread
constexpr int kScatterThreads = 128;

__device__ __forceinline__ int clamp_expert(int e, int E) { return e < 0 ? 0 : (e >= E ? E - 1 : e); }

__global__ void __launch_bounds__(kHistThreads) dispatch_histogram_kernel(
    const int32_t* __restrict__ indices, int S, int E, int C, int32_t* __restrict__ hist, int32_t* __restrict__ base,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int* ticket, ErrorWord* ew) {
  pdl_begin();
  extern __shared__ int sh_hist[];  // [E]
  __shared__ int s_last;
  __shared__ int warp_sums[kHistThreads / 32];
  const int lane = threadIdx.x & 31;
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
  // ticket).
  dispatch_finish_scan(hist, (int)gridDim.x, E, S, base, counts, offsets, ticket, warp_sums);
}

// Row copy of the scatter kernel, bulk mode: one thread per block moves every row with the copy
// engine -- each token's row (every segment of it, see RowCopy) is loaded into shared memory once
// (cp.async.bulk, completion on an mbarrier) and stored to its k rows from there (contiguous bulk
// stores), with up to kMaxRowBufs rows in flight; a buffer is reloaded once the stores of the token
// before it no longer read it.  The register mode (rows too long for the buffers) is a warp-per-piece
// copy with 16-byte vectors.
constexpr int kMaxRowBufs = 4;

template <bool kBulk>
__global__ void __launch_bounds__(kScatterThreads) dispatch_scatter_kernel(
    const int32_t* __restrict__ indices, int T, int k, int E, int C, int F, const int32_t* __restrict__ base,
    const int32_t* __restrict__ offsets, int32_t* __restrict__ row_of_slot, int32_t* __restrict__ tok_of_row,
    const float* __restrict__ weights, float* __restrict__ w_perm, RowCopy rc, int nbuf, ErrorWord* ew) {
  extern __shared__ __align__(128) uint8_t sm_raw[];
  int rec_bytes = 0;                            // one row record: every segment, each a multiple of 16 bytes
  for (int g = 0; g < rc.nseg; ++g) rec_bytes += rc.bytes[g];
  uint8_t* bufs = sm_raw;                       // [nbuf][rec_bytes] (bulk mode)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm_raw + (kBulk ? (size_t)nbuf * rec_bytes : 0));   // [nbuf]
  int* cursor = reinterpret_cast<int*>(bars + (kBulk ? kMaxRowBufs : 0));   // [E]: slots of each expert so far
  int* rows = cursor + E;                       // [F * k]: the rows of this block's slots, for the copy
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = T * k;
  const int t0 = blockIdx.x * F, t1 = min(T, t0 + F);
  const int s0 = t0 * k, s1 = t1 * k;
  const int c0 = s0 / C;
  if (kBulk && threadIdx.x == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(&bars[b], 1);
    fence_barrier_init();
  }
  pdl_begin();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] = 0;
  __syncthreads();
  // slots of the coarse block c0 that precede this block's own: eight loads per thread in flight at
  // once, then warp-aggregated counts (the same trip count in every lane)
  for (int p0 = c0 * C; p0 < s0; p0 += 8 * (int)blockDim.x) {
    int ev[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int p = p0 + i * (int)blockDim.x + (int)threadIdx.x;
      ev[i] = p < s0 ? clamp_expert(__ldg(indices + p), E) : -1;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const unsigned peers = __match_any_sync(0xffffffffu, ev[i]);
      if (ev[i] >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cursor[ev[i]], __popc(peers));
    }
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
  if (rc.nseg == 0) return;   // the permutation only (the expert GEMM gathers the rows of x itself)
  if constexpr (kBulk) {
    if (threadIdx.x != 0) return;
    const int ntok = t1 - t0;
    auto load = [&](int b, int tt) {
      mbar_arrive_expect_tx(&bars[b], rec_bytes);
      uint8_t* dst = bufs + (size_t)b * rec_bytes;
      for (int g = 0; g < rc.nseg; ++g) {
        bulk_load(dst, rc.src[g] + (size_t)(t0 + tt) * rc.bytes[g], rc.bytes[g], &bars[b]);
        dst += rc.bytes[g];
      }
    };
    for (int b = 0; b < nbuf && b < ntok; ++b) load(b, b);
    int loaded = min(nbuf, ntok);   // tokens whose load has been issued
    bool ok = true;
    for (int tt = 0; tt < ntok; ++tt) {
      const int b = tt % nbuf;
      if (!mbar_wait(&bars[b], (uint32_t)(tt / nbuf) & 1u, nullptr, ew, 301)) { ok = false; break; }
      const uint8_t* src = bufs + (size_t)b * rec_bytes;
      for (int g = 0; g < rc.nseg; ++g) {
        for (int j = 0; j < k; ++j) bulk_store(rc.dst[g] + (size_t)rows[tt * k + j] * rc.bytes[g], src, rc.bytes[g]);
        src += rc.bytes[g];
      }
      bulk_commit();
      // refill the previous token's buffer once its stores have read it
      if (tt >= 1 && loaded < ntok) {
        bulk_wait_read<1>();
        load((tt - 1) % nbuf, loaded);
        ++loaded;
      }
    }
    if (!ok) {   // a load never landed: wait (bounded) for every load still in flight before leaving
      for (int tt = 0; tt < loaded; ++tt)
        mbar_wait(&bars[tt % nbuf], (uint32_t)(tt / nbuf) & 1u, nullptr, nullptr, 0, 200000000LL);
    }
    bulk_wait_all<0>();
  } else {
    // units of (token, segment, 4 KB piece of the segment), one warp per unit, eight 16-byte loads in
    // flight per lane, then k streaming stores of each vector
    for (int g = 0; g < rc.nseg; ++g) {
      const int nvec = rc.bytes[g] / 16;
      const int npiece = (nvec + 255) / 256;
      const int units = (t1 - t0) * npiece;
      for (int u = warp; u < units; u += blockDim.x >> 5) {
        const int tt = u / npiece, piece = u - tt * npiece;
        const uint4* srcv = reinterpret_cast<const uint4*>(rc.src[g] + (size_t)(t0 + tt) * rc.bytes[g]);
        const int v0 = piece * 256 + lane;
        uint4 r[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (v0 + 32 * i < nvec) r[i] = __ldg(srcv + v0 + 32 * i);
        for (int j = 0; j < k; ++j) {
          uint4* dstv = reinterpret_cast<uint4*>(rc.dst[g] + (size_t)rows[tt * k + j] * rc.bytes[g]);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (v0 + 32 * i < nvec) __stcs(dstv + v0 + 32 * i, r[i]);
        }
      }
    }
  }
}

// dst rows r = src rows tok_of_row[r] for every segment: one warp per (row, segment), 16-byte vectors;
// tokens outside [0, T) are clamped.
__global__ void __launch_bounds__(256) gather_rows_kernel(RowCopy rc, const int32_t* __restrict__ tok_of_row, int S,
                                                          int T) {
  pdl_begin();
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
  const long units = (long)S * rc.nseg;
  for (long u = blockIdx.x * (long)(blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += nwarps) {
    const int r = (int)(u / rc.nseg), g = (int)(u - (long)r * rc.nseg);
    int t = tok_of_row[r];
    t = t < 0 ? 0 : (t >= T ? T - 1 : t);
    const uint4* src = reinterpret_cast<const uint4*>(rc.src[g] + (size_t)t * rc.bytes[g]);
    uint4* dst = reinterpret_cast<uint4*>(rc.dst[g] + (size_t)r * rc.bytes[g]);
    for (int v = lane; v < rc.bytes[g] / 16; v += 32) dst[v] = __ldg(src + v);
  }
}

cudaError_t launch_gather_rows(const RowCopy& rc, const int32_t* tok_of_row, int S, int T, int num_sms,
                               cudaStream_t stream) {
  if (S == 0 || rc.nseg == 0) return cudaSuccess;
  const long want = ((long)S * rc.nseg + 7) / 8;
  const int grid = (int)(want < 4L * num_sms ? want : 4L * num_sms);
  return launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, stream, rc, tok_of_row, S, T);
}

DispatchPlan dispatch_plan(long S, int k, int num_sms) {
  DispatchPlan p;
  // coarse blocks: about 64 of them (at least 1024 slots each, at most 8192, multiples of 256)
  long c = (S + 63) / 64;
  c = (c + 255) / 256 * 256;
  p.coarse = (int)(c < 1024 ? 1024 : (c > 8192 ? 8192 : c));
  p.n_coarse = (int)((S + p.coarse - 1) / p.coarse);
  // fine blocks: about four per SM, 1 to 16 tokens each
  const long T = S / k;
  long f = (T + 4L * num_sms - 1) / (4L * num_sms);
  p.fine_tokens = (int)(f < 1 ? 1 : (f > 16 ? 16 : f));
  p.n_fine = (int)((T + p.fine_tokens - 1) / p.fine_tokens);
  return p;
}

cudaError_t launch_dispatch_scatter(const int32_t* indices, int S, int k, int E, const RowCopy& rc, int coarse,
                                    const int32_t* base, const int32_t* offsets, int32_t* row_of_slot,
                                    int32_t* tok_of_row, ErrorWord* ew, cudaStream_t stream, const float* weights,
                                    float* w_perm) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const DispatchPlan p = dispatch_plan(S, k, sms);
  // bulk row copies when up to kMaxRowBufs row records (at least two) fit in 48 KB of buffers
  size_t rec_bytes = 0;
  for (int g = 0; g < rc.nseg; ++g) rec_bytes += (size_t)rc.bytes[g];
  int nbuf = rec_bytes > 0 ? (int)((48 * 1024) / rec_bytes) : 0;
  nbuf = nbuf > kMaxRowBufs ? kMaxRowBufs : nbuf;
  const bool bulk = rc.nseg > 0 && nbuf >= 2;
  const size_t idx_bytes = (size_t)(E + p.fine_tokens * k) * sizeof(int);
  if (bulk) {
    const size_t smem = (size_t)nbuf * rec_bytes + kMaxRowBufs * sizeof(uint64_t) + idx_bytes;
    cudaError_t err =
        cudaFuncSetAttribute(dispatch_scatter_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(dispatch_scatter_kernel<true>, dim3(p.n_fine), dim3(kScatterThreads), smem, stream, indices,
                      S / k, k, E, coarse, p.fine_tokens, base, offsets, row_of_slot, tok_of_row, weights, w_perm, rc,
                      nbuf, ew);
  }
  return launch_pdl(dispatch_scatter_kernel<false>, dim3(p.n_fine), dim3(kScatterThreads), idx_bytes, stream, indices,
                    S / k, k, E, coarse, p.fine_tokens, base, offsets, row_of_slot, tok_of_row, weights, w_perm, rc, 0,
                    ew);
}

cudaError_t launch_dispatch(const int32_t* indices, int S, int k, int E, const RowCopy& rc, int32_t* hist,
                            int32_t* base, int* ticket, int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                            int32_t* tok_of_row, ErrorWord* ew, cudaStream_t stream, const float* weights,
                            float* w_perm) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const DispatchPlan p = dispatch_plan(S, k, sms);
  cudaError_t err = launch_pdl(dispatch_histogram_kernel, dim3(p.n_coarse), dim3(kHistThreads), E * sizeof(int),
                               stream, indices, S, E, p.coarse, hist, base, counts, offsets, ticket, ew);
  if (err != cudaSuccess) return err;
  return launch_dispatch_scatter(indices, S, k, E, rc, p.coarse, base, offsets, row_of_slot, tok_of_row, ew, stream,
                                 weights, w_perm);
}

}  // namespace moe
