// Grouped SwiGLU expert GEMMs ("From One Giant FFN to 384 Tiny Experts", section 1:
// y = W_down(SiLU(W_gate u) * W_up u); w1 = gate branch, w3 = value branch, w2 = down projection).
//
// Every routed expert e owns the rows offsets[e] .. offsets[e+1] of the permuted activations; the
// shared expert (group E) owns all T token rows.  Work is split into tiles
//   (group g, 128 weight rows m, token chunk c of <= 128 rows)
// and the weights are the MMA's M operand ("swap AB"): a tile computes D[128 x n] = W_tile . X_chunk^T
// with n = the chunk's rows rounded up to 16, so a ragged expert wastes at most 15 token columns
// instead of up to 127 token rows.
//
// Two launches of one kernel template (kMode):
//   kSwiGLU : D_g = W1 . X^T and D_v = W3 . X^T share each X tile; the epilogue writes
//             h = bf16(silu(D_g) * D_v) into H[row, m] (H is [S + T, I]);
//   kPair   : D = W2 . H^T for two adjacent 128-row weight tiles sharing each H tile (halves the
//             L2 -> SM traffic of H per weight byte); the epilogue writes bf16(D) into out[row, m];
//   kSingle : as kPair with one weight tile (used when the output width is an odd multiple of 128).
//
// Kernel structure (one CTA per SM, persistent, static round-robin over the device-built tile list):
//   warp 0      TMA producer: weight tile(s) [128 x 64] and the chunk's token rows [n x 64] per K step,
//               in the 128-byte swizzled K-major layout the MMA descriptors expect;
//   warp 1      allocates TMEM and issues tcgen05.mma (one thread), committing each stage back to the
//               producer and each finished accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, SwiGLU (or plain cast), bf16 stores.
// Two accumulator buffers in TMEM let the epilogue of tile i overlap the MMAs of tile i+1.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxStages = 8;

struct GemmSmem {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int total_tiles;
};

// chunk_prefix[g] = sum over groups h < g of ceil(rows_h / bn); rows of the shared group E = T.
__global__ void expert_tiles_kernel(const int32_t* __restrict__ offsets, int E, int T, int S, int bn,
                                    int32_t* __restrict__ chunk_prefix, ErrorWord* ew) {
  __shared__ int warp_sums[32];
  const int g = threadIdx.x;  // blockDim = 1024 >= E + 1
  int rows = 0;
  if (g < E) {
    const int a = offsets[g], b = offsets[g + 1];
    if (a < 0 || b < a || b > S) {
      record_error(ew, MOE_ERR_DEVICE, g);
    } else {
      rows = b - a;
    }
  } else if (g == E) {
    rows = T;
  }
  const int chunks = (rows + bn - 1) / bn;
  const int lane = g & 31, warp = g >> 5;
  int incl = chunks;
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
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int excl = incl - chunks + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (g <= E) chunk_prefix[g] = excl;
  if (g == E) chunk_prefix[E + 1] = excl + chunks;
}

struct TileInfo {
  int g;        // group (E = shared expert)
  int a_row;    // first weight row in the stacked [(E+1) * M_total, K] weight matrix
  int b_row;    // first token row in the B tensor map
  int out_row;  // first output row (in out_routed, or in out_shared for the shared expert)
  int n;        // valid token rows (1..bn)
  int m;        // weight-row tile index
};

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

template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                       const __grid_constant__ CUtensorMap map_b_routed,
                       const __grid_constant__ CUtensorMap map_b_shared, GemmParams p) {
  constexpr bool kDual = kMode != kGemmSingle;           // two weight tiles and two accumulators
  constexpr int kABytes = kGemmBM * 128;                 // 128 rows x 64 bf16
  constexpr int kBBytes = kGemmBN * 128;                 // up to 128 token rows x 64 bf16
  constexpr int kStageBytes = (kDual ? 2 : 1) * kABytes + kBBytes;
  constexpr int kAccCols = (kDual ? 2 : 1) * kGemmBN;    // fp32 columns of one accumulator buffer
  constexpr int kTmemCols = 2 * kAccCols;                // two buffers
  constexpr int kBoxRows = 32;                           // token rows per B TMA box

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmem* sm = reinterpret_cast<GemmSmem*>(smem + p.stages * kStageBytes);
  int* s_prefix = reinterpret_cast<int*>(sm + 1);        // [E + 2]
  int* s_offsets = s_prefix + (p.E + 2);                 // [E + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_prefix[i] = p.chunk_prefix[i];
  for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_offsets[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 4);   // one arrival per epilogue warp
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_a0);
    if (kDual) tma_prefetch_desc(&map_a1);
    tma_prefetch_desc(&map_b_routed);
    tma_prefetch_desc(&map_b_shared);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) sm->total_tiles = p.m_tiles * s_prefix[p.E + 1];
  __syncthreads();
  const int total = sm->total_tiles;
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int nk = p.K / 64;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int st = 0;
      uint32_t ph = 0;
      int last_par[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) last_par[s] = -1;
      for (int w = blockIdx.x; w < total && !*abort; w += gridDim.x) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const CUtensorMap* mb = (t.g < p.E) ? &map_b_routed : &map_b_shared;
        const int nbox = (t.n + kBoxRows - 1) / kBoxRows;
        const uint32_t bytes = (kDual ? 2 : 1) * kABytes + nbox * kBoxRows * 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 201)) break;
          last_par[st] = static_cast<int>(ph);
          uint8_t* sa0 = smem + st * kStageBytes;
          uint8_t* sb = sa0 + (kDual ? 2 : 1) * kABytes;
          mbar_arrive_expect_tx(&sm->full[st], bytes);
          tma_load_2d(sa0, &map_a0, &sm->full[st], kb * 64, t.a_row);
          if (kMode == kGemmSwiGLU) tma_load_2d(sa0 + kABytes, &map_a1, &sm->full[st], kb * 64, t.a_row);
          if (kMode == kGemmPair) tma_load_2d(sa0 + kABytes, &map_a0, &sm->full[st], kb * 64, t.a_row + kGemmBM);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(sb + bx * kBoxRows * 128, mb, &sm->full[st], kb * 64, t.b_row + bx * kBoxRows);
          if (++st == p.stages) { st = 0; ph ^= 1; }
        }
      }
      if (*abort) {
        for (int s = 0; s < p.stages; ++s)
          if (last_par[s] >= 0) mbar_wait(&sm->full[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int st = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const uint32_t idesc = idesc_bf16_f32(kGemmBM, (t.n + 15) & ~15);
        if (!mbar_wait(&sm->acc_empty[acc], acc_ph ^ 1, abort, p.ew, 202)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem + acc * kAccCols;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->full[st], ph, abort, p.ew, 203)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa0 = smem_u32(smem + st * kStageBytes);
          const uint64_t a0 = sdesc_kmajor_sw128(sa0);
          const uint64_t a1 = sdesc_kmajor_sw128(sa0 + kABytes);
          const uint64_t b = sdesc_kmajor_sw128(sa0 + (kDual ? 2 : 1) * kABytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb | kk) != 0;
            umma_bf16(d0, a0 + 2 * kk, b + 2 * kk, idesc, accum);
            if (kDual) umma_bf16(d0 + kGemmBN, a1 + 2 * kk, b + 2 * kk, idesc, accum);
          }
          umma_commit(&sm->empty[st]);
          if (++st == p.stages) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&sm->acc_full[acc]);
        if (++acc == 2) { acc = 0; acc_ph ^= 1; }
      }
      if (!ok) {
        umma_commit(&sm->drain);
        mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    // A warp owns 32 output features (its TMEM lanes) of the tile.  Each 16-token chunk is rounded to
    // bf16, transposed through a 1 KB per-warp staging buffer, and written as 16-byte vectors: every
    // token row's 32 features (64 contiguous bytes) take four lanes, two store instructions per chunk.
    const int q = warp & 3;                    // TMEM lane quadrant this warp may access
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
                               (reinterpret_cast<uintptr_t>(s_offsets + (p.E + 1)) + 15) & ~uintptr_t(15)) +
                           (warp - 2) * 16 * 32;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      if (!mbar_wait_warp(&sm->acc_full[acc], acc_ph, abort, p.ew, 204)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      __nv_bfloat16* out = (t.g < p.E) ? p.out_routed : p.out_shared;
      out += (size_t)t.out_row * p.M_total + t.m * p.m_rows + q * 32;
      for (int c0 = 0; c0 < t.n; c0 += 16) {
        float v0[16], v1[16];
        tmem_ld16(taddr + c0, v0);
        if (kDual) tmem_ld16(taddr + kGemmBN + c0, v1);
        tmem_ld_wait();
#pragma unroll
        for (int half = 0; half < (kMode == kGemmPair ? 2 : 1); ++half) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float o;
            if (kMode == kGemmSwiGLU) o = silu(v0[i]) * v1[i];
            else o = half == 0 ? v0[i] : v1[i];
            stage[i * 32 + lane] = __float2bfloat16_rn(o);
          }
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int vv = lane + 32 * r, tok = vv >> 2, part = vv & 3;
            if (c0 + tok < t.n) {
              const uint4 val = *reinterpret_cast<const uint4*>(stage + tok * 32 + part * 8);
              *reinterpret_cast<uint4*>(out + (size_t)(c0 + tok) * p.M_total + half * kGemmBM + part * 8) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_ph ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------------------------------------
// CTA-pair variant (clusters of two CTAs, cta_group::2 MMAs of M = 256)
//
// A pair tile covers FB weight rows of one expert -- 256 features of w1 and w3 (SwiGLU: each CTA holds
// the w1 and w3 rows of 128 features), 512 rows of w2 (pair: each CTA holds two adjacent 128-row
// tiles) or 256 rows of w2 (single: one 128-row tile per CTA) -- against one token chunk of up to
// 128 or 256 rows, of which each CTA loads half.  Eight epilogue warps (two per TMEM lane quadrant,
// each taking every other 16-token column block) drain the accumulators.  Per weight byte
// this halves the token-row traffic from L2 compared with the single-CTA kernel, and the smaller B
// half leaves room for five pipeline stages.  The even CTA issues the MMAs; each CTA's TMEM receives
// the accumulators of its own weight rows, and each CTA runs the epilogue for them.
// ------------------------------------------------------------------------------------------------
constexpr int kPairBoxRows = 16;

constexpr int kPairThreads = 320;   // producer warp, MMA warp, eight epilogue warps

// Pipeline depth that fits in shared memory: 40 KB stages (two weight tiles + 64 token rows) -> 5,
// 48 KB -> 4, 32 KB (one weight tile + 128 token rows) -> 6, 24 KB -> 8.
__host__ __device__ constexpr int pair_stages(int mode, int bn) {
  return mode == kGemmSingle ? (bn == 128 ? 8 : 6) : (bn == 128 ? 5 : 4);
}

// kBN: token chunk (128 or 256 rows).  With 256, the two accumulators fill TMEM, so the epilogue of
// one tile and the MMAs of the next take turns instead of overlapping.
template <int kMode, int kBN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                            const __grid_constant__ CUtensorMap map_b_routed,
                            const __grid_constant__ CUtensorMap map_b_shared, GemmParams p) {
  constexpr bool kDual = kMode != kGemmSingle;            // two weight tiles and two accumulators per CTA
  constexpr int kPairStages = pair_stages(kMode, kBN);
  constexpr int kABytes = kGemmBM * 128;                  // 128 rows x 64 bf16
  constexpr int kBBytes = (kBN / 2) * 128;                // up to kBN/2 token rows x 64 bf16
  constexpr int kStageBytes = (kDual ? 2 : 1) * kABytes + kBBytes;
  constexpr int kAccCols = (kDual ? 2 : 1) * kBN;         // accumulators of up to kBN columns
  constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
  constexpr int kTmemCols = 512;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmem* sm = reinterpret_cast<GemmSmem*>(smem + kPairStages * kStageBytes);
  int* s_prefix = reinterpret_cast<int*>(sm + 1);         // [E + 2]
  int* s_offsets = s_prefix + (p.E + 2);                  // [E + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int half_rows = p.m_rows / 2;                     // weight rows (features) of this CTA per tile

  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_prefix[i] = p.chunk_prefix[i];
  for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_offsets[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 16);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_a0);
    if (kMode == kGemmSwiGLU) tma_prefetch_desc(&map_a1);
    tma_prefetch_desc(&map_b_routed);
    tma_prefetch_desc(&map_b_shared);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote signal
  tc_fence_after();
  const int total = p.m_tiles * s_prefix[p.E + 1];
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int nk = p.K / 64;
  const uint32_t full_leader = cluster_addr(&sm->full[0], 0);           // + 8 * stage
  const uint32_t acc_empty_leader = cluster_addr(&sm->acc_empty[0], 0);  // + 8 * buffer

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int st = 0;
      uint32_t ph = 0;
      int last_par[kPairStages];
      for (int s = 0; s < kPairStages; ++s) last_par[s] = -1;
      for (int w = cluster; w < total && !*abort; w += nclusters) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const CUtensorMap* mb = (t.g < p.E) ? &map_b_routed : &map_b_shared;
        const int nmma = (t.n + 31) & ~31;
        const int bhalf = nmma / 2;
        const uint32_t bytes_cta = (kDual ? 2 : 1) * kABytes + bhalf * 128;
        const int a_row = t.a_row + rank * half_rows;
        const int a1_row = kMode == kGemmSwiGLU ? a_row : a_row + kGemmBM;
        const CUtensorMap* ma1 = kMode == kGemmSwiGLU ? &map_a1 : &map_a0;
        const int b_row = t.b_row + rank * bhalf;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 211)) break;
          last_par[st] = static_cast<int>(ph);
          uint8_t* sa0 = smem + st * kStageBytes;
          uint8_t* sb = sa0 + (kDual ? 2 : 1) * kABytes;
          const uint32_t fb = full_leader + 8u * st;
          if (leader) mbar_arrive_expect_tx(&sm->full[st], 2 * bytes_cta);
          tma_load_2d_pair(sa0, &map_a0, fb, kb * 64, a_row);
          if (kDual) tma_load_2d_pair(sa0 + kABytes, ma1, fb, kb * 64, a1_row);
          for (int bx = 0; bx < bhalf / kPairBoxRows; ++bx)
            tma_load_2d_pair(sb + bx * kPairBoxRows * 128, mb, fb, kb * 64, b_row + bx * kPairBoxRows);
          if (++st == kPairStages) { st = 0; ph ^= 1; }
        }
      }
      if (*abort && leader) {
        for (int s = 0; s < kPairStages; ++s)
          if (last_par[s] >= 0) mbar_wait(&sm->full[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA) ----------------
      int st = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int w = cluster; w < total && ok; w += nclusters) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const uint32_t idesc = idesc_bf16_f32(2 * kGemmBM, (t.n + 31) & ~31);
        if (!mbar_wait(&sm->acc_empty[acc], acc_ph ^ 1, abort, p.ew, 212)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem + acc * kAccCols;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->full[st], ph, abort, p.ew, 213)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa0 = smem_u32(smem + st * kStageBytes);
          const uint64_t a0 = sdesc_kmajor_sw128(sa0);
          const uint64_t a1 = sdesc_kmajor_sw128(sa0 + kABytes);
          const uint64_t b = sdesc_kmajor_sw128(sa0 + (kDual ? 2 : 1) * kABytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb | kk) != 0;
            umma_bf16_pair(d0, a0 + 2 * kk, b + 2 * kk, idesc, accum);
            if (kDual) umma_bf16_pair(d0 + kBN, a1 + 2 * kk, b + 2 * kk, idesc, accum);
          }
          umma_commit_pair_both(&sm->empty[st]);
          if (++st == kPairStages) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair_both(&sm->acc_full[acc]);
        if (++acc == kAccBufs) { acc = 0; acc_ph ^= 1; }
      }
      if (!ok) {
        umma_commit_pair(&sm->drain);
        mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    const int q = warp & 3;                     // TMEM lane quadrant
    const int part = (warp - 2) >> 2;           // 0 or 1: which 16-token column blocks
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
                               (reinterpret_cast<uintptr_t>(s_offsets + (p.E + 1)) + 15) & ~uintptr_t(15)) +
                           (warp - 2) * 16 * 32;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int w = cluster; w < total; w += nclusters) {
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      if (!mbar_wait_warp(&sm->acc_full[acc], acc_ph, abort, p.ew, 214)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      __nv_bfloat16* out = (t.g < p.E) ? p.out_routed : p.out_shared;
      out += (size_t)t.out_row * p.M_total + t.m * p.m_rows + rank * half_rows + q * 32;
      for (int c0 = part * 16; c0 < t.n; c0 += 32) {
        float v0[16], v1[16];
        tmem_ld16(taddr + c0, v0);
        if (kDual) tmem_ld16(taddr + kBN + c0, v1);
        tmem_ld_wait();
#pragma unroll
        for (int half = 0; half < (kMode == kGemmPair ? 2 : 1); ++half) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float o;
            if (kMode == kGemmSwiGLU) o = silu(v0[i]) * v1[i];
            else o = half == 0 ? v0[i] : v1[i];
            stage[i * 32 + lane] = __float2bfloat16_rn(o);
          }
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int vv = lane + 32 * r, tok = vv >> 2, sub = vv & 3;
            if (c0 + tok < t.n) {
              const uint4 val = *reinterpret_cast<const uint4*>(stage + tok * 32 + sub * 8);
              *reinterpret_cast<uint4*>(out + (size_t)(c0 + tok) * p.M_total + half * kGemmBM + sub * 8) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader + 8u * acc);
      if (++acc == kAccBufs) { acc = 0; acc_ph ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote signal or MMA of either CTA is outstanding past this point
  if (*abort) {
    // a wait ran out: give any TMA copy this CTA may still have in flight time to land
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
  }
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

cudaError_t launch_expert_tiles(const int32_t* offsets, int E, int T, int S, int bn, int32_t* chunk_prefix,
                                ErrorWord* ew, cudaStream_t stream) {
  expert_tiles_kernel<<<1, 1024, 0, stream>>>(offsets, E, T, S, bn, chunk_prefix, ew);
  return cudaGetLastError();
}

int expert_gemm_stages(int mode) {
  const int stage = (mode == kGemmSingle ? 1 : 2) * kGemmBM * 128 + kGemmBN * 128;
  int stages = (196 * 1024) / stage;
  return stages > kMaxStages ? kMaxStages : stages;
}

size_t expert_gemm_smem_bytes(int mode, int E, int stages) {
  const size_t stage = (size_t)(mode == kGemmSingle ? 1 : 2) * kGemmBM * 128 + kGemmBN * 128;
  return 1024 + stages * stage + sizeof(GemmSmem) + (2 * (size_t)E + 3) * sizeof(int) + 16 + 4 * 16 * 32 * 2;
}

template <int kMode>
static cudaError_t launch_mode(const CUtensorMap& map_a0, const CUtensorMap& map_a1, const CUtensorMap& map_b_routed,
                               const CUtensorMap& map_b_shared, const GemmParams& p, int grid, cudaStream_t stream) {
  const size_t smem = expert_gemm_smem_bytes(kMode, p.E, p.stages);
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  expert_gemm_kernel<kMode><<<grid, kGemmThreads, smem, stream>>>(map_a0, map_a1, map_b_routed, map_b_shared, p);
  return cudaGetLastError();
}

size_t expert_gemm_pair_smem_bytes(int mode, int E, int bn) {
  const size_t stage = (size_t)(mode == kGemmSingle ? 1 : 2) * kGemmBM * 128 + (size_t)(bn / 2) * 128;
  return 1024 + pair_stages(mode, bn) * stage + sizeof(GemmSmem) + (2 * (size_t)E + 3) * sizeof(int) + 16 +
         8 * 16 * 32 * 2;
}

template <int kMode, int kBN>
static cudaError_t launch_pair_mode(const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                                    const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared,
                                    const GemmParams& p, int max_clusters, cudaStream_t stream) {
  const size_t smem = expert_gemm_pair_smem_bytes(kMode, p.E, kBN);
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_pair_kernel<kMode, kBN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int clusters = max_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, expert_gemm_pair_kernel<kMode, kBN>, &cfg) == cudaSuccess &&
      active > 0 && active < clusters)
    clusters = active;
  (void)cudaGetLastError();
  expert_gemm_pair_kernel<kMode, kBN><<<2 * clusters, kPairThreads, smem, stream>>>(map_a0, map_a1, map_b_routed,
                                                                                   map_b_shared, p);
  return cudaGetLastError();
}

cudaError_t launch_expert_gemm_pair(int mode, const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                                    const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared,
                                    const GemmParams& p, int max_clusters, cudaStream_t stream) {
#define MOE_PAIR_CASE(MODE, BN)                                                                          \
  if (mode == MODE && p.bn == BN)                                                                       \
    return launch_pair_mode<MODE, BN>(map_a0, map_a1, map_b_routed, map_b_shared, p, max_clusters, stream);
  MOE_PAIR_CASE(kGemmSwiGLU, 128)
  MOE_PAIR_CASE(kGemmSwiGLU, 256)
  MOE_PAIR_CASE(kGemmPair, 128)
  MOE_PAIR_CASE(kGemmPair, 256)
  MOE_PAIR_CASE(kGemmSingle, 128)
  MOE_PAIR_CASE(kGemmSingle, 256)
#undef MOE_PAIR_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_expert_gemm(int mode, const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                               const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared, const GemmParams& p,
                               int grid, cudaStream_t stream) {
  switch (mode) {
    case kGemmSwiGLU: return launch_mode<kGemmSwiGLU>(map_a0, map_a1, map_b_routed, map_b_shared, p, grid, stream);
    case kGemmPair: return launch_mode<kGemmPair>(map_a0, map_a1, map_b_routed, map_b_shared, p, grid, stream);
    default: return launch_mode<kGemmSingle>(map_a0, map_a1, map_b_routed, map_b_shared, p, grid, stream);
  }
}

}  // namespace moe
