// Grouped SwiGLU expert GEMMs ("From One Giant FFN to 384 Tiny Experts", section 1:
// y = W_down(SiLU(W_gate u) * W_up u); w1 = gate branch, w3 = value branch, w2 = down projection).
//
// Every routed expert e owns the rows offsets[e] .. offsets[e+1] of the permuted activations; the
// shared expert (group E) owns all T token rows.  Work is split into tiles
//   (group g, 128 weight rows m, token chunk c of <= 128 rows; the CTA-pair kernels below use
//    256 weight rows per pair and chunks of up to 256 rows)
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
// Two kernels share the tile list and the epilogues: expert_gemm_kernel (below, single CTA, the
// fallback for shapes the pairs do not take) and expert_gemm_pair_kernel (further below, clusters of
// two CTAs sharing each MMA; the default, and the only one with the MXFP4 weight variant).
//
// Single-CTA kernel structure (one CTA per SM, persistent, static round-robin over the tile list):
//   warp 0      TMA producer: weight tile(s) [128 x 64] and the chunk's token rows [n x 64] per K step,
//               in the 128-byte swizzled K-major layout the MMA descriptors expect;
//   warp 1      allocates TMEM and issues tcgen05.mma (one thread), committing each stage back to the
//               producer and each finished accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, SwiGLU (or plain cast), bf16 stores.
// Two accumulator buffers in TMEM let the epilogue of tile i overlap the MMAs of tile i+1.
#include "common.cuh"
#include "expert_tiles.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxStages = 8;

constexpr int kCvtSlots = 3;   // MXFP4: most decoded slots (each holding the A tiles of kCvtSteps K steps)
constexpr int kCvtSteps = 1;   // (two steps per slot, with the smem that leaves for 3 stages, was slower)

// MXFP4 decoded slots per chunk size (measured on the V3 layers: two slots with seven stages, 8.7 ms;
// three slots with four or five stages, 5.7 ms; four slots, no better than three).
__host__ __device__ constexpr int cvt_slots(int bn) { return 3; }

struct GemmSmem {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t afull[kMaxStages];        // MXFP4: this CTA's packed weight tiles of a stage have landed
  uint64_t cvt_local[kCvtSlots];     // MXFP4: this CTA's decode warps have filled a slot
  uint64_t cvt_peer[kCvtSlots];      // MXFP4, even CTA: the odd CTA's slot is full (forwarded arrival)
  uint64_t cvt_empty[kCvtSlots];     // MXFP4: the MMAs reading a decoded slot are done
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
  pdl_begin();
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
  // the setup above (shared memory only) overlaps the predecessor's tail; its outputs are read below
  pdl_begin();
  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_prefix[i] = p.chunk_prefix[i];
  for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_offsets[i] = p.offsets[i];
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
            if (kMode == kGemmSwiGLU) {
              const float wr = (p.row_weight != nullptr && t.g < p.E && c0 + i < t.n)
                                   ? p.row_weight[t.out_row + c0 + i] : 1.f;
              o = swiglu(v0[i], v1[i], p.swiglu_limit, wr);
            } else {
              o = half == 0 ? v0[i] : v1[i];
            }
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
// 128 or 256 rows, of which each CTA loads half (whole 128- and 64-row blocks as single TMA boxes,
// the rest in 16-row boxes: the number of TMA operations per K step, not their bytes, limited the
// token-row loads).  Per weight byte this halves the token-row traffic from L2 compared with the
// single-CTA kernel, and the smaller B half leaves room for five pipeline stages.  The even CTA
// issues the MMAs; each CTA's TMEM receives the accumulators of its own weight rows, and each CTA
// runs the epilogue for them: eight epilogue warps (two per TMEM lane quadrant, each taking every
// other 16-token column block; sixteen measured no faster) convert their share into registers,
// release TMEM to the MMA warp, and only then store, so the stores overlap the next tile's MMAs.
// ------------------------------------------------------------------------------------------------
constexpr int kPairBoxRows = 16;

constexpr int kPairThreads = 320;       // producer warp, MMA warp, eight epilogue warps
constexpr int kPairThreadsFp4 = 576;    // ... and eight MXFP4 decode warps
constexpr int pair_epi_warps(bool) { return 8; }
constexpr int kConvWarp0 = 10;
constexpr int kConvWarps = 8;
constexpr int kFp4TileBytes = kGemmBM * 32;   // 128 rows x 64 E2M1 codes
constexpr int kFp4ScaleBytes = kGemmBM * 16;  // 128 rows x 16 block scales (the 8 K steps around this one)

// Pipeline depth that fits in shared memory.  bf16 weights: 40 KB stages (two weight tiles + 64 token
// rows) -> 5, 48 KB -> 4, 32 KB (one weight tile + 128 token rows) -> 6, 24 KB -> 8.  MXFP4 weights
// (three 32 KB decoded slots besides the stages): 20 KB stages -> 5, 28 KB -> 4.
__host__ __device__ constexpr int pair_stages(int mode, int bn, bool fp4 = false) {
  return fp4 ? (bn == 128 ? 5 : 4) : (mode == kGemmSingle ? (bn == 128 ? 8 : 6) : (bn == 128 ? 5 : 4));
}

// prmt.b32 in its default mode: byte i of the result is byte (sel_i & 7) of {b, a} (a = bytes 0-3), or,
// when bit 3 of selector nibble sel_i is set, that byte's top bit replicated over all eight bits.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight E2M1 codes (element i in bits 4i..4i+3 of w: element 2j in the low nibble of byte j) to eight
// bf16 values times the block scale 2^(s-127), given as the bf16 pair scale2.  The magnitudes 0, 0.5,
// 1, 1.5, 2, 3, 4, 6 of codes 0..7 are looked up as the low and high bytes of their bf16 encodings
// (byte permutes over two 8-entry byte tables); a sign-replicating permute of w and w << 4 turns the
// codes' sign bits into byte masks that set the high bytes' sign bits; the bytes are interleaved into
// bf16 pairs and multiplied by the power-of-two scale, exact for every scale in [2, 252].
__device__ __forceinline__ uint4 e2m1x8_to_bf16(uint32_t w, uint32_t scale2) {
  const uint32_t idx = w & 0x77777777u;                 // 3-bit magnitude codes
  const uint32_t lo_a = 0xC0800000u, lo_b = 0xC0804000u;  // low bytes of bf16(0, .5, 1, 1.5 | 2, 3, 4, 6)
  const uint32_t hi_a = 0x3F3F3F00u, hi_b = 0x40404040u;  // high bytes
  const uint32_t L0 = prmt(lo_a, lo_b, idx), L1 = prmt(lo_a, lo_b, idx >> 16);
  const uint32_t w4 = w << 4;                           // byte j's low-nibble sign now at bit 7
  const uint32_t M0 = prmt(w4, w, 0xD9C8u), M1 = prmt(w4, w, 0xFBEAu);  // 0xFF bytes for negative codes
  const uint32_t H0 = prmt(hi_a, hi_b, idx) | (M0 & 0x80808080u);
  const uint32_t H1 = prmt(hi_a, hi_b, idx >> 16) | (M1 & 0x80808080u);
  uint32_t o[4] = {prmt(L0, H0, 0x5140u), prmt(L0, H0, 0x7362u), prmt(L1, H1, 0x5140u), prmt(L1, H1, 0x7362u)};
  const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162*>(&scale2);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&o[q]), sc);
    o[q] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// bf16 pair holding 2^(s-127) twice; s is first clamped to [2, 252] (reported when outside), the
// range in which every scaled E2M1 value is a normal bf16 number.
__device__ __forceinline__ uint32_t scale_pair(uint32_t s, ErrorWord* ew) {
  if (s < 2u || s > 252u) {
    record_error(ew, MOE_ERR_DEVICE, 0x10000 + (int)s);
    s = s < 2u ? 2u : 252u;
  }
  return (s << 7) | (s << 23);
}

// kBN: token chunk (128 or 256 rows).  With 256, the two accumulators fill TMEM, so the epilogue of
// one tile and the MMAs of the next take turns instead of overlapping.
// kFp4: the weights are MXFP4 (E2M1 codes, 1x32 blocks of UE8M0 scales; "From One Giant FFN to 384
// Tiny Experts", section 11.6).  TMA stages the packed codes (a quarter of the bf16 bytes) next to
// the token rows; eight converter warps per CTA decode each stage's weight rows (a row per thread)
// into bf16 tiles in the 128-byte swizzled layout of a TMA load, in a ring of three slots that the
// MMA reads as its A operand.  The decoded weights are exact, so the MMAs are those of bf16 weights.
template <int kMode, int kBN, bool kFp4>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFp4 ? kPairThreadsFp4 : kPairThreads, 1)
    expert_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                            const __grid_constant__ CUtensorMap map_b_routed,
                            const __grid_constant__ CUtensorMap map_b_shared,
                            const __grid_constant__ CUtensorMap map_s0, const __grid_constant__ CUtensorMap map_s1,
                            const __grid_constant__ CUtensorMap map_bw_routed,
                            const __grid_constant__ CUtensorMap map_bw_shared,
                            const __grid_constant__ CUtensorMap map_bx_routed,
                            const __grid_constant__ CUtensorMap map_bx_shared, GemmParams p) {
  constexpr bool kDual = kMode != kGemmSingle;            // two weight tiles and two accumulators per CTA
  constexpr int kNA = kDual ? 2 : 1;
  constexpr int kPairStages = pair_stages(kMode, kBN, kFp4);
  constexpr int kABytes = kGemmBM * 128;                  // 128 rows x 64 bf16
  constexpr int kBBytes = (kBN / 2) * 128;                // up to kBN/2 token rows x 64 bf16
  constexpr int kAStageBytes = kNA * (kFp4 ? kFp4TileBytes + kFp4ScaleBytes : kABytes);
  constexpr int kStageBytes = kAStageBytes + kBBytes;
  constexpr int kCvtStepBytes = kNA * kABytes;           // decoded A tiles of one K step
  constexpr int kCvtSlotBytes = kCvtSteps * kCvtStepBytes;
  constexpr int kSlots = cvt_slots(kBN);
  constexpr int kCvtBytes = kFp4 ? kSlots * kCvtSlotBytes : 0;
  constexpr int kAccCols = (kDual ? 2 : 1) * kBN;         // accumulators of up to kBN columns
  constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
  constexpr int kTmemCols = 512;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* cvt = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem = cvt + kCvtBytes;                        // pipeline stages
  GemmSmem* sm = reinterpret_cast<GemmSmem*>(smem + kPairStages * kStageBytes);
  int* s_prefix = reinterpret_cast<int*>(sm + 1);         // [E + 2]
  int* s_offsets = s_prefix + (p.E + 2);                  // [E + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int half_rows = p.m_rows / 2;                     // weight rows (features) of this CTA per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
      mbar_init(&sm->afull[s], 1);
    }
    for (int c = 0; c < kSlots; ++c) {
      mbar_init(&sm->cvt_local[c], kConvWarps);   // one arrival per decode warp of this CTA
      mbar_init(&sm->cvt_peer[c], 1);
      mbar_init(&sm->cvt_empty[c], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 2 * pair_epi_warps(kFp4));  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_a0);
    if (kMode == kGemmSwiGLU) tma_prefetch_desc(&map_a1);
    tma_prefetch_desc(&map_b_routed);
    tma_prefetch_desc(&map_b_shared);
    if (kFp4) {
      tma_prefetch_desc(&map_s0);
      if (kMode == kGemmSwiGLU) tma_prefetch_desc(&map_s1);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // the setup above (shared memory only) overlaps the predecessor's tail; its outputs are read below
  pdl_begin();
  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_prefix[i] = p.chunk_prefix[i];
  for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_offsets[i] = p.offsets[i];
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
    // ---------------- TMA producer (both CTAs) ----------------
    // Lane 0 waits for a free stage and loads the weight tiles.  The token rows of a routed tile are
    // either boxes of x_perm (lane 0 alone runs the loop) or, with p.gather_rows, gathered from x:
    // four rows per tile::gather4 load, one load per lane and K step, with loop control uniform
    // across the warp.
    const bool warp_wide = kMode == kGemmSwiGLU && p.gather_rows != nullptr;
    const unsigned pmask = warp_wide ? 0xffffffffu : 1u;
    int st = 0;
    uint32_t ph = 0;
    int last_par[kPairStages];
    for (int s = 0; s < kPairStages; ++s) last_par[s] = -1;
    for (int w = cluster; w < total && (warp_wide || lane == 0); w += nclusters) {
      if (__shfl_sync(pmask, (*abort != 0 || p.test_stall != 0) ? 1 : 0, 0)) break;
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      const bool gather = kMode == kGemmSwiGLU && p.gather_rows != nullptr && t.g < p.E;
      const CUtensorMap* mb = (t.g < p.E) ? &map_b_routed : &map_b_shared;
      const int nmma = (t.n + 31) & ~31;
      const int bhalf = nmma / 2;
      const uint32_t bytes_cta = (kFp4 ? 0 : kAStageBytes) + bhalf * 128;
      const int a_row = t.a_row + rank * half_rows;
      const int a1_row = kMode == kGemmSwiGLU ? a_row : a_row + kGemmBM;
      const CUtensorMap* ma1 = kMode == kGemmSwiGLU ? &map_a1 : &map_a0;
      const int b_row = t.b_row + rank * bhalf;
      // this lane's four gathered rows; rows past the tile's end repeat its first token (their
      // accumulator columns are never stored)
      const bool my_gather = gather && 4 * lane < bhalf;
      int g0 = 0, g1 = 0, g2 = 0, g3 = 0;
      if (my_gather) {
        const int end = t.b_row + t.n, r = b_row + 4 * lane;
        const int pad = gather_row(p, t.b_row);
        g0 = r < end ? gather_row(p, r) : pad;
        g1 = r + 1 < end ? gather_row(p, r + 1) : pad;
        g2 = r + 2 < end ? gather_row(p, r + 2) : pad;
        g3 = r + 3 < end ? gather_row(p, r + 3) : pad;
      }
      for (int kb = 0; kb < nk; ++kb) {
        int got = 1;
        uint8_t* sa0 = smem + st * kStageBytes;
        uint8_t* sb = sa0 + kAStageBytes;
        const uint32_t fb = full_leader + 8u * st;
        if (lane == 0) {
          got = (kFp4 ? mbar_wait_sleepy(&sm->empty[st], ph ^ 1, abort, p.ew, 211, 64)
                      : mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 211))
                    ? 1
                    : 0;
          if (got) {
            last_par[st] = static_cast<int>(ph);
            if (leader) mbar_arrive_expect_tx(&sm->full[st], 2 * bytes_cta);
            if (kFp4) {
              // packed codes and the 16 block scales around this K step into this CTA's stage, counted
              // on its own barrier (the converters wait there)
              const CUtensorMap* ms1 = kMode == kGemmSwiGLU ? &map_s1 : &map_s0;
              uint8_t* ss = sa0 + kNA * kFp4TileBytes;
              mbar_arrive_expect_tx(&sm->afull[st], kAStageBytes);
              tma_load_2d(sa0, &map_a0, &sm->afull[st], kb * 32, a_row);
              tma_load_2d(ss, &map_s0, &sm->afull[st], (kb >> 3) * 16, a_row);
              if (kDual) {
                tma_load_2d(sa0 + kFp4TileBytes, ma1, &sm->afull[st], kb * 32, a1_row);
                tma_load_2d(ss + kFp4ScaleBytes, ms1, &sm->afull[st], (kb >> 3) * 16, a1_row);
              }
            } else {
              tma_load_2d_pair(sa0, &map_a0, fb, kb * 64, a_row);
              if (kDual) tma_load_2d_pair(sa0 + kABytes, ma1, fb, kb * 64, a1_row);
            }
            if (!gather) {
              // whole double-wide and wide boxes first, then 16-row boxes for the rest (bhalf is a
              // multiple of 16)
              const CUtensorMap* mbw = (t.g < p.E) ? &map_bw_routed : &map_bw_shared;
              const CUtensorMap* mbx = (t.g < p.E) ? &map_bx_routed : &map_bx_shared;
              int r = 0;
              if (p.b_wide > 0) {
                for (; r + 2 * p.b_wide <= bhalf; r += 2 * p.b_wide)
                  tma_load_2d_pair(sb + r * 128, mbx, fb, kb * 64, b_row + r);
                for (; r + p.b_wide <= bhalf; r += p.b_wide) tma_load_2d_pair(sb + r * 128, mbw, fb, kb * 64, b_row + r);
              }
              for (; r < bhalf; r += kPairBoxRows) tma_load_2d_pair(sb + r * 128, mb, fb, kb * 64, b_row + r);
            }
          }
        }
        got = __shfl_sync(pmask, got, 0);  // the stage is free for every lane from here on
        if (!got) break;
        if (my_gather) tma_gather4_pair(sb + lane * 512, &map_b_routed, fb, kb * 64, g0, g1, g2, g3);
        if (++st == kPairStages) { st = 0; ph ^= 1; }
      }
    }
    if (lane == 0 && *abort) {  // let every load already issued land before the CTA can exit
      for (int s = 0; s < kPairStages; ++s) {
        if (last_par[s] < 0) continue;
        if (leader) mbar_wait(&sm->full[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
        if (kFp4) mbar_wait(&sm->afull[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA) ----------------
      int st = 0;
      uint32_t ph = 0;
      int cs = 0;
      uint32_t cph = 0;
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
          const int sub = kb % kCvtSteps;                 // MXFP4: K step within the decoded slot
          if (kFp4 && sub == 0) {
            if (!mbar_wait(&sm->cvt_local[cs], cph, abort, p.ew, 215)) { ok = false; break; }
            if (!mbar_wait_cluster(&sm->cvt_peer[cs], cph, abort, p.ew, 218)) { ok = false; break; }
          }
          tc_fence_after();
          const uint32_t sst = smem_u32(smem + st * kStageBytes);
          const uint32_t sa0 = kFp4 ? smem_u32(cvt + cs * kCvtSlotBytes + sub * kCvtStepBytes) : sst;
          const uint64_t a0 = sdesc_kmajor_sw128(sa0);
          const uint64_t a1 = sdesc_kmajor_sw128(sa0 + kABytes);
          const uint64_t b = sdesc_kmajor_sw128(sst + kAStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t accum = (kb | kk) != 0;
            umma_bf16_pair(d0, a0 + 2 * kk, b + 2 * kk, idesc, accum);
            if (kDual) umma_bf16_pair(d0 + kBN, a1 + 2 * kk, b + 2 * kk, idesc, accum);
          }
          umma_commit_pair_both(&sm->empty[st]);
          if (++st == kPairStages) { st = 0; ph ^= 1; }
          if (kFp4 && sub == kCvtSteps - 1) {
            umma_commit_pair_both(&sm->cvt_empty[cs]);
            if (++cs == kSlots) { cs = 0; cph ^= 1; }
          }
        }
        if (!ok) break;
        umma_commit_pair_both(&sm->acc_full[acc]);
        if (++acc == kAccBufs) { acc = 0; acc_ph ^= 1; }
      }
      if (!ok) {
        umma_commit_pair(&sm->drain);
        mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
      }
    } else if (kFp4 && lane == 0) {
      // ---------------- MXFP4, odd CTA: forward "slot full" to the even CTA's MMA thread ----------------
      // One cluster-scope release per decoded slot (instead of one per decode warp and K step): the
      // decode warps' own CTA-scope arrivals are acquired here and passed on.
      const uint32_t peer_leader = cluster_addr(&sm->cvt_peer[0], 0);   // + 8 * slot
      int cs = 0;
      uint32_t cph = 0;
      bool ok = true;
      for (int w = cluster; w < total && ok; w += nclusters) {
        for (int kb = 0; kb < nk; kb += kCvtSteps) {
          if (!mbar_wait_sleepy(&sm->cvt_local[cs], cph, abort, p.ew, 219, 32)) { ok = false; break; }
          mbar_arrive_remote_release(peer_leader + 8u * cs);
          if (++cs == kSlots) { cs = 0; cph ^= 1; }
        }
      }
    }
    __syncwarp();
  } else if (kFp4 && warp >= kConvWarp0) {
    // ---------------- MXFP4 converters (warps 10..17 of both CTAs) ----------------
    // 256 threads per CTA: with two weight tiles, thread ct decodes row ct % 128 of tile ct / 128; with
    // one, the 16-byte output chunks 4h .. 4h+3 (h = ct / 128) of row ct % 128.  Each thread turns 32
    // bytes (or 16) of codes into 128 bytes (or 64) of bf16 per stage.  The two 16-byte halves of a row
    // are read in an order that alternates every four rows, so that eight consecutive rows hit 32
    // distinct banks; the decoded 16-byte chunks are stored with the 128-byte swizzle (chunk j of row r
    // at j ^ (r & 7)), also conflict-free.
    const int ct = (warp - kConvWarp0) * 32 + lane;
    const int r = ct & 127;
    const int a = kNA == 2 ? ct >> 7 : 0;                 // which weight tile
    const int j0 = kNA == 2 ? 0 : 4 * (ct >> 7);          // first output chunk
    const int nj = kNA == 2 ? 8 : 4;
    const int sw = (r >> 2) & 1;
    int st = 0;
    uint32_t ph = 0;
    int cs = 0;
    uint32_t cph = 0;
    bool ok = true;
    for (int w = cluster; w < total && ok; w += nclusters) {
      for (int kb = 0; kb < nk; ++kb) {
        const int sub = kb % kCvtSteps;
        if (sub == 0) {
          if (!mbar_wait_warp_sleepy(&sm->cvt_empty[cs], cph ^ 1, abort, p.ew, 217, 64)) { ok = false; break; }
          mbar_try_wait(&sm->cvt_empty[cs], cph ^ 1);   // per-lane acquire of the completed phase
        }
        if (!mbar_wait_warp_sleepy(&sm->afull[st], ph, abort, p.ew, 216, 32)) { ok = false; break; }
        mbar_try_wait(&sm->afull[st], ph);
        // scales of blocks 2kb, 2kb+1: bytes 2 (kb % 8) and 2 (kb % 8) + 1 of the row's staged 16
        const uint8_t* srow = smem + st * kStageBytes + kNA * kFp4TileBytes + a * kFp4ScaleBytes + r * 16;
        const uint32_t sv = *reinterpret_cast<const unsigned short*>(srow + 2 * (kb & 7));
        const uint32_t sclo = scale_pair(sv & 0xFFu, p.ew), schi = scale_pair(sv >> 8, p.ew);
        const uint8_t* raw = smem + st * kStageBytes + a * kFp4TileBytes + r * 32;
        uint8_t* drow = cvt + cs * kCvtSlotBytes + sub * kCvtStepBytes + a * kABytes + r * 128;
        uint32_t words[8];
        if (kNA == 2) {
          const uint4 first = *reinterpret_cast<const uint4*>(raw + 16 * sw);
          const uint4 second = *reinterpret_cast<const uint4*>(raw + 16 * (sw ^ 1));
          const uint4 lo = sw ? second : first;   // elements 0..31 (block 2kb)
          const uint4 hi = sw ? first : second;   // elements 32..63 (block 2kb+1)
          words[0] = lo.x; words[1] = lo.y; words[2] = lo.z; words[3] = lo.w;
          words[4] = hi.x; words[5] = hi.y; words[6] = hi.z; words[7] = hi.w;
        } else {
          const uint4 half = *reinterpret_cast<const uint4*>(raw + 4 * j0);
          words[0] = half.x; words[1] = half.y; words[2] = half.z; words[3] = half.w;
          words[4] = words[5] = words[6] = words[7] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < nj) {
            const int jj = j0 + j;
            *reinterpret_cast<uint4*>(drow + ((jj ^ (r & 7)) << 4)) = e2m1x8_to_bf16(words[j], jj < 4 ? sclo : schi);
          }
        }
        if (++st == kPairStages) { st = 0; ph ^= 1; }
        if (sub == kCvtSteps - 1) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm->cvt_local[cs]);
          if (++cs == kSlots) { cs = 0; cph ^= 1; }
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    constexpr int kParts = pair_epi_warps(kFp4) / 4;   // epilogue warps per TMEM lane quadrant
    const int q = warp & 3;                     // TMEM lane quadrant
    const int part = (warp - 2) >> 2;           // which 16-token column blocks: part, part + kParts, ...
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
                               (reinterpret_cast<uintptr_t>(s_offsets + (p.E + 1)) + 15) & ~uintptr_t(15)) +
                           (warp - 2) * 16 * 32;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int w = cluster; w < total; w += nclusters) {
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      const bool have = kFp4 ? mbar_wait_warp_backoff(&sm->acc_full[acc], acc_ph, abort, p.ew, 214)
                             : mbar_wait_warp(&sm->acc_full[acc], acc_ph, abort, p.ew, 214);
      if (!have) break;
      tc_fence_after();
      const uint32_t taddr = tmem + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      __nv_bfloat16* out = (t.g < p.E) ? p.out_routed : p.out_shared;
      out += (size_t)t.out_row * p.M_total + t.m * p.m_rows + rank * half_rows + q * 32;
      const float* rw = (p.row_weight != nullptr && t.g < p.E) ? p.row_weight + t.out_row : nullptr;
      constexpr int kNH = kMode == kGemmPair ? 2 : 1;   // output column blocks (two w2 tiles per CTA)
      // one 16-token block of this warp's accumulator lanes -> bf16 pairs (token 2i, 2i + 1)
      auto convert = [&](int c0, uint32_t (&hb)[kNH][8]) {
        float v0[16], v1[16];
        tmem_ld16(taddr + c0, v0);
        if (kDual) tmem_ld16(taddr + kBN + c0, v1);
        tmem_ld_wait();
#pragma unroll
        for (int half = 0; half < kNH; ++half) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float o0, o1;
            if (kMode == kGemmSwiGLU) {
              const float w0 = (rw != nullptr && c0 + 2 * i < t.n) ? rw[c0 + 2 * i] : 1.f;
              const float w1 = (rw != nullptr && c0 + 2 * i + 1 < t.n) ? rw[c0 + 2 * i + 1] : 1.f;
              o0 = swiglu(v0[2 * i], v1[2 * i], p.swiglu_limit, w0);
              o1 = swiglu(v0[2 * i + 1], v1[2 * i + 1], p.swiglu_limit, w1);
            } else {
              o0 = half == 0 ? v0[2 * i] : v1[2 * i];
              o1 = half == 0 ? v0[2 * i + 1] : v1[2 * i + 1];
            }
            hb[half][i] = bf16x2_bits(o0, o1);
          }
        }
      };
      // a 16-token block through this warp's staging buffer into 16-byte stores of whole 64-byte
      // row segments (the token rows past the chunk's end are not stored)
      auto store = [&](int c0, const uint32_t (&hb)[kNH][8]) {
        uint16_t* st16 = reinterpret_cast<uint16_t*>(stage);
#pragma unroll
        for (int half = 0; half < kNH; ++half) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            st16[(2 * i) * 32 + lane] = static_cast<uint16_t>(hb[half][i] & 0xffffu);
            st16[(2 * i + 1) * 32 + lane] = static_cast<uint16_t>(hb[half][i] >> 16);
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
      };
      if constexpr (!kFp4) {
        // The whole accumulator share of this warp (kBN / 32 blocks) is converted into registers and
        // TMEM is handed back to the MMA warp before any store: the next tile's MMAs then overlap
        // this tile's stores, which wait on a memory system that the weight stream keeps busy.
        constexpr int kJ = kBN / 32;
        uint32_t hv[kJ][kNH][8];
#pragma unroll
        for (int j = 0; j < kJ; ++j)
          if (part * 16 + 32 * j < t.n) convert(part * 16 + 32 * j, hv[j]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader + 8u * acc);
#pragma unroll
        for (int j = 0; j < kJ; ++j)
          if (part * 16 + 32 * j < t.n) store(part * 16 + 32 * j, hv[j]);
      } else {
        // MXFP4 kernels (576 threads, fewer registers each): one block at a time, TMEM released last
        for (int c0 = part * 16; c0 < t.n; c0 += 16 * kParts) {
          uint32_t hb[kNH][8];
          convert(c0, hb);
          store(c0, hb);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader + 8u * acc);
      }
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
  return launch_pdl(expert_tiles_kernel, dim3(1), dim3(1024), 0, stream, offsets, E, T, S, bn, chunk_prefix, ew);
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
  return launch_pdl(expert_gemm_kernel<kMode>, dim3(grid), dim3(kGemmThreads), smem, stream, map_a0, map_a1,
                    map_b_routed, map_b_shared, p);
}

size_t expert_gemm_pair_smem_bytes(int mode, int E, int bn, bool fp4) {
  const size_t na = mode == kGemmSingle ? 1 : 2;
  const size_t stage = na * (fp4 ? kFp4TileBytes + kFp4ScaleBytes : kGemmBM * 128) + (size_t)(bn / 2) * 128;
  const size_t cvt = fp4 ? (size_t)cvt_slots(bn) * kCvtSteps * na * kGemmBM * 128 : 0;
  return 1024 + cvt + pair_stages(mode, bn, fp4) * stage + sizeof(GemmSmem) + (2 * (size_t)E + 3) * sizeof(int) +
         16 + (size_t)pair_epi_warps(fp4) * 16 * 32 * 2;
}

template <int kMode, int kBN, bool kFp4>
static cudaError_t launch_pair_mode(const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                                    const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared,
                                    const CUtensorMap& map_s0, const CUtensorMap& map_s1,
                                    const CUtensorMap& map_bw_routed, const CUtensorMap& map_bw_shared,
                                    const CUtensorMap& map_bx_routed, const CUtensorMap& map_bx_shared,
                                    const GemmParams& p, int max_clusters, cudaStream_t stream) {
  const size_t smem = expert_gemm_pair_smem_bytes(kMode, p.E, kBN, kFp4);
  const int threads = kFp4 ? kPairThreadsFp4 : kPairThreads;
  cudaError_t err = cudaFuncSetAttribute(expert_gemm_pair_kernel<kMode, kBN, kFp4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int clusters = max_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, expert_gemm_pair_kernel<kMode, kBN, kFp4>, &cfg) == cudaSuccess &&
      active > 0 && active < clusters)
    clusters = active;
  (void)cudaGetLastError();
  return launch_pdl(expert_gemm_pair_kernel<kMode, kBN, kFp4>, dim3(2 * clusters), dim3(threads), smem, stream,
                    map_a0, map_a1, map_b_routed, map_b_shared, map_s0, map_s1, map_bw_routed, map_bw_shared,
                    map_bx_routed, map_bx_shared, p);
}

cudaError_t launch_expert_gemm_pair(int mode, const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                                    const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared,
                                    const GemmParams& p, int max_clusters, cudaStream_t stream,
                                    const CUtensorMap* map_s0, const CUtensorMap* map_s1,
                                    const CUtensorMap* map_bw_routed, const CUtensorMap* map_bw_shared,
                                    const CUtensorMap* map_bx_routed, const CUtensorMap* map_bx_shared) {
  const bool fp4 = map_s0 != nullptr;
  const CUtensorMap& s0 = fp4 ? *map_s0 : map_a0;
  const CUtensorMap& s1 = fp4 ? *map_s1 : map_a0;
  if (p.b_wide > 0 && (map_bw_routed == nullptr || map_bw_shared == nullptr || map_bx_routed == nullptr ||
                       map_bx_shared == nullptr))
    return cudaErrorInvalidValue;
  const CUtensorMap& bwr = map_bw_routed != nullptr ? *map_bw_routed : map_b_routed;
  const CUtensorMap& bws = map_bw_shared != nullptr ? *map_bw_shared : map_b_shared;
  const CUtensorMap& bxr = map_bx_routed != nullptr ? *map_bx_routed : map_b_routed;
  const CUtensorMap& bxs = map_bx_shared != nullptr ? *map_bx_shared : map_b_shared;
#define MOE_PAIR_CASE(MODE, BN, FP4)                                                                          \
  if (mode == MODE && p.bn == BN && fp4 == FP4)                                                               \
    return launch_pair_mode<MODE, BN, FP4>(map_a0, map_a1, map_b_routed, map_b_shared, s0, s1, bwr, bws, bxr, \
                                           bxs, p, max_clusters, stream);
  MOE_PAIR_CASE(kGemmSwiGLU, 128, false)
  MOE_PAIR_CASE(kGemmSwiGLU, 256, false)
  MOE_PAIR_CASE(kGemmPair, 128, false)
  MOE_PAIR_CASE(kGemmPair, 256, false)
  MOE_PAIR_CASE(kGemmSingle, 128, false)
  MOE_PAIR_CASE(kGemmSingle, 256, false)
  MOE_PAIR_CASE(kGemmSwiGLU, 128, true)
  MOE_PAIR_CASE(kGemmSwiGLU, 256, true)
  MOE_PAIR_CASE(kGemmPair, 128, true)
  MOE_PAIR_CASE(kGemmPair, 256, true)
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
