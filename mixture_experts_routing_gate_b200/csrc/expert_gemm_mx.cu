// Grouped SwiGLU expert GEMMs with MXFP4 expert weights on the block-scaled tensor cores ("From One
// Giant FFN to 384 Tiny Experts", section 11.6: expert weights in FP4 E2M1 with a power-of-two scale
// per 1x32 block, computation in FP8 E4M3; everything else in FP8 with UE8M0 scales).
//
// The tile list and the CTA-pair structure are those of expert_gemm.cu's expert_gemm_pair_kernel: a
// pair tile is (group, 256 or 512 weight rows, token chunk of up to kMxMaxChunk rows), the even CTA
// issues the M = 256 MMAs and each CTA loads its own weight rows and half of the chunk's token rows.
// What differs:
//   * operands: TMA (tensor-map type 16U4_ALIGN16B) places every 16 packed E2M1 codes of the weights
//     (8 bytes) in a 16-byte slot of the 128-byte swizzled layout, as kind::mxf8f6f4 reads 4-bit
//     operands, and the token rows are E4M3 bytes: a K step covers 128 elements (four MMAs of K = 32)
//     in 128-byte rows, half the shared-memory bytes of a bf16 K step of 64;
//   * scales: scale warps in each CTA read, with plain 16-byte loads, their weight rows' scales
//     (row-major, 16 bytes per row cover 4 K steps) and the scales of all the chunk's token rows
//     (each CTA's tensor core needs all of B's scales), and rearranges them, a group of 4 K steps at
//     a time, into 512-byte chunks per K step and 128 rows (line l: rows l, l+32, l+64, l+96) in a
//     ring of three groups, so that it runs up to two groups ahead of the MMAs; the MMA thread copies
//     a K step's chunks into TMEM columns next to the accumulators with tcgen05.cp, then issues
//     kind::mxf8f6f4.block_scale MMAs that name the K block's byte of each scale word; tcgen05
//     operations run in issue order, so one set of scale columns serves every K step;
//   * bytes in flight: a weight tile is 8 KB in HBM but 16 KB in shared memory (16 codes per 16-byte
//     slot), and a load takes microseconds to land, so the ring's depth sets the pace when the MMAs
//     are small; token chunks of up to 96 rows (MxShape<true>) take 5 stages of 38 KB, longer ones 4
//     of 46 KB;
//   * token chunks of up to 96 rows get two accumulator buffers (the next tile's MMAs run while the
//     epilogue drains the last one); longer chunks fill TMEM with one;
//   * batches of at most 64 tokens (decode) run one CTA per tile instead of a pair (MxShape solo:
//     M = 128, each CTA loading all of its chunk's token rows): with two rows per expert the MMAs are
//     tiny and a K step's time is the MMA thread's issue of its scale copies and MMAs, so one issuing
//     thread per SM instead of per pair doubles the rate;
//   * the up projection's epilogue quantises h = silu(g) * v to E4M3 with a UE8M0 scale per 32
//     features (one warp's 32 TMEM lanes are one block: the block maximum is a single redux.sync),
//     which the down projection reads as its B operand and B scales.
// TMEM: accumulators in columns 0..447 (one pair of up to 224 columns, or two buffers of two times up
// to 96 at columns 0 / 112 and 224 / 336), then 8 columns of weight scales and 8 of token-row scales; 512 columns are allocated.
#include "common.cuh"
#include "expert_tiles.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMxThreads = 384;       // producer, MMA, eight epilogue warps, two scale warps
constexpr int kMxScaleWarp = 10;      // the first scale warp
constexpr int kMxMaxStages = 5;
constexpr int kMxMaxChunkSlots = 3;
constexpr int kMxTileBytes = kGemmBM * 128;          // 128 weight rows x 128 elements (128 bytes)
constexpr int kMxTileTxBytes = kGemmBM * 64;         // what a weight tile's TMA load counts: the packed
                                                     // codes it reads (half a byte each), not the gaps

// Ring geometry by variant: CTA pairs with token chunks of up to 224 rows (112 token rows x 128
// bytes per CTA in each stage) or of up to 96 rows (smaller stages: room for a fifth), or single CTAs
// with chunks of up to 64 rows (all of them in the CTA's stage).
constexpr int kMxLong = 0, kMxShort = 1, kMxSolo = 2;
template <int kVariant>
struct MxShape {
  static constexpr bool kPair = kVariant != kMxSolo;
  static constexpr int kMaxN = kVariant == kMxLong ? kMxMaxChunk : (kVariant == kMxShort ? kMxTwoBufChunk : kMxSoloChunk);
  static constexpr int kBBytes = (kPair ? kMaxN / 2 : kMaxN) * 128;
  static constexpr int kStageBytes = 2 * kMxTileBytes + kBBytes;   // a multiple of 1024
  static constexpr int kStages = kVariant == kMxShort ? 5 : 4;
  static constexpr int kChunkSlots = kVariant == kMxShort ? 2 : 3;   // scale chunks, one group of 4 K steps each
  static constexpr int kSfStageBytes = kPair ? 0 : 3 * 12 * 512;   // single CTA: cp.async staging of scale rows
};

// Staging of the single-CTA form's scale rows: three groups in flight, each 12 rows x 32 lanes x 16 bytes.
constexpr int kMxSfStageSlots = 3;
constexpr int kMxSfStageSlot = 12 * 512;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The single-CTA forms of the pair operations (the MMA thread of every CTA issues for its own tile).
__device__ __forceinline__ void umma_mx_solo(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tmem_cp_chunk_solo(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
constexpr int kMxStepChunkBytes = 4 * 512;           // one K step: two weight-scale + two token-scale chunks
constexpr int kMxChunkBytes = 4 * kMxStepChunkBytes;  // a group of 4 K steps
constexpr int kMxAccCols = kMxMaxChunk;               // columns of one accumulator of a long chunk
constexpr uint32_t kMxSfaCol = 2 * kMxAccCols;        // 448: weight scales (4 columns per tile)
constexpr uint32_t kMxSfbCol = kMxSfaCol + 8;         // 456: token-row scales (4 columns per 128 rows)
constexpr int kMxBoxRows = 16;
constexpr int kMxWideRows = 64;

struct MxSmem {
  uint64_t full[kMxMaxStages];
  uint64_t empty[kMxMaxStages];
  uint64_t chunk_full[kMxMaxChunkSlots];   // even CTA: both CTAs' scale warps have filled the chunk slot
  uint64_t chunk_empty[kMxMaxChunkSlots];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// E4M3 codes and UE8M0 scales of bf16 rows: one thread per 32-element block (four 16-byte loads,
// two 16-byte stores and one scale byte), blocks strided over a grid sized to the SM count.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, long nblocks,
                                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  pdl_begin();
  for (long b = blockIdx.x * (long)blockDim.x + threadIdx.x; b < nblocks; b += (long)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x) + b * 4;
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldg(src + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
        v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_scale_exponent(amax);
    const float inv = mx_inv_scale(e);
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      q[i] = e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) | (e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
    uint4* dst = reinterpret_cast<uint4*>(codes) + b * 2;
    dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
    dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
    scales[b] = static_cast<uint8_t>(e + 127);
  }
}

cudaError_t launch_quantize_rows(const __nv_bfloat16* x, long R, int d, uint8_t* codes, uint8_t* scales, int num_sms,
                                 cudaStream_t stream) {
  const long nblocks = R * (d / 32);
  if (nblocks == 0) return cudaSuccess;
  const long want = (nblocks + 255) / 256;
  const int grid = (int)(want < 8L * num_sms ? want : 8L * num_sms);
  return launch_pdl(quantize_rows_kernel, dim3(grid), dim3(256), 0, stream, x, nblocks, codes, scales);
}

template <int kMode, int kVariant>
__global__ void __launch_bounds__(kMxThreads, 1)
    expert_gemm_mx_kernel(const __grid_constant__ MxMaps maps, GemmParams p) {
  constexpr bool kSwiGLU = kMode == kGemmSwiGLU;
  using Shape = MxShape<kVariant>;
  constexpr bool kPair = Shape::kPair;   // clusters of two CTAs (launched with a cluster dimension of 2)
  constexpr int kMxStages = Shape::kStages;
  constexpr int kMxStageBytes = Shape::kStageBytes;
  constexpr int kMxChunkSlots = Shape::kChunkSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* chunks = smem + kMxStages * kMxStageBytes;                  // [kMxChunkSlots][kMxChunkBytes]
  uint8_t* epi_stage = chunks + kMxChunkSlots * kMxChunkBytes;         // 8 warps x 1 KB
  uint8_t* sf_stage = epi_stage + 8 * 1024;                             // single CTA: staged scale rows
  MxSmem* sm = reinterpret_cast<MxSmem*>(sf_stage + Shape::kSfStageBytes);
  int* s_prefix = reinterpret_cast<int*>(sm + 1);                      // [E + 2]
  int* s_offsets = s_prefix + (p.E + 2);                               // [E + 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0;
  const bool leader = rank == 0;
  const int cluster = kPair ? (blockIdx.x >> 1) : blockIdx.x, nclusters = kPair ? (gridDim.x >> 1) : gridDim.x;
  const int half_rows = kPair ? p.m_rows / 2 : p.m_rows;   // weight rows of this CTA per tile (128 for SwiGLU, 256 for w2)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int s = 0; s < kMxChunkSlots; ++s) {
      mbar_init(&sm->chunk_full[s], kPair ? 2 : 1);   // one arrival per CTA's scale warp (on the even CTA)
      mbar_init(&sm->chunk_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->acc_full[b], 1);
      mbar_init(&sm->acc_empty[b], kPair ? 16 : 8);   // one arrival per epilogue warp of the tile's CTAs
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&maps.a0);
    tma_prefetch_desc(&maps.a1);
    tma_prefetch_desc(&maps.b_routed);
    tma_prefetch_desc(&maps.b_shared);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(&sm->tmem_base, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&sm->tmem_base, 512);
      tmem_relinquish();
    }
  }
  pdl_begin();
  for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s_prefix[i] = p.chunk_prefix[i];
  for (int i = threadIdx.x; i < p.E + 1; i += blockDim.x) s_offsets[i] = p.offsets[i];
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // both CTAs' barriers are initialised before any remote signal
  tc_fence_after();
  const int total = p.m_tiles * s_prefix[p.E + 1];
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int nk = p.K / 128;   // K steps of 128 elements (K % 512 == 0: a whole number of scale groups)
  // the even CTA's barriers, in the cluster's shared-memory window (pairs only)
  const uint32_t full_leader = kPair ? cluster_addr(&sm->full[0], 0) : smem_u32(&sm->full[0]);
  const uint32_t chunk_full_leader = kPair ? cluster_addr(&sm->chunk_full[0], 0) : smem_u32(&sm->chunk_full[0]);
  const uint32_t acc_empty_leader = kPair ? cluster_addr(&sm->acc_empty[0], 0) : smem_u32(&sm->acc_empty[0]);
  // accumulators: chunks of up to 96 rows (MMA N <= 96) get two buffers (columns 0 and 224), the
  // second accumulator (v, or the second w2 tile) vcol columns after the first
  const bool two_bufs = p.bn <= kMxTwoBufChunk;
  const uint32_t vcol = two_bufs ? kMxAccCols / 2 : kMxAccCols;
  const int sf_row_bytes = p.K / 32;   // scale bytes per row (a multiple of 16)

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int st = 0;
      uint32_t ph = 0;
      int last_par[kMxStages];
      for (int s = 0; s < kMxStages; ++s) last_par[s] = -1;
      for (int w = cluster; w < total && !*abort && p.test_stall == 0; w += nclusters) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const bool routed = t.g < p.E;
        const int nmma = (t.n + 31) & ~31;
        const int bhalf = kPair ? nmma / 2 : nmma;   // this CTA's token rows of the chunk
        const int a_row = t.a_row + rank * half_rows;
        const int a1_row = kSwiGLU ? a_row : a_row + kGemmBM;
        const int b_row = t.b_row + rank * bhalf;
        const uint32_t bytes_cta = 2 * kMxTileTxBytes + bhalf * 128;
        const CUtensorMap* mb = routed ? &maps.b_routed : &maps.b_shared;
        const CUtensorMap* mbw = routed ? &maps.bw_routed : &maps.bw_shared;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 232)) { ok = false; break; }
          last_par[st] = static_cast<int>(ph);
          uint8_t* sa = smem + st * kMxStageBytes;
          uint8_t* sb = sa + 2 * kMxTileBytes;
          const uint32_t fb = full_leader + 8u * st;
          if (leader) mbar_arrive_expect_tx(&sm->full[st], (kPair ? 2 : 1) * bytes_cta);
          auto load = [&](void* dst, const CUtensorMap* map, int c0, int c1) {
            if constexpr (kPair) tma_load_2d_pair(dst, map, fb, c0, c1);
            else tma_load_2d(dst, map, &sm->full[st], c0, c1);
          };
          load(sa, &maps.a0, kb * 128, a_row);
          load(sa + kMxTileBytes, kSwiGLU ? &maps.a1 : &maps.a0, kb * 128, a1_row);
          int r = 0;
          for (; r + kMxWideRows <= bhalf; r += kMxWideRows) load(sb + r * 128, mbw, kb * 128, b_row + r);
          for (; r < bhalf; r += kMxBoxRows) load(sb + r * 128, mb, kb * 128, b_row + r);
          if (++st == kMxStages) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
      if (*abort) {  // let every load already issued land before the CTA can exit
        for (int s = 0; s < kMxStages; ++s)
          if (last_par[s] >= 0 && leader) mbar_wait(&sm->full[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else if (warp >= kMxScaleWarp) {
    // ---------------- scale warps (both CTAs): scales -> 512-byte chunks, a group of 4 K steps at once ----------------
    // Group g of the (tile, group) sequence goes to chunk slot g % kMxChunkSlots.  CTA pairs: the two
    // scale warps take the even and the odd groups, each with its next group's loads in flight while
    // the current one waits for its chunk slot and is written (two groups' loads in flight per CTA).
    const int sw = warp - kMxScaleWarp;
    // Row l + 32 j's 16 bytes hold its 4 K-block scales of each of the group's 4 K steps.
    auto load_group = [&](int w, int kg, uint4 (&va)[2][4], uint4 (&vb)[2][4]) -> int {
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      const int nbchunks = ((t.n + 31) & ~31) > 128 ? 2 : 1;
      const bool routed = t.g < p.E;
      const int a_row = t.a_row + rank * half_rows;
      const uint8_t* pa0 = maps.sa0 + (size_t)(a_row + lane) * sf_row_bytes + kg * 4;
      const uint8_t* pa1 = (kSwiGLU ? maps.sa1 : maps.sa0) +
                           (size_t)((kSwiGLU ? a_row : a_row + kGemmBM) + lane) * sf_row_bytes + kg * 4;
      const uint8_t* sb = routed ? maps.sb_routed : maps.sb_shared;
      const int brows = routed ? maps.sb_routed_rows : maps.sb_shared_rows;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        va[0][j] = __ldg(reinterpret_cast<const uint4*>(pa0 + (size_t)32 * j * sf_row_bytes));
        va[1][j] = __ldg(reinterpret_cast<const uint4*>(pa1 + (size_t)32 * j * sf_row_bytes));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          // token rows past the chunk (the MMA's padding columns) read a clamped row: their products
          // land in accumulator columns that nothing stores
          int r = t.b_row + 128 * c + lane + 32 * j;
          r = r < brows ? r : brows - 1;
          vb[c][j] = (c < nbchunks) ? __ldg(reinterpret_cast<const uint4*>(sb + (size_t)r * sf_row_bytes + kg * 4))
                                    : make_uint4(0, 0, 0, 0);
        }
      }
      return nbchunks;
    };
    // group g's scales (weight rows in ca, token rows in cb): range check, chunk slot, arrival
    auto emit = [&](int g, uint4 (&ca)[2][4], uint4 (&cb)[2][4], int cnb) -> bool {
      const int cs = g % kMxChunkSlots;
      const uint32_t cph = static_cast<uint32_t>(g / kMxChunkSlots) & 1u;   // this slot's use count, mod 2
      // weight scales outside [2, 252] are clamped into it and reported, as in the bf16 decode
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t* u = reinterpret_cast<uint32_t*>(&ca[c][j]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if ((__vcmpltu4(u[i], 0x02020202u) | __vcmpgtu4(u[i], 0xFCFCFCFCu)) != 0u) {
              for (int b = 0; b < 4; ++b) {
                const uint32_t sv = (u[i] >> (8 * b)) & 0xFFu;
                if (sv < 2u || sv > 252u) record_error(p.ew, MOE_ERR_DEVICE, 0x10000 + (int)sv);
              }
              u[i] = __vmaxu4(__vminu4(u[i], 0xFCFCFCFCu), 0x02020202u);
            }
          }
        }
      if (!mbar_wait_warp(&sm->chunk_empty[cs], cph ^ 1, abort, p.ew, 234)) return false;
      uint8_t* ch = chunks + cs * kMxChunkBytes + lane * 16;
#pragma unroll
      for (int sub = 0; sub < 4; ++sub) {
        // chunk c of K step sub: weight tile c (c < 2) or token rows 128 (c - 2) .. (c < 4)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c >= 2 + cnb) break;
          const uint4* v = c < 2 ? ca[c] : cb[c - 2];
          const uint32_t w0 = reinterpret_cast<const uint32_t*>(&v[0])[sub];
          const uint32_t w1 = reinterpret_cast<const uint32_t*>(&v[1])[sub];
          const uint32_t w2 = reinterpret_cast<const uint32_t*>(&v[2])[sub];
          const uint32_t w3 = reinterpret_cast<const uint32_t*>(&v[3])[sub];
          *reinterpret_cast<uint4*>(ch + sub * kMxStepChunkBytes + c * 512) = make_uint4(w0, w1, w2, w3);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&sm->chunk_full[cs]);
        else mbar_arrive_remote_release(chunk_full_leader + 8u * cs);
      }
      return true;
    };
    auto next = [&](int& w, int& kg) {
      kg += 4;
      if (kg >= nk) { kg = 0; w += nclusters; }
    };
    if constexpr (kPair) {
      int w = cluster, kg = 0, g = sw;
      if (sw == 1) next(w, kg);
      bool have = w < total && p.test_stall == 0;
      uint4 ca[2][4], cb[2][4];
      int cnb = have ? load_group(w, kg, ca, cb) : 1;
      while (have) {
        int nw = w, nkg = kg;
        next(nw, nkg);
        next(nw, nkg);
        const bool have_next = nw < total;
        uint4 na[2][4], nb[2][4];
        const int nnb = have_next ? load_group(nw, nkg, na, nb) : 1;
        if (!emit(g, ca, cb, cnb)) break;
        g += 2;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ca[c][j] = na[c][j];
            cb[c][j] = nb[c][j];
          }
        cnb = nnb;
        w = nw;
        kg = nkg;
        have = have_next;
      }
    } else if (sw == 0) {
      // single CTA (chunks of at most 64 token rows), the first scale warp only: each lane copies its
      // 12 rows' 16 bytes of a group into a staging slot with cp.async, three groups in flight, so
      // that the scale rows' memory latency is covered without holding them in registers
      auto issue = [&](int slot, int w, int kg) {
        if (w < total) {
          const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
          const bool routed = t.g < p.E;
          const uint8_t* pa0 = maps.sa0 + (size_t)(t.a_row + lane) * sf_row_bytes + kg * 4;
          const uint8_t* pa1 = (kSwiGLU ? maps.sa1 : maps.sa0) +
                               (size_t)((kSwiGLU ? t.a_row : t.a_row + kGemmBM) + lane) * sf_row_bytes + kg * 4;
          const uint8_t* sb = routed ? maps.sb_routed : maps.sb_shared;
          const int brows = routed ? maps.sb_routed_rows : maps.sb_shared_rows;
          uint8_t* dst = sf_stage + slot * kMxSfStageSlot + lane * 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            int r = t.b_row + lane + 32 * j;   // padding rows read a clamped row (columns nothing stores)
            r = r < brows ? r : brows - 1;
            cp_async16(dst + (0 * 4 + j) * 512, pa0 + (size_t)32 * j * sf_row_bytes);
            cp_async16(dst + (1 * 4 + j) * 512, pa1 + (size_t)32 * j * sf_row_bytes);
            cp_async16(dst + (2 * 4 + j) * 512, sb + (size_t)r * sf_row_bytes + kg * 4);
          }
        }
        cp_async_commit();
      };
      int iw = cluster, ikg = 0;
      if (p.test_stall == 0)
        for (int s = 0; s < kMxSfStageSlots; ++s) {
          issue(s, iw, ikg);
          next(iw, ikg);
        }
      int slot = 0;
      for (int w = cluster, kg = 0, g = 0; w < total && p.test_stall == 0; next(w, kg), ++g) {
        cp_async_wait<kMxSfStageSlots - 1>();   // this group's copies (this lane's own) have landed
        const uint8_t* src = sf_stage + slot * kMxSfStageSlot + lane * 16;
        uint4 ca[2][4], cb[2][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          ca[0][j] = *reinterpret_cast<const uint4*>(src + (0 * 4 + j) * 512);
          ca[1][j] = *reinterpret_cast<const uint4*>(src + (1 * 4 + j) * 512);
          cb[0][j] = *reinterpret_cast<const uint4*>(src + (2 * 4 + j) * 512);
          cb[1][j] = make_uint4(0, 0, 0, 0);
        }
        if (!emit(g, ca, cb, 1)) break;   // (uses the values read: the slot is free once this returns)
        issue(slot, iw, ikg);          // the slot takes the group three ahead
        next(iw, ikg);
        if (++slot == kMxSfStageSlots) slot = 0;
      }
      cp_async_wait<0>();   // no copy into shared memory is left in flight
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA) ----------------
      int st = 0, cs = 0;
      uint32_t ph = 0, cph = 0;
      bool ok = true;
      for (int w = cluster, it = 0; w < total && ok; w += nclusters, ++it) {
        const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
        const int nmma = (t.n + 31) & ~31;
        const int buf = two_bufs ? (it & 1) : 0;
        const uint32_t use = two_bufs ? (it >> 1) : it;
        const uint32_t acc = tmem + buf * kMxAccCols;
        if (!mbar_wait(&sm->acc_empty[buf], (use & 1) ^ 1, abort, p.ew, 235)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm->full[st], ph, abort, p.ew, 236)) { ok = false; break; }
          if ((kb & 3) == 0 && !mbar_wait_cluster(&sm->chunk_full[cs], cph, abort, p.ew, 237)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sc = smem_u32(chunks + cs * kMxChunkBytes + (kb & 3) * kMxStepChunkBytes);
          auto cp = [&](uint32_t col, uint32_t chunk) {
            if constexpr (kPair) tmem_cp_chunk_pair(tmem + col, sdesc_scale_chunk(chunk));
            else tmem_cp_chunk_solo(tmem + col, sdesc_scale_chunk(chunk));
          };
          cp(kMxSfaCol, sc);
          cp(kMxSfaCol + 4, sc + 512);
          cp(kMxSfbCol, sc + 1024);
          if (nmma > 128) cp(kMxSfbCol + 4, sc + 1536);
          const uint32_t sa = smem_u32(smem + st * kMxStageBytes);
          const uint64_t a0 = sdesc_kmajor_sw128(sa);
          const uint64_t a1 = sdesc_kmajor_sw128(sa + kMxTileBytes);
          const uint64_t b = sdesc_kmajor_sw128(sa + 2 * kMxTileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t idesc = idesc_mx_e2m1_e4m3((kPair ? 2 : 1) * kGemmBM, nmma, kk, kk);
            const uint32_t byte = static_cast<uint32_t>(kk) << 30;
            const uint32_t accum = (kb | kk) != 0;
            if constexpr (kPair) {
              umma_mx_pair(acc, a0 + 2 * kk, b + 2 * kk, idesc, (tmem + kMxSfaCol) | byte,
                           (tmem + kMxSfbCol) | byte, accum);
              umma_mx_pair(acc + vcol, a1 + 2 * kk, b + 2 * kk, idesc, (tmem + kMxSfaCol + 4) | byte,
                           (tmem + kMxSfbCol) | byte, accum);
            } else {
              umma_mx_solo(acc, a0 + 2 * kk, b + 2 * kk, idesc, (tmem + kMxSfaCol) | byte,
                           (tmem + kMxSfbCol) | byte, accum);
              umma_mx_solo(acc + vcol, a1 + 2 * kk, b + 2 * kk, idesc, (tmem + kMxSfaCol + 4) | byte,
                           (tmem + kMxSfbCol) | byte, accum);
            }
          }
          if constexpr (kPair) umma_commit_pair_both(&sm->empty[st]);
          else umma_commit(&sm->empty[st]);
          if (++st == kMxStages) { st = 0; ph ^= 1; }
          if ((kb & 3) == 3) {   // the group's scale chunks have been copied into TMEM
            if constexpr (kPair) umma_commit_pair_both(&sm->chunk_empty[cs]);
            else umma_commit(&sm->chunk_empty[cs]);
            if (++cs == kMxChunkSlots) { cs = 0; cph ^= 1; }
          }
        }
        if (!ok) break;
        if constexpr (kPair) umma_commit_pair_both(&sm->acc_full[buf]);
        else umma_commit(&sm->acc_full[buf]);
      }
      if (!ok) {
        if constexpr (kPair) umma_commit_pair(&sm->drain);
        else umma_commit(&sm->drain);
        mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    const int q = warp & 3;                     // TMEM lane quadrant: features 32q .. 32q+31 of the tile
    const int part = (warp - 2) >> 2;           // 16-token column blocks part, part + 2, ...
    uint8_t* stage = epi_stage + (warp - 2) * 1024;
    for (int w = cluster, it = 0; w < total; w += nclusters, ++it) {
      const TileInfo t = decode_tile(w, s_prefix, s_offsets, p);
      const int buf = two_bufs ? (it & 1) : 0;
      const uint32_t use = two_bufs ? (it >> 1) : it;
      if (!mbar_wait_warp_backoff(&sm->acc_full[buf], use & 1, abort, p.ew, 238)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + buf * kMxAccCols + (static_cast<uint32_t>(q * 32) << 16);
      const uint32_t acc_empty_buf = acc_empty_leader + 8u * buf;
      const bool routed = t.g < p.E;
      const int feat0 = t.m * p.m_rows + rank * half_rows + q * 32;
      constexpr int kJ = kMxMaxChunk / 32;        // 16-token blocks of this warp (every other one)
      if constexpr (kSwiGLU) {
        // h = silu(g) * v per (feature = lane, token), quantised per token over the warp's 32 features
        const float* rw = (p.row_weight != nullptr && routed) ? p.row_weight + t.out_row : nullptr;
        uint32_t codes[kJ][4];
        int scale_of_lane[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
          const int c0 = part * 16 + 32 * j;
          if (c0 >= t.n) continue;
          float v0[16], v1[16];
          tmem_ld16(taddr + c0, v0);
          tmem_ld16(taddr + vcol + c0, v1);
          tmem_ld_wait();
          float a[16];
          int mine = 0;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float wr = (rw != nullptr && c0 + i < t.n) ? rw[c0 + i] : 1.f;
            a[i] = swiglu(v0[i], v1[i], p.swiglu_limit, wr);
            const uint32_t amax_bits = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(a[i])));
            const int e = mx_scale_exponent(__uint_as_float(amax_bits));
            a[i] *= mx_inv_scale(e);
            if (i == lane) mine = e + 127;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
            codes[j][i] = e4m3x2(a[4 * i], a[4 * i + 1]) | (e4m3x2(a[4 * i + 2], a[4 * i + 3]) << 16);
          scale_of_lane[j] = mine;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // TMEM is free for the next tile's MMAs
          if constexpr (kPair) mbar_arrive_remote(acc_empty_buf);
          else mbar_arrive(&sm->acc_empty[buf]);
        }
        uint8_t* qbase = routed ? p.q_routed : p.q_shared;
        uint8_t* sbase = routed ? p.s_routed : p.s_shared;
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
          const int c0 = part * 16 + 32 * j;
          if (c0 >= t.n) continue;
          // transpose through shared memory: byte (token i, feature lane), then 16-byte row pieces
#pragma unroll
          for (int i = 0; i < 16; ++i) stage[i * 32 + lane] = static_cast<uint8_t>(codes[j][i >> 2] >> (8 * (i & 3)));
          __syncwarp();
          const int tok = lane >> 1, half = lane & 1;
          if (c0 + tok < t.n) {
            const uint4 val = *reinterpret_cast<const uint4*>(stage + tok * 32 + half * 16);
            *reinterpret_cast<uint4*>(qbase + (size_t)(t.out_row + c0 + tok) * p.M_total + feat0 + half * 16) = val;
          }
          if (lane < 16 && c0 + lane < t.n)
            sbase[(size_t)(t.out_row + c0 + lane) * (p.M_total / 32) + feat0 / 32] = static_cast<uint8_t>(scale_of_lane[j]);
          __syncwarp();
        }
      } else {
        // two w2 tiles per CTA: bf16 outputs of features feat0 .. and feat0 + 128 ..
        uint32_t hv[kJ][2][8];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
          const int c0 = part * 16 + 32 * j;
          if (c0 >= t.n) continue;
          float v0[16], v1[16];
          tmem_ld16(taddr + c0, v0);
          tmem_ld16(taddr + vcol + c0, v1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            hv[j][0][i] = bf16x2_bits(v0[2 * i], v0[2 * i + 1]);
            hv[j][1][i] = bf16x2_bits(v1[2 * i], v1[2 * i + 1]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (kPair) mbar_arrive_remote(acc_empty_buf);
          else mbar_arrive(&sm->acc_empty[buf]);
        }
        __nv_bfloat16* out = routed ? p.out_routed : p.out_shared;
        uint16_t* st16 = reinterpret_cast<uint16_t*>(stage);
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
          const int c0 = part * 16 + 32 * j;
          if (c0 >= t.n) continue;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              st16[(2 * i) * 32 + lane] = static_cast<uint16_t>(hv[j][h][i] & 0xffffu);
              st16[(2 * i + 1) * 32 + lane] = static_cast<uint16_t>(hv[j][h][i] >> 16);
            }
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int vv = lane + 32 * r, tok = vv >> 2, sub = vv & 3;
              if (c0 + tok < t.n) {
                const uint4 val = *reinterpret_cast<const uint4*>(st16 + tok * 32 + sub * 8);
                *reinterpret_cast<uint4*>(out + (size_t)(t.out_row + c0 + tok) * p.M_total + feat0 + h * kGemmBM +
                                          sub * 8) = val;
              }
            }
            __syncwarp();
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // no remote signal or MMA of either CTA is outstanding past this point
  if (*abort) {
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000LL) {
    }
  }
  tc_fence_after();
  if (warp == 1) {
    if constexpr (kPair) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

template <int kVariant>
size_t mx_smem_bytes(int E) {
  using Shape = MxShape<kVariant>;
  return 1024 + (size_t)Shape::kStages * Shape::kStageBytes + (size_t)Shape::kChunkSlots * kMxChunkBytes + 8 * 1024 +
         (size_t)Shape::kSfStageBytes +
         sizeof(MxSmem) + (2 * (size_t)E + 3) * sizeof(int);
}

size_t expert_gemm_mx_smem_bytes(int E) {
  const size_t a = mx_smem_bytes<kMxLong>(E), b = mx_smem_bytes<kMxShort>(E), c = mx_smem_bytes<kMxSolo>(E);
  return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

template <int kMode, int kVariant>
static cudaError_t launch_mx_mode(const MxMaps& maps, const GemmParams& p, int max_ctas, cudaStream_t stream) {
  constexpr bool kPair = MxShape<kVariant>::kPair;
  const size_t smem = mx_smem_bytes<kVariant>(p.E);
  auto kernel = expert_gemm_mx_kernel<kMode, kVariant>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kPair ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  int ctas = kPair ? max_ctas & ~1 : max_ctas;
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kMxThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (kPair) {   // as many pairs as can be resident at once
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kernel, &cfg) == cudaSuccess && active > 0 && 2 * active < ctas)
      ctas = 2 * active;
    (void)cudaGetLastError();
  }
  cfg.gridDim = dim3(ctas);
  if (kPair) {
    cfg.numAttrs = 1 + pdl_attr(attr + 1);
  } else {   // no cluster: programmatic dependent launch only
    cfg.attrs = attr + 1;
    cfg.numAttrs = pdl_attr(attr + 1);
  }
  return cudaLaunchKernelEx(&cfg, kernel, maps, p);
}

// max_ctas: the most CTAs worth launching (twice the pair tiles, or the tiles of the single-CTA form).
cudaError_t launch_expert_gemm_mx(int mode, const MxMaps& maps, const GemmParams& p, int max_ctas,
                                  cudaStream_t stream) {
  if (p.bn > kMxMaxChunk || p.K % 512 != 0) return cudaErrorInvalidValue;
  if (p.solo && p.bn > kMxSoloChunk) return cudaErrorInvalidValue;
  const int v = p.solo ? kMxSolo : (p.bn <= kMxTwoBufChunk ? kMxShort : kMxLong);
  if (mode == kGemmSwiGLU)
    return v == kMxSolo ? launch_mx_mode<kGemmSwiGLU, kMxSolo>(maps, p, max_ctas, stream)
         : v == kMxShort ? launch_mx_mode<kGemmSwiGLU, kMxShort>(maps, p, max_ctas, stream)
                         : launch_mx_mode<kGemmSwiGLU, kMxLong>(maps, p, max_ctas, stream);
  if (mode == kGemmPair)
    return v == kMxSolo ? launch_mx_mode<kGemmPair, kMxSolo>(maps, p, max_ctas, stream)
         : v == kMxShort ? launch_mx_mode<kGemmPair, kMxShort>(maps, p, max_ctas, stream)
                         : launch_mx_mode<kGemmPair, kMxLong>(maps, p, max_ctas, stream);
  return cudaErrorInvalidValue;
}

}  // namespace moe
