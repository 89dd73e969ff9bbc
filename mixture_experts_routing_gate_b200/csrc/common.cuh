// Device-side building blocks shared by the libmoe kernels (sm_100a only).
//
// * mbarrier helpers whose waits are bounded in time: a wait that runs out records
//   MOE_ERR_TIMEOUT in the workspace error word and returns false, so no kernel can hang;
// * TMA (cp.async.bulk.tensor) tile loads, never with cluster multicast;
// * tcgen05 tensor-core helpers: TMEM allocation, the bf16 x bf16 -> fp32 MMA with operands in
//   shared memory, commit to an mbarrier, and TMEM -> register loads for the epilogues;
// * the shared-memory matrix descriptor for K-major tiles in the 128-byte swizzle layout that
//   TMA writes, and the instruction descriptor of kind::f16 MMAs.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------------------------------------------------
// error word (first 256 bytes of every workspace)
// ------------------------------------------------------------------------------------------------
struct ErrorWord {
  int status;           // 0 or the first moe_status recorded
  int info;             // the offending value (index, token id, or a wait site)
  int dispatch_ticket;  // dispatch's count of finished histogram blocks (0 between calls)
  int pad[61];
};

__device__ __forceinline__ void record_error(ErrorWord* ew, int status, int info) {
  if (ew == nullptr) return;
  if (atomicCAS(&ew->status, 0, status) == 0) atomicExch(&ew->info, info);
}

// ------------------------------------------------------------------------------------------------
// small helpers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_one_lane() { return (threadIdx.x & 31) == 0; }

// ------------------------------------------------------------------------------------------------
// programmatic dependent launch: every kernel of the library is launched so that it may start
// while its predecessor on the stream drains; its first statement waits for the predecessor to
// complete (griddepcontrol.wait, a no-op without one), so stream order is kept, and it then lets
// its own successor launch early.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void pdl_begin() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Default bound on any single pipeline wait, in SM clock cycles (about 2 s at the B200's 1.9 GHz
// boost clock, longer at lower clocks).  A correct pipeline never waits more than a few
// microseconds; the bound only has to be far above that and far below a watchdog.  The SM's own
// cycle counter is cheap to read, unlike the global timer.
constexpr long long kWaitLimitCycles = 4000000000LL;

// Waits for the phase of `parity` to complete.  Gives up (returns false) when `*abort` becomes
// non-zero (another role of the CTA gave up) or after `limit` cycles, recording MOE_ERR_TIMEOUT with
// `site` as info.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          ErrorWord* ew, int site, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255) == 0) {
      if (abort != nullptr && *abort) return false;
      if (clock64() - t0 > limit) {
        record_error(ew, MOE_ERR_TIMEOUT, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// As mbar_wait for waiters off the critical path: after a few failed polls the thread sleeps
// `sleep_ns` between polls, leaving the issue slots of its SM sub-partition to warps doing work.
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                 ErrorWord* ew, int site, unsigned sleep_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (it > 4) __nanosleep(sleep_ns);
    if ((it & 15) == 0) {
      if (abort != nullptr && *abort) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        record_error(ew, MOE_ERR_TIMEOUT, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// As mbar_wait, with cluster-scope acquire (for phases completed by arrivals from the other CTA).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity);
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  ErrorWord* ew, int site, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 255) == 0) {
      if (abort != nullptr && *abort) return false;
      if (clock64() - t0 > limit) {
        record_error(ew, MOE_ERR_TIMEOUT, site);
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// mbar_wait by lane 0 only; the result is shared with the warp (whose lanes then see the phase
// completed through the warp synchronisation).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               ErrorWord* ew, int site) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, ew, site);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// mbar_wait_sleepy by lane 0, the result shared with the warp.
__device__ __forceinline__ bool mbar_wait_warp_sleepy(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                      ErrorWord* ew, int site, unsigned sleep_ns) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_sleepy(bar, parity, abort, ew, site, sleep_ns);
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// As mbar_wait_warp for long waits (a whole tile's K loop): lane 0 sleeps briefly between polls, so
// that the waiting warps leave the issue slots to the warps doing work.
__device__ __forceinline__ bool mbar_wait_warp_backoff(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                       ErrorWord* ew, int site) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) {
    if (mbar_try_wait(bar, parity)) {
      ok = 1;
    } else {
      const long long t0 = clock64();
      for (;;) {
        __nanosleep(200);
        if (mbar_try_wait(bar, parity)) { ok = 1; break; }
        if (abort != nullptr && *abort) break;
        if (clock64() - t0 > kWaitLimitCycles) {
          record_error(ew, MOE_ERR_TIMEOUT, site);
          if (abort != nullptr) *abort = 1;
          break;
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ------------------------------------------------------------------------------------------------
// TMA
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2-D tiled load of the box at (c0 = innermost coordinate, c1 = row) into shared memory; completes
// `bytes` (the full box) of transaction count on `bar`.  c0 must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copies (cp.async.bulk): both addresses 16-byte aligned, the size a multiple of 16.
// A load completes `bytes` of transaction count on `bar`; stores are tracked in the issuing thread's
// bulk async-groups (bulk_commit closes a group, bulk_wait_read<N> waits until at most N of the most
// recent groups may still be reading shared memory, bulk_wait_all<N> until their writes are done).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(smem_src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------------------------------------
// tcgen05 / TMEM
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, A: M x 16, B: N x 16, both K-major bf16, D fp32.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Each thread of the warp reads 16 consecutive fp32 columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory descriptor of a K-major bf16 tile written by TMA with 128-byte swizzle: rows of
// 64 elements (128 bytes), 8-row swizzle atoms of 1024 bytes stacked along M/N (stride 1024).
// The tile must start on a 1024-byte boundary; the K offset inside the 64-wide atom is added to the
// start address field (32 bytes per 16-element step).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address, 16-byte units
  d |= static_cast<uint64_t>(1u) << 16;                // leading-dimension offset (unused here)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;        // stride between 8-row groups
  d |= static_cast<uint64_t>(1u) << 46;                // descriptor version of sm_100
  d |= static_cast<uint64_t>(2u) << 61;                // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                     // D format fp32
         | (1u << 7)                                   // A format bf16
         | (1u << 10)                                  // B format bf16
         | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);      // M / 16
}

// ------------------------------------------------------------------------------------------------
// CTA pairs (clusters of two CTAs sharing one tcgen05 MMA, "cta_group::2")
//
// The even CTA of the pair issues every MMA; each MMA reads 128 rows of A from each CTA's shared
// memory and N/2 rows of B from each, and writes its 128 x N accumulator into each CTA's TMEM.
// Both CTAs' TMA loads signal the even CTA's "full" barrier; MMA completion is multicast to both
// CTAs' barriers.  No TMA load here uses cluster multicast: each CTA loads its own halves.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of both CTAs: arrive (release) and wait (acquire) on the cluster barrier.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of this CTA's shared variable `p` as seen in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// Arrive on a barrier of the pair with cluster-scope release: orders this thread's earlier writes
// (made visible to the async proxy by fence_proxy_async) before the phase completion it contributes to.
__device__ __forceinline__ void mbar_arrive_remote_release(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// One non-blocking test of a phase with cluster-scope acquire.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Generic-proxy shared-memory writes of this thread become visible to the async proxy (TMA, MMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte store into the shared memory of a CTA of the cluster (address from cluster_addr).
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the barrier at `cluster_bar`
// (the pair's even CTA).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t cluster_bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(cluster_bar)
      : "memory");
}

// Four rows of a 2D tensor map, gathered (tile::gather4): the map's box is one row of 64 elements and
// rows r0..r3 land as consecutive 128-byte rows (swizzled like any box) at smem_dst, which is 512-byte
// aligned; completion is counted on the barrier at `cluster_bar` (the pair's even CTA).
__device__ __forceinline__ void tma_gather4_pair(void* smem_dst, const CUtensorMap* map, uint32_t cluster_bar,
                                                 int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(smem_dst)),
      "l"(map), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(cluster_bar)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (+)= A * B^T over the CTA pair: A is 256 x 16 (128 rows per CTA), B is N x 16 (N/2 rows per CTA).
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// Arrives once on the barrier at this offset in both CTAs of the pair when all prior MMAs complete.
__device__ __forceinline__ void umma_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}

// Arrives once on this CTA's barrier when all prior MMAs of the pair complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ------------------------------------------------------------------------------------------------
// block-scaled MMAs (kind::mxf8f6f4): E2M1 weights x E4M3 activations with UE8M0 scales per 32 of K
//
// Operands in shared memory are K-major 128-byte swizzled rows of 128 elements (E4M3: one byte each;
// E2M1: 16 packed codes in each 16-byte slot, 8 bytes then 8 unused, as the 16U4_ALIGN16B tensor-map
// type lays them out); one MMA covers K = 32.
// The scales live in TMEM: a 32-bit column word holds the scales of four consecutive K blocks of one
// row; a 512-byte "scale chunk" in shared memory -- line l (16 bytes) holding the four K blocks'
// scales of rows l, l + 32, l + 64 and l + 96 -- is moved by one tcgen05.cp 32x128b.warpx4 into
// lanes l (replicated over the four lane quadrants) and four consecutive columns, column j holding
// row l + 32 j.  Each MMA names its K block's byte of the word (the scale-factor id).
// ------------------------------------------------------------------------------------------------
// Instruction descriptor of kind::mxf8f6f4 with UE8M0 scales: A = E2M1, B = E4M3, fp32 D, both
// K-major, M x N; sf_a / sf_b select the byte of the scale words.
__host__ __device__ constexpr uint32_t idesc_mx_e2m1_e4m3(int M, int N, uint32_t sf_a, uint32_t sf_b) {
  return (sf_b << 4)                                   // B scale-factor id
         | (5u << 7)                                   // A format E2M1
         | (0u << 10)                                  // B format E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)       // N / 8
         | (1u << 23)                                  // scale format UE8M0
         | (static_cast<uint32_t>(M >> 4) << 24)       // M / 16
         | (sf_a << 29);                               // A scale-factor id
}

// D (+)= (A * sfa) (B * sfb)^T over the CTA pair: A 256 x 32 (128 rows per CTA), B N x 32 (N/2 rows
// per CTA); sfa_tmem / sfb_tmem: TMEM addresses of the scale words, the byte id in bits 30-31.
__device__ __forceinline__ void umma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// A 512-byte scale chunk (32 lines of 16 bytes, contiguous) from each CTA's shared memory into four
// columns of its TMEM at taddr, replicated over the four lane quadrants; issued by the pair's even CTA.
__device__ __forceinline__ void tmem_cp_chunk_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a scale chunk: unswizzled K-major rows of 16 bytes, 8-row core matrices
// of 128 contiguous bytes stacked along the rows (stride 128 bytes).
__device__ __forceinline__ uint64_t sdesc_scale_chunk(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address, 16-byte units
  d |= static_cast<uint64_t>(1u) << 16;                // leading-dimension offset (one 16-byte column)
  d |= static_cast<uint64_t>(128u >> 4) << 32;         // stride between 8-row core matrices
  d |= static_cast<uint64_t>(1u) << 46;                // descriptor version of sm_100
  return d;                                            // layout type 0: no swizzle
}

// ------------------------------------------------------------------------------------------------
// numerics
// ------------------------------------------------------------------------------------------------
// The affinity of a logit, with the fast exponential and reciprocal (a few fp32 ulp, far below the
// 2e-5 relative agreement asked of the gate weights and the 1e-5 near-tie rule of the selection).
__device__ __forceinline__ float affinity(float l, int score_func) {
  if (score_func == MOE_SCORE_SQRT_SOFTPLUS) {
    const float sp = fmaxf(l, 0.f) + log1pf(__expf(-fabsf(l)));
    return sqrtf(sp);
  }
  return __fdividef(1.f, 1.f + __expf(-l));  // sigmoid (softmax is handled by the caller)
}

// Two floats rounded to bf16 (round to nearest even), packed with `lo` in the low 16 bits.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// silu(z) = z / (1 + e^-z) with the fast approximate exponential and division (a few ulp of fp32,
// far below the bf16 rounding of the result); for z < -87 the quotient flushes to zero.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// UE8M0 exponent of the scale of an FP8 block whose largest magnitude is amax (>= 0): the least e
// with 448 * 2^e >= amax, from amax's bits (448 = 1.75 * 2^8: e = F - 8 when amax = m * 2^F with
// m <= 1.75, else F - 7); -127 for zero or subnormal amax, at most 127.
__device__ __forceinline__ int mx_scale_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int biased = (int)((bits >> 23) & 0xFFu);
  if (biased == 0) return -127;
  int e = biased - 127 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e > 127 ? 127 : e;
}

// 2^-e as an fp32 (e in [-127, 127]; 2^127 and the subnormal 2^-127 included).
__device__ __forceinline__ float mx_inv_scale(int e) {
  return e > -127 ? __uint_as_float((uint32_t)(127 - e) << 23)
                  : __uint_as_float(0x7F000000u);   // e = -127: 2^127
}

// Two fp32 values to E4M3 codes (round to nearest even; |v| <= 448 never saturates), packed with
// the first in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// SwiGLU of one gate / value pair, with the optional clamp (limit > 0) and row weight.
__device__ __forceinline__ float swiglu(float g, float v, float limit, float w) {
  if (limit > 0.f) {
    g = fminf(g, limit);
    v = fminf(fmaxf(v, -limit), limit);
  }
  return silu(g) * v * w;
}

}  // namespace moe
