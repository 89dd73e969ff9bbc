// Router kernels: the Gate of "DeepSeek-V3.2-Exp - Routing weights" (gate-forward excerpt) and the
// hash-routed gates of "From One Giant FFN to 384 Tiny Experts" (section 11.1) and "How was
// DeepSeek V4's tid2eid derived?" (the token-id table; the 2-gram hash of "An extreme case").
//
// Three kernels: router_cluster_kernel (further below; the default, K split over a cluster of CTAs,
// with top-k, table and 2-gram selection modes), router_kernel (next; one CTA per 128 tokens, for
// the layouts the cluster epilogue does not take), and hash_gate_kernel (one warp per token, for the
// hash gates of those layouts).
//
// router_kernel: one CTA per 128 tokens.  The logits l = x . W^T are a [128 x E] fp32 tile computed
// on the tensor cores (tcgen05, bf16 operands, fp32 accumulation in TMEM), with x and W staged by
// TMA.  bf16 x bf16 products are exact in fp32, so when the router weights are bf16-exact the MMA
// yields the fp32 dot product up to summation order; general fp32 router weights are first split
// exactly into three bf16 parts (hi + mid + lo) and the K loop runs over all three.  The epilogue
// then reads the tile straight out of TMEM, on all 16 warps (lane quadrant x expert range):
// affinity, selection bias, group top-2 scores, the best groups, the top-k experts, and the
// renormalised, scaled gate weights.
#include "common.cuh"
#include "dispatch_scan.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouterThreads = 512;  // 16 warps: 2 pipeline roles, all 16 in the epilogue
constexpr int kMaxTopk = kMaxRouteTopk;

// ------------------------------------------------------------------------------------------------
// fp32 router weight -> three bf16 planes with w = hi + mid + lo exactly; flag = any(mid or lo != 0)
// ------------------------------------------------------------------------------------------------
__global__ void gate_planes_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ planes, long n,
                                   int* __restrict__ inexact_flag) {
  pdl_begin();
  int inexact = 0;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);   // exact (Sterbenz)
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);  // exact
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    planes[i] = hi;
    planes[n + i] = mid;
    planes[2 * n + i] = lo;
    inexact |= (r1 != 0.f);
  }
  inexact = __any_sync(0xffffffffu, inexact);
  if (inexact && (threadIdx.x & 31) == 0) atomicOr(inexact_flag, 1);
}

// ------------------------------------------------------------------------------------------------
// tcgen05 router
// ------------------------------------------------------------------------------------------------
struct RouterSmem {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full;
  uint64_t drain;
  uint64_t recv_full;   // cluster router: every partial logit of this CTA's tokens has arrived
  uint32_t tmem_base;
  int abort;
  int nplanes;
};

// The epilogue splits each token's E experts into nsplit contiguous column ranges; warp w reads
// TMEM lane quadrant w % 4 (32 tokens) and column range w / 4.  Its shared-memory exchange area
// reuses the drained pipeline stages:
//   part1, part2 [nsplit][G][128] : per range, best and second-best biased score of every group
//   kept         [128]            : kept-group mask per token
//   pmax, psum   [nsplit][128]    : softmax partial maximum and normaliser
//   tkb, tks     [nsplit][k][128] : per range, sorted top-k selection scores and unbiased scores
//   tki          [nsplit][k][128] : their expert indices
size_t router_epilogue_bytes(int nsplit, int G, int k) {
  return (size_t)nsplit * G * 128 * 8 + 128 * 4 + (size_t)nsplit * 128 * 8 + (size_t)nsplit * k * 128 * 12;
}

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                  RouterParams p) {
  pdl_begin();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = 128 * 128;           // 128 tokens x 64 bf16
  const int b_bytes = p.E * 128;           // E experts x 64 bf16
  const int stage_bytes = a_bytes + b_bytes;
  RouterSmem* sm = reinterpret_cast<RouterSmem*>(smem + p.region_bytes);
  float* s_bias = reinterpret_cast<float*>(sm + 1);
  float* s_off = s_bias + p.E;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 128;
  const int nk = p.d / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->acc_full, 1);
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    sm->nplanes = (p.plane_flag != nullptr && *p.plane_flag) ? 3 : 1;
    fence_barrier_init();
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
  }
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    s_bias[e] = p.bias ? p.bias[e] : 0.f;
    s_off[e] = p.logit_offset ? p.logit_offset[e] : 0.f;
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int total = sm->nplanes * nk;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    int st = 0;
    uint32_t ph = 0;
    int last_par[8];
    for (int s = 0; s < 8; ++s) last_par[s] = -1;
    for (int it = 0; it < total; ++it) {
      const int plane = it / nk, kb = it - plane * nk;
      if (!mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 101)) break;
      last_par[st] = static_cast<int>(ph);
      uint8_t* sa = smem + st * stage_bytes;
      uint8_t* sb = sa + a_bytes;
      mbar_arrive_expect_tx(&sm->full[st], stage_bytes);
      tma_load_2d(sa, &map_x, &sm->full[st], kb * 64, t0);
      for (int h = 0; h < p.n_split; ++h)
        tma_load_2d(sb + h * p.n_half * 128, &map_w, &sm->full[st], kb * 64, plane * p.E + h * p.n_half);
      if (++st == p.stages) { st = 0; ph ^= 1; }
    }
    if (*abort) {  // let every load already issued land before the CTA can exit
      for (int s = 0; s < p.stages; ++s)
        if (last_par[s] >= 0) mbar_wait(&sm->full[s], last_par[s], nullptr, nullptr, 0, 200000000LL);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(128, p.n_half);
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = 0; it < total; ++it) {
      if (!mbar_wait(&sm->full[st], ph, abort, p.ew, 102)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + st * stage_bytes);
      const uint64_t adesc = sdesc_kmajor_sw128(sa);
      const uint64_t bdesc = sdesc_kmajor_sw128(sa + a_bytes);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        for (int h = 0; h < p.n_split; ++h) {
          umma_bf16(tmem + h * p.n_half, adesc + 2 * kk, bdesc + ((h * p.n_half * 128) >> 4) + 2 * kk, idesc,
                    (it | kk) != 0);
        }
      }
      umma_commit(&sm->empty[st]);
      if (++st == p.stages) { st = 0; ph ^= 1; }
    }
    if (ok) {
      umma_commit(&sm->acc_full);
    } else {
      umma_commit(&sm->drain);
      mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
    }
  }
  __syncwarp();

  // ---------------- epilogue ----------------
  const bool have_acc = mbar_wait_warp(&sm->acc_full, 0, abort, p.ew, 103);
  tc_fence_after();
  const int E = p.E, G = p.G, K = p.k, NS = p.nsplit;
  const int q = warp & 3, c = warp >> 2;         // TMEM lane quadrant, expert column range
  const int tok = q * 32 + lane;                 // row of the tile
  const int W = E / NS;                          // experts per range
  const int cbeg = c * W;
  const bool active = have_acc && c < NS;        // warp-uniform
  const bool has_bias = p.bias != nullptr;
  const int per = E / G;
  const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
  float* part1 = reinterpret_cast<float*>(smem);
  float* part2 = part1 + NS * G * 128;
  uint32_t* s_kept = reinterpret_cast<uint32_t*>(part2 + NS * G * 128);
  float* s_pmax = reinterpret_cast<float*>(s_kept + 128);
  float* s_psum = s_pmax + NS * 128;
  float* tkb = s_psum + NS * 128;
  float* tks = tkb + NS * K * 128;
  int* tki = reinterpret_cast<int*>(tks + NS * K * 128);

  // softmax: every range contributes its maximum and normaliser
  float smax = 0.f, sden = 1.f;
  if (p.score_func == MOE_SCORE_SOFTMAX) {
    if (active) {
      float m = -INFINITY, z = 0.f;
      for (int c0 = cbeg; c0 < cbeg + W; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float l = v[i] + s_off[c0 + i];
          if (l > m) { z = z * __expf(m - l) + 1.f; m = l; }
          else { z += __expf(l - m); }
        }
      }
      s_pmax[c * 128 + tok] = m;
      s_psum[c * 128 + tok] = z;
    }
    __syncthreads();
    if (have_acc) {
      smax = -INFINITY;
      for (int cc = 0; cc < NS; ++cc) smax = fmaxf(smax, s_pmax[cc * 128 + tok]);
      sden = 0.f;
      for (int cc = 0; cc < NS; ++cc) sden += s_psum[cc * 128 + tok] * __expf(s_pmax[cc * 128 + tok] - smax);
    }
  }
  auto score = [&](float l, int e) -> float {
    const float z = l + s_off[e];
    if (p.score_func == MOE_SCORE_SOFTMAX) return __expf(z - smax) / sden;
    return affinity(z, p.score_func);
  };

  // groups: each range scores the groups it covers (best and second-best biased score)
  uint32_t kept = 0xffffffffu;
  if (G > 1) {
    if (active) {
      for (int g = 0; g < G; ++g) {
        part1[(c * G + g) * 128 + tok] = -INFINITY;
        part2[(c * G + g) * 128 + tok] = -INFINITY;
      }
      int cg = cbeg / per, next_b = (cg + 1) * per;
      float c1 = -INFINITY, c2 = -INFINITY;
      for (int c0 = cbeg; c0 < cbeg + W; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c0 + i;
          if (e == next_b) {
            part1[(c * G + cg) * 128 + tok] = c1;
            part2[(c * G + cg) * 128 + tok] = c2;
            ++cg;
            next_b += per;
            c1 = -INFINITY;
            c2 = -INFINITY;
          }
          const float b = __fadd_rn(score(v[i], e), s_bias[e]);
          if (b > c1) { c2 = c1; c1 = b; }
          else if (b > c2) { c2 = b; }
        }
      }
      part1[(c * G + cg) * 128 + tok] = c1;
      part2[(c * G + cg) * 128 + tok] = c2;
    }
    __syncthreads();
    if (have_acc && c == 0) {
      // merge the ranges' partial top-2 into each group's score (kept in part1 of range 0)
      for (int g = 0; g < G; ++g) {
        float m1 = -INFINITY, m2 = -INFINITY;
        for (int cc = 0; cc < NS; ++cc) {
          const float a = part1[(cc * G + g) * 128 + tok], b = part2[(cc * G + g) * 128 + tok];
          if (a > m1) { m2 = fmaxf(m1, b); m1 = a; }
          else if (a > m2) { m2 = a; }
        }
        part1[g * 128 + tok] = has_bias ? __fadd_rn(m1, m2) : m1;
      }
      uint32_t km = 0;
      for (int r = 0; r < p.g; ++r) {  // best remaining group, lower index on ties
        int best = -1;
        float bs = -INFINITY;
        for (int g = 0; g < G; ++g) {
          if (km & (1u << g)) continue;
          const float gs = part1[g * 128 + tok];
          if (best < 0 || gs > bs) { best = g; bs = gs; }
        }
        km |= 1u << best;
      }
      s_kept[tok] = km;
    }
    __syncthreads();
    kept = s_kept[tok];
  }

  // top-k of each range over its kept experts: sorted descending, equal scores keep the lower index
  if (active) {
    float tb[kMaxTopk], ts[kMaxTopk];
    int ti[kMaxTopk];
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) { tb[j] = -INFINITY; ts[j] = 0.f; ti[j] = 0; }
    int cg = cbeg / per, next_b = (cg + 1) * per;
    for (int c0 = cbeg; c0 < cbeg + W; c0 += 16) {
      const int g_first = c0 / per, g_last = (c0 + 15) / per;
      const uint32_t span = (g_last - g_first >= 31) ? 0xffffffffu : ((2u << (g_last - g_first)) - 1u);
      const bool any = ((kept >> g_first) & span) != 0;
      if (!__any_sync(0xffffffffu, any)) {  // the TMEM load is warp-collective: skip per warp
        while (next_b <= c0 + 15) { ++cg; next_b += per; }
        continue;
      }
      float v[16];
      tmem_ld16(trow + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = c0 + i;
        if (e == next_b) { ++cg; next_b += per; }
        if (!((kept >> cg) & 1u)) continue;
        float cs = score(v[i], e);
        float cb = __fadd_rn(cs, s_bias[e]);
        if (!(cb > tb[kMaxTopk - 1])) continue;
        int ci = e;
#pragma unroll
        for (int j = 0; j < kMaxTopk; ++j) {
          if (cb > tb[j]) {
            const float xb = tb[j], xs = ts[j];
            const int xi = ti[j];
            tb[j] = cb; ts[j] = cs; ti[j] = ci;
            cb = xb; cs = xs; ci = xi;
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) {
      if (j < K) {
        tkb[(c * K + j) * 128 + tok] = tb[j];
        tks[(c * K + j) * 128 + tok] = ts[j];
        tki[(c * K + j) * 128 + tok] = ti[j];
      }
    }
  }
  __syncthreads();

  // merge the ranges' sorted lists (earlier range first on equal scores) and write the gate
  if (have_acc && c == 0) {
    const int t = t0 + tok;
    int h0 = 0, h1 = 0, h2 = 0, h3 = 0;
    float ws_[kMaxTopk];
    int wi_[kMaxTopk];
    float total_s = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) {
      if (j >= K) break;
      int best = -1;
      float bb = -INFINITY;
      for (int cc = 0; cc < NS; ++cc) {
        const int h = cc == 0 ? h0 : cc == 1 ? h1 : cc == 2 ? h2 : h3;
        if (h >= K) continue;
        const float b = tkb[(cc * K + h) * 128 + tok];
        if (best < 0 || b > bb) { best = cc; bb = b; }
      }
      const int h = best == 0 ? h0 : best == 1 ? h1 : best == 2 ? h2 : h3;
      ws_[j] = tks[(best * K + h) * 128 + tok];
      wi_[j] = tki[(best * K + h) * 128 + tok];
      if (best == 0) ++h0; else if (best == 1) ++h1; else if (best == 2) ++h2; else ++h3;
      total_s = __fadd_rn(total_s, ws_[j]);
    }
    if (t < p.T) {
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        if (j >= K) break;
        float w = ws_[j];
        if (p.renorm) w = __fdiv_rn(w, total_s);
        w = __fmul_rn(w, p.route_scale);
        p.indices[(size_t)t * K + j] = wi_[j];
        p.weights[(size_t)t * K + j] = w;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

// ------------------------------------------------------------------------------------------------
// split-K cluster router
//
// A cluster of KS CTAs (1, 2, 4 or 8) shares one 128-token tile: CTA r runs the r-th contiguous
// slice of the K loop (over all bf16 planes), so a batch of T tokens keeps about KS * T / 128 SMs
// busy instead of T / 128.  Each CTA leaves a partial [128 x E] fp32 logit tile in TMEM.  After a
// cluster barrier (every CTA's pipeline drained), each CTA pushes its partial rows, through
// distributed shared memory, to the CTA that owns those tokens: CTA r owns tokens
// [r * 128/KS, (r+1) * 128/KS) and keeps one slot per source, so the owner adds the KS partials in a
// fixed order (deterministic results).  A second barrier, then the owner's epilogue runs 16 lanes
// per token, each lane holding PL = E / 16 consecutive experts: affinity and bias per lane; group
// scores (sum of the two best biased scores, or the best without a bias) reduced with shuffles over
// the 16 / G lanes of a group; the kept groups ranked from the G scores broadcast by shuffles; and k
// rounds of a 16-lane shuffle arg-max (equal scores: lower expert index) select the experts.  In the
// hash modes the same kernel serves the token-id table and the 2-gram hash: the experts come from
// the table (or the hash), and each one's affinity is shuffled from the lane that holds it.
// ------------------------------------------------------------------------------------------------
// Physical column of logical column col in a row of the partial-logit exchange buffer: 16-byte chunks
// are XOR-swizzled within aligned groups of eight, so that the epilogue's 16 lanes of a token (each
// reading its own run of PL consecutive columns) hit distinct bank groups; rows are E + 4 floats apart,
// so the exchange's writes (lanes = consecutive rows, the same columns) stay conflict-free too.
__device__ __forceinline__ int recv_col(int col) {
  const int ch = col >> 2;
  return ((ch ^ ((ch >> 3) & 7)) << 2) | (col & 3);
}

// Asynchronous 16-byte store into a CTA of the cluster, counted (16 bytes of transaction) on that
// CTA's barrier at `remote_bar`.
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
               : "memory");
}

bool router_cluster_supported(int E, int G) {
  if (E % 16 != 0 || 16 % G != 0) return false;
  const int pl = E / 16;
  return pl == 1 || pl == 2 || pl == 4 || pl == 8 || pl == 16 || pl == 24;
}

template <int PL>
__global__ void __launch_bounds__(kRouterThreads, 1)
    router_cluster_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                          RouterParams p) {
  pdl_begin();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int E = 16 * PL;
  const int a_bytes = 128 * 128;           // 128 tokens x 64 bf16
  const int b_bytes = E * 128;             // E experts x 64 bf16
  const int stage_bytes = a_bytes + b_bytes;
  RouterSmem* sm = reinterpret_cast<RouterSmem*>(smem + p.region_bytes);
  float* s_bias = reinterpret_cast<float*>(sm + 1);
  float* s_off = s_bias + E;
  int* s_hist = reinterpret_cast<int*>(s_off + E);   // [E] fused dispatch histogram of this CTA's slots
  int* s_wsum = s_hist + E;                          // [16] its last CTA's scan
  int* s_flag = s_wsum + 16;
  float* recv = reinterpret_cast<float*>(smem);   // [KS][128 / KS][e_pad], after the pipeline drained

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = p.ksplit;
  const int rank = (int)cluster_ctarank();
  const int tile = blockIdx.x / KS;
  const int t0 = tile * 128;
  const int TPC = 128 / KS;                // tokens owned by each CTA of the cluster
  const int nk = p.d / 64;

  if (threadIdx.x == 0) {
    for (int st = 0; st < p.stages; ++st) {
      mbar_init(&sm->full[st], 1);
      mbar_init(&sm->empty[st], 1);
    }
    mbar_init(&sm->recv_full, 1);
    mbar_init(&sm->acc_full, 1);
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    sm->nplanes = (p.plane_flag != nullptr && *p.plane_flag) ? 3 : 1;
    fence_barrier_init();
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    s_bias[e] = p.bias ? p.bias[e] : 0.f;
    s_off[e] = p.logit_offset ? p.logit_offset[e] : 0.f;
    s_hist[e] = 0;
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;
  const int total = sm->nplanes * nk;
  const int it0 = (int)((long)rank * total / KS), it1 = (int)((long)(rank + 1) * total / KS);

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer: this CTA's slice of the K loop ----------------
    int st = 0;
    uint32_t ph = 0;
    int last_par[8];
    for (int i = 0; i < 8; ++i) last_par[i] = -1;
    for (int it = it0; it < it1; ++it) {
      const int plane = it / nk, kb = it - plane * nk;
      if (!mbar_wait(&sm->empty[st], ph ^ 1, abort, p.ew, 121)) break;
      last_par[st] = static_cast<int>(ph);
      uint8_t* sa = smem + st * stage_bytes;
      uint8_t* sb = sa + a_bytes;
      mbar_arrive_expect_tx(&sm->full[st], stage_bytes);
      tma_load_2d(sa, &map_x, &sm->full[st], kb * 64, t0);
      for (int h = 0; h < p.n_split; ++h)
        tma_load_2d(sb + h * p.n_half * 128, &map_w, &sm->full[st], kb * 64, plane * E + h * p.n_half);
      if (++st == p.stages) { st = 0; ph ^= 1; }
    }
    if (*abort) {  // let every load already issued land before the stages are reused
      for (int i = 0; i < p.stages; ++i)
        if (last_par[i] >= 0) mbar_wait(&sm->full[i], last_par[i], nullptr, nullptr, 0, 200000000LL);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(128, p.n_half);
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = it0; it < it1; ++it) {
      if (!mbar_wait(&sm->full[st], ph, abort, p.ew, 122)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + st * stage_bytes);
      const uint64_t adesc = sdesc_kmajor_sw128(sa);
      const uint64_t bdesc = sdesc_kmajor_sw128(sa + a_bytes);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        for (int h = 0; h < p.n_split; ++h) {
          umma_bf16(tmem + h * p.n_half, adesc + 2 * kk, bdesc + ((h * p.n_half * 128) >> 4) + 2 * kk, idesc,
                    (it != it0 || kk != 0) ? 1u : 0u);
        }
      }
      umma_commit(&sm->empty[st]);
      if (++st == p.stages) { st = 0; ph ^= 1; }
    }
    if (ok) {
      umma_commit(&sm->acc_full);
    } else {
      umma_commit(&sm->drain);
      mbar_wait(&sm->drain, 0, nullptr, nullptr, 0, 200000000LL);
    }
  }
  __syncwarp();
  const bool have_acc = mbar_wait_warp(&sm->acc_full, 0, abort, p.ew, 123);
  tc_fence_after();

  // ---------------- exchange of the partial logits ----------------
  // Rows of tokens past T are neither sent nor expected.  Each owner's barrier expects the partial
  // rows of its valid tokens from every CTA of the cluster (its own included), delivered by
  // asynchronous stores that count their bytes on it.
  if (threadIdx.x == 0) {
    int nvalid = p.T - (t0 + rank * TPC);
    nvalid = nvalid < 0 ? 0 : (nvalid > TPC ? TPC : nvalid);
    mbar_arrive_expect_tx(&sm->recv_full, (uint32_t)(KS * nvalid * E * 4));
  }
  cluster_sync();  // every CTA's pipeline has drained: the stage region becomes the receive buffer
  {
    const int q = warp & 3;                           // TMEM lane quadrant: tokens 32q .. 32q+31
    const int nranges = E % 64 == 0 ? 4 : 1;          // column ranges of E / 4 (or all E) experts
    const int c = warp >> 2;
    const int W = E / nranges;
    if (have_acc && c < nranges) {
      const int tl = q * 32 + lane;                   // token row of the tile
      const bool valid = t0 + tl < p.T;
      const int owner = tl / TPC, local = tl - owner * TPC;
      const uint32_t row = cluster_addr(recv + ((size_t)rank * TPC + local) * p.e_pad, owner);
      const uint32_t bar = cluster_addr(&sm->recv_full, owner);
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      for (int cb = c * W; cb < (c + 1) * W; cb += 64) {
        // up to 64 columns: every TMEM load issued before one wait, then the DSMEM stores
        float v[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (cb + 16 * j < (c + 1) * W) tmem_ld16(trow + cb + 16 * j, v[j]);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (cb + 16 * j >= (c + 1) * W) break;
          if (!valid) continue;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            st_async_v4(row + recv_col(cb + 16 * j + i) * 4, v[j][i], v[j][i + 1], v[j][i + 2], v[j][i + 3], bar);
        }
      }
    }
  }
  tc_fence_before();
  // every partial of this CTA's tokens has arrived (or, after an abort anywhere, the bounded wait
  // records a timeout)
  const bool have_all = mbar_wait_warp(&sm->recv_full, 0, abort, p.ew, 124);
  if (have_all) (void)mbar_try_wait(&sm->recv_full, 0);   // every lane observes the completed phase

  // ---------------- epilogue: 16 lanes per owned token ----------------
  const int K = p.k, G = p.G;
  const int L = 16 / G;                               // lanes per group
  const bool has_bias = p.bias != nullptr;
  const int sub = lane & 15;
  for (int base = 0; base < TPC; base += 32) {
    const int local = base + (threadIdx.x >> 4);
    const bool in_tile = local < TPC;
    const int t = t0 + rank * TPC + local;
    float sc[PL], bb[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) sc[i] = 0.f;
    if (in_tile) {
      for (int src = 0; src < KS; ++src) {
        const float* r = recv + ((size_t)src * TPC + local) * p.e_pad;
        if (PL % 4 == 0) {
#pragma unroll
          for (int i = 0; i < PL; i += 4) {
            const float4 v = *reinterpret_cast<const float4*>(r + recv_col(sub * PL + i));
            sc[i] += v.x; sc[i + 1] += v.y; sc[i + 2] += v.z; sc[i + 3] += v.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < PL; ++i) sc[i] += r[recv_col(sub * PL + i)];
        }
      }
    }
    // logits -> affinities (softmax: maximum and normaliser over the token's 16 lanes)
#pragma unroll
    for (int i = 0; i < PL; ++i) sc[i] += s_off[sub * PL + i];
    if (p.score_func == MOE_SCORE_SOFTMAX) {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < PL; ++i) m = fmaxf(m, sc[i]);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < PL; ++i) { sc[i] = __expf(sc[i] - m); z += sc[i]; }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
      for (int i = 0; i < PL; ++i) sc[i] = sc[i] / z;
    } else {
#pragma unroll
      for (int i = 0; i < PL; ++i) sc[i] = affinity(sc[i], p.score_func);
    }
    if (p.sel_mode != 0) {
      // hash-routed gate: the experts come from the token-id table or the 2-gram hash; each expert's
      // affinity is taken from the lane that holds it
      const bool live = in_tile && t < p.T && have_acc && have_all;
      int tok = 0, prev = 0;
      if (in_tile && t < p.T) {
        tok = p.token_ids[t];
        if (tok < 0 || tok >= p.vocab) {
          if (sub == 0) record_error(p.ew, MOE_ERR_DEVICE, tok);
          tok = tok < 0 ? 0 : p.vocab - 1;
        }
        if (p.sel_mode == 2) {
          prev = p.prev_ids[t];
          if (prev < 0 || prev >= p.vocab) {
            if (sub == 0) record_error(p.ew, MOE_ERR_DEVICE, prev);
            prev = prev < 0 ? 0 : p.vocab - 1;
          }
        }
      }
      int hsel_e[kMaxTopk];
      float hsel_s[kMaxTopk];
      float htotal = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        hsel_e[j] = 0;
        hsel_s[j] = 0.f;
        if (j >= K) continue;
        int e = 0;
        if (in_tile && t < p.T) {
          e = p.sel_mode == 1 ? p.tid2eid[(size_t)tok * K + j]
                              : (int)(((unsigned long long)prev * p.primes[j] + (unsigned long long)tok) %
                                      (unsigned long long)E);
          if (e < 0 || e >= E) {
            if (sub == 0) record_error(p.ew, MOE_ERR_DEVICE, e);
            e = e < 0 ? 0 : E - 1;
          }
        }
        float mine = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i)
          if (sub * PL + i == e) mine = sc[i];
        const float se = __shfl_sync(0xffffffffu, mine, (lane & 16) + e / PL);
        hsel_e[j] = e;
        hsel_s[j] = se;
        htotal = __fadd_rn(htotal, se);
      }
      if (live && sub == 0) {
#pragma unroll
        for (int j = 0; j < kMaxTopk; ++j) {
          if (j >= K) break;
          float w = hsel_s[j];
          if (p.renorm) w = __fdiv_rn(w, htotal);
          w = __fmul_rn(w, p.route_scale);
          p.indices[(size_t)t * K + j] = hsel_e[j];
          p.weights[(size_t)t * K + j] = w;
          if (p.hist != nullptr) atomicAdd(&s_hist[hsel_e[j]], 1);
        }
      }
      continue;
    }
#pragma unroll
    for (int i = 0; i < PL; ++i) bb[i] = __fadd_rn(sc[i], s_bias[sub * PL + i]);

    // kept groups
    bool kept = true;
    if (G > 1) {
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        if (bb[i] > m1) { m2 = m1; m1 = bb[i]; }
        else if (bb[i] > m2) { m2 = bb[i]; }
      }
      for (int o = 1; o < L; o <<= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, m1, o), o2 = __shfl_xor_sync(0xffffffffu, m2, o);
        const float n1 = fmaxf(m1, o1);
        const float n2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = n1;
        m2 = n2;
      }
      const float gs = has_bias ? __fadd_rn(m1, m2) : m1;
      const int my_g = sub / L;
      int better = 0;
      for (int j = 0; j < G; ++j) {
        const float gj = __shfl_sync(0xffffffffu, gs, j * L, 16);
        better += (gj > gs || (gj == gs && j < my_g)) ? 1 : 0;
      }
      kept = better < p.g;
    }

    // top-k: k rounds of a 16-lane arg-max over the kept, not yet chosen experts
    uint32_t taken = kept ? 0u : 0xffffffffu;
    int sel_e[kMaxTopk];
    float sel_s[kMaxTopk];
    float total_s = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) {
      sel_e[j] = 0;
      sel_s[j] = 0.f;
      if (j >= K) continue;
      float vb = -INFINITY, vs = 0.f;
      int ve = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < PL; ++i) {
        if (!((taken >> i) & 1u) && (ve == 0x7fffffff || bb[i] > vb)) {
          vb = bb[i];
          vs = sc[i];
          ve = sub * PL + i;
        }
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, vb, o);
        const float os = __shfl_xor_sync(0xffffffffu, vs, o);
        const int oe = __shfl_xor_sync(0xffffffffu, ve, o);
        if (ob > vb || (ob == vb && oe < ve)) { vb = ob; vs = os; ve = oe; }
      }
      if (ve / PL == sub) taken |= 1u << (ve - sub * PL);
      sel_e[j] = ve;
      sel_s[j] = vs;
      total_s = __fadd_rn(total_s, vs);
    }
    if (in_tile && t < p.T && sub == 0 && have_acc && have_all) {
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        if (j >= K) break;
        float w = sel_s[j];
        if (p.renorm) w = __fdiv_rn(w, total_s);
        w = __fmul_rn(w, p.route_scale);
        p.indices[(size_t)t * K + j] = sel_e[j];
        p.weights[(size_t)t * K + j] = w;
        if (p.hist != nullptr && sel_e[j] >= 0 && sel_e[j] < E) atomicAdd(&s_hist[sel_e[j]], 1);
      }
    }
  }

  if (p.hist != nullptr) {
    // dispatch's histogram: this CTA's row (its tokens' slots), then the last CTA's scan
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) p.hist[(size_t)blockIdx.x * E + e] = s_hist[e];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *s_flag = atomicAdd(p.ticket, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (*s_flag)
      dispatch_finish_scan(p.hist, (int)gridDim.x, E, p.T * K, p.base, p.counts, p.offsets, p.ticket, s_wsum);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

size_t router_cluster_smem_bytes(const RouterParams& p) {
  return 1024 + (size_t)p.region_bytes + sizeof(RouterSmem) + 2 * (size_t)p.E * sizeof(float) +
         ((size_t)p.E + 32) * sizeof(int);
}

template <int PL>
static cudaError_t launch_router_cluster_pl(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                                            cudaStream_t stream) {
  const size_t smem = router_cluster_smem_bytes(p);
  cudaError_t err =
      cudaFuncSetAttribute(router_cluster_kernel<PL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((p.T + 127) / 128) * p.ksplit);
  cfg.blockDim = dim3(kRouterThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + pdl_attr(attr + 1);
  return cudaLaunchKernelEx(&cfg, router_cluster_kernel<PL>, map_x, map_w, p);
}

cudaError_t launch_router_cluster(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                                  cudaStream_t stream) {
  switch (p.E / 16) {
    case 1: return launch_router_cluster_pl<1>(map_x, map_w, p, stream);
    case 2: return launch_router_cluster_pl<2>(map_x, map_w, p, stream);
    case 4: return launch_router_cluster_pl<4>(map_x, map_w, p, stream);
    case 8: return launch_router_cluster_pl<8>(map_x, map_w, p, stream);
    case 16: return launch_router_cluster_pl<16>(map_x, map_w, p, stream);
    case 24: return launch_router_cluster_pl<24>(map_x, map_w, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

// ------------------------------------------------------------------------------------------------
// hash gates (token-id table or 2-gram hash): one warp per token, k dot products of length d
// ------------------------------------------------------------------------------------------------
__global__ void hash_gate_kernel(HashGateParams p) {
  pdl_begin();
  const int warps = blockDim.x >> 5;
  const int t = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= p.T) return;
  int tok = p.token_ids[t];
  if (tok < 0 || tok >= p.vocab) {
    if (lane == 0) record_error(p.ew, MOE_ERR_DEVICE, tok);
    tok = tok < 0 ? 0 : p.vocab - 1;
  }
  int prev = 0;
  if (p.prev_ids != nullptr) {
    prev = p.prev_ids[t];
    if (prev < 0 || prev >= p.vocab) {
      if (lane == 0) record_error(p.ew, MOE_ERR_DEVICE, prev);
      prev = prev < 0 ? 0 : p.vocab - 1;
    }
  }
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.d);
  float s[kMaxTopk];
  int ex[kMaxTopk];
  float total_s = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopk; ++j) {
    if (j >= p.k) break;
    int e;
    if (p.prev_ids != nullptr) {
      // 2-gram hash: (a * q_j + b) mod E, exact in 64-bit unsigned arithmetic (a, b < 2^31, q_j < 2^32)
      e = (int)(((unsigned long long)prev * p.primes[j] + (unsigned long long)tok) % (unsigned long long)p.E);
    } else {
      e = p.tid2eid[(size_t)tok * p.k + j];
    }
    if (e < 0 || e >= p.E) {
      if (lane == 0) record_error(p.ew, MOE_ERR_DEVICE, e);
      e = e < 0 ? 0 : p.E - 1;
    }
    const float4* wr = reinterpret_cast<const float4*>(p.w_gate + (size_t)e * p.d);
    float acc = 0.f;
    for (int c = lane; c < p.d / 8; c += 32) {
      const uint4 xv = xr[c];
      const float4 w0 = wr[2 * c], w1 = wr[2 * c + 1];
      const __nv_bfloat162* xb = reinterpret_cast<const __nv_bfloat162*>(&xv);
      const float2 a = __bfloat1622float2(xb[0]), b = __bfloat1622float2(xb[1]);
      const float2 cc = __bfloat1622float2(xb[2]), dd = __bfloat1622float2(xb[3]);
      acc = fmaf(a.x, w0.x, acc); acc = fmaf(a.y, w0.y, acc);
      acc = fmaf(b.x, w0.z, acc); acc = fmaf(b.y, w0.w, acc);
      acc = fmaf(cc.x, w1.x, acc); acc = fmaf(cc.y, w1.y, acc);
      acc = fmaf(dd.x, w1.z, acc); acc = fmaf(dd.y, w1.w, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    s[j] = affinity(acc, p.score_func);
    ex[j] = e;
    total_s = __fadd_rn(total_s, s[j]);
  }
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) {
      if (j >= p.k) break;
      float w = s[j];
      if (p.renorm) w = __fdiv_rn(w, total_s);
      w = __fmul_rn(w, p.route_scale);
      p.indices[(size_t)t * p.k + j] = ex[j];
      p.weights[(size_t)t * p.k + j] = w;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------------
cudaError_t launch_gate_planes(const float* w, __nv_bfloat16* planes, long n, int* inexact_flag, int num_sms,
                               cudaStream_t stream) {
  const long want = (n + 255) / 256;
  const int grid = (int)(want < 4L * num_sms ? (want > 0 ? want : 1) : 4L * num_sms);
  return launch_pdl(gate_planes_kernel, dim3(grid), dim3(256), 0, stream, w, planes, n, inexact_flag);
}

size_t router_smem_bytes(const RouterParams& p) {
  return 1024 + (size_t)p.region_bytes + sizeof(RouterSmem) + 2 * (size_t)p.E * sizeof(float);
}

cudaError_t launch_router(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                          cudaStream_t stream) {
  const size_t smem = router_smem_bytes(p);
  cudaError_t err = cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = (p.T + 127) / 128;
  return launch_pdl(router_kernel, dim3(grid), dim3(kRouterThreads), smem, stream, map_x, map_w, p);
}

cudaError_t launch_hash_gate(const HashGateParams& p, cudaStream_t stream) {
  const int warps = 8;
  return launch_pdl(hash_gate_kernel, dim3((p.T + warps - 1) / warps), dim3(warps * 32), 0, stream, p);
}

}  // namespace moe
