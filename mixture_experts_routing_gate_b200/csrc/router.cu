// Router kernels: the Gate of "DeepSeek-V3.2-Exp - Routing weights" (gate-forward excerpt) and the
// hash-routed gate of "From One Giant FFN to 384 Tiny Experts" (section 11.1).
//
// router_kernel: one CTA per 128 tokens.  The logits l = x . W^T are a [128 x E] fp32 tile computed
// on the tensor cores (tcgen05, bf16 operands, fp32 accumulation in TMEM), with x and W staged by
// TMA.  bf16 x bf16 products are exact in fp32, so when the router weights are bf16-exact the MMA
// yields the fp32 dot product up to summation order; general fp32 router weights are first split
// exactly into three bf16 parts (hi + mid + lo) and the K loop runs over all three.  The epilogue
// then runs one token per thread straight out of TMEM: affinity, selection bias, group top-2 scores,
// the best groups, the top-k experts, and the renormalised, scaled gate weights.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouterThreads = 128;
constexpr int kMaxTopk = 8;

// ------------------------------------------------------------------------------------------------
// fp32 router weight -> three bf16 planes with w = hi + mid + lo exactly; flag = any(mid or lo != 0)
// ------------------------------------------------------------------------------------------------
__global__ void gate_planes_kernel(const float* __restrict__ w, __nv_bfloat16* __restrict__ planes, long n,
                                   int* __restrict__ inexact_flag) {
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
  uint32_t tmem_base;
  int abort;
  int nplanes;
};

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                  RouterParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = 128 * 128;           // 128 tokens x 64 bf16
  const int b_bytes = p.E * 128;           // E experts x 64 bf16
  const int stage_bytes = a_bytes + b_bytes;
  RouterSmem* sm = reinterpret_cast<RouterSmem*>(smem + p.stages * stage_bytes);
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

  // ---------------- epilogue: one token per thread, straight from TMEM ----------------
  const bool have_acc = mbar_wait_warp(&sm->acc_full, 0, abort, p.ew, 103);
  tc_fence_after();
  if (have_acc) {
    const int t = t0 + threadIdx.x;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int E = p.E;
    const bool has_bias = p.bias != nullptr;

    // softmax needs the row maximum and normaliser first
    float smax = 0.f, sden = 1.f;
    if (p.score_func == MOE_SCORE_SOFTMAX) {
      smax = -INFINITY;
      for (int c0 = 0; c0 < E; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) smax = fmaxf(smax, v[i] + s_off[c0 + i]);
      }
      sden = 0.f;
      for (int c0 = 0; c0 < E; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) sden += expf(v[i] + s_off[c0 + i] - smax);
      }
    }
    auto score = [&](float l, int e) -> float {
      const float z = l + s_off[e];
      if (p.score_func == MOE_SCORE_SOFTMAX) return expf(z - smax) / sden;
      return affinity(z, p.score_func);
    };

    // group scores: sum of the two best biased scores of each group (max without a bias).  Groups are
    // contiguous runs of `per` experts, so the current group's best two stay in registers and each
    // finished group's score goes to shared memory (the drained pipeline stages), [group][thread].
    uint32_t kept = 0xffffffffu;
    const int per = E / p.G;
    if (p.G > 1) {
      float* s_gs = reinterpret_cast<float*>(smem);
      float c1 = -INFINITY, c2 = -INFINITY;
      int cg = 0, next_b = per;
      for (int c0 = 0; c0 < E; c0 += 16) {
        float v[16];
        tmem_ld16(trow + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = c0 + i;
          if (e == next_b) {
            s_gs[cg * kRouterThreads + threadIdx.x] = has_bias ? __fadd_rn(c1, c2) : c1;
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
      s_gs[cg * kRouterThreads + threadIdx.x] = has_bias ? __fadd_rn(c1, c2) : c1;
      kept = 0;
      for (int r = 0; r < p.g; ++r) {  // best remaining group, lower index on ties
        int best = -1;
        float bs = -INFINITY;
        for (int g = 0; g < p.G; ++g) {
          if (kept & (1u << g)) continue;
          const float gs = s_gs[g * kRouterThreads + threadIdx.x];
          if (best < 0 || gs > bs) { best = g; bs = gs; }
        }
        kept |= 1u << best;
      }
    }

    // top-k over the kept experts: sorted descending, equal scores keep the lower index first
    float tb[kMaxTopk], ts[kMaxTopk];
    int ti[kMaxTopk];
#pragma unroll
    for (int j = 0; j < kMaxTopk; ++j) { tb[j] = -INFINITY; ts[j] = 0.f; ti[j] = 0; }
    for (int c0 = 0; c0 < E; c0 += 16) {
      // skip whole chunks that lie in dropped groups (the load is warp-collective, so decide per warp)
      bool any = false;
      for (int i = 0; i < 16; ++i) any |= ((kept >> ((c0 + i) / per)) & 1u) != 0;
      if (!__any_sync(0xffffffffu, any)) continue;
      float v[16];
      tmem_ld16(trow + c0, v);
      tmem_ld_wait();
      const int g0 = c0 / per;
      int bnd = (g0 + 1) * per;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int e = c0 + i;
        const int g = g0 + (e >= bnd ? (e - bnd) / per + 1 : 0);
        if (!((kept >> g) & 1u)) continue;
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

    if (t < p.T) {
      float total_s = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j)
        if (j < p.k) total_s = __fadd_rn(total_s, ts[j]);
#pragma unroll
      for (int j = 0; j < kMaxTopk; ++j) {
        if (j < p.k) {
          float w = ts[j];
          if (p.renorm) w = __fdiv_rn(w, total_s);
          w = __fmul_rn(w, p.route_scale);
          p.indices[(size_t)t * p.k + j] = ti[j];
          p.weights[(size_t)t * p.k + j] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, p.tmem_cols);
}

// ------------------------------------------------------------------------------------------------
// hash gate: one warp per token, k dot products of length d
// ------------------------------------------------------------------------------------------------
__global__ void hash_gate_kernel(HashGateParams p) {
  const int warps = blockDim.x >> 5;
  const int t = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= p.T) return;
  int tok = p.token_ids[t];
  if (tok < 0 || tok >= p.vocab) {
    if (lane == 0) record_error(p.ew, MOE_ERR_DEVICE, tok);
    tok = tok < 0 ? 0 : p.vocab - 1;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.d);
  float s[kMaxTopk];
  int ex[kMaxTopk];
  float total_s = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopk; ++j) {
    if (j >= p.k) break;
    int e = p.tid2eid[(size_t)tok * p.k + j];
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
  gate_planes_kernel<<<grid, 256, 0, stream>>>(w, planes, n, inexact_flag);
  return cudaGetLastError();
}

size_t router_smem_bytes(int E, int stages) {
  return 1024 + (size_t)stages * (128 * 128 + (size_t)E * 128) + sizeof(RouterSmem) + 2 * (size_t)E * sizeof(float);
}

cudaError_t launch_router(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                          cudaStream_t stream) {
  const size_t smem = router_smem_bytes(p.E, p.stages);
  cudaError_t err = cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = (p.T + 127) / 128;
  router_kernel<<<grid, kRouterThreads, smem, stream>>>(map_x, map_w, p);
  return cudaGetLastError();
}

cudaError_t launch_hash_gate(const HashGateParams& p, cudaStream_t stream) {
  const int warps = 8;
  hash_gate_kernel<<<(p.T + warps - 1) / warps, warps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
