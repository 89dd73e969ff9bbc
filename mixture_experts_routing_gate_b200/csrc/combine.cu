// Combine: "DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt (fp32 accumulator
// y[idx] += expert(x[idx]) * w, then y += shared_experts(x)) and "DeepSeek V4.1 - Add shared"
// (cast back to the input dtype).  A gather formulation: one block per token reads its k expert
// rows and the shared row, so each output element is summed by one thread in a fixed order
// (slot order, shared term last) with no atomics -- the result is deterministic.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxCombineK = 8;   // topk <= 8 (checked with the layer descriptor)

__global__ void __launch_bounds__(128) combine_kernel(const __nv_bfloat16* __restrict__ out_perm,
                                                      const int32_t* __restrict__ row_of_slot,
                                                      const float* __restrict__ weights,
                                                      const __nv_bfloat16* __restrict__ out_shared,
                                                      __nv_bfloat16* __restrict__ y, int T, int k, int d, int S) {
  pdl_begin();
  __shared__ int s_row[16];
  __shared__ float s_w[16];
  const int nvec = d / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      int r = row_of_slot[(size_t)t * k + threadIdx.x];
      s_row[threadIdx.x] = r < 0 ? 0 : (r >= S ? S - 1 : r);
      s_w[threadIdx.x] = weights != nullptr ? weights[(size_t)t * k + threadIdx.x] : 1.f;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      // all k expert rows and the shared row in flight at once, then summed in slot order
      uint4 ov[kMaxCombineK];
#pragma unroll
      for (int j = 0; j < kMaxCombineK; ++j)
        if (j < k) ov[j] = __ldcs(reinterpret_cast<const uint4*>(out_perm + (size_t)s_row[j] * d) + v);
      uint4 sv = make_uint4(0u, 0u, 0u, 0u);
      if (out_shared != nullptr) sv = __ldcs(reinterpret_cast<const uint4*>(out_shared + (size_t)t * d) + v);
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxCombineK; ++j) {
        if (j >= k) break;
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov[j]);
        const float w = s_w[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(o2[i]);
          acc[2 * i] = __fadd_rn(acc[2 * i], weights != nullptr ? __fmul_rn(f.x, w) : f.x);
          acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], weights != nullptr ? __fmul_rn(f.y, w) : f.y);
        }
      }
      if (out_shared != nullptr) {
        const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(&sv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(s2[i]);
          acc[2 * i] = __fadd_rn(acc[2 * i], f.x);
          acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], f.y);
        }
      }
      uint4 outv;
      __nv_bfloat162* out2 = reinterpret_cast<__nv_bfloat162*>(&outv);
#pragma unroll
      for (int i = 0; i < 4; ++i) out2[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      reinterpret_cast<uint4*>(y + (size_t)t * d)[v] = outv;
    }
    __syncthreads();
  }
}

cudaError_t launch_combine(const __nv_bfloat16* out_perm, const int32_t* row_of_slot, const float* weights,
                           const __nv_bfloat16* out_shared, __nv_bfloat16* y, int T, int k, int d, int S, int num_sms,
                           cudaStream_t stream) {
  const int grid = T < 16 * num_sms ? T : 16 * num_sms;
  return launch_pdl(combine_kernel, dim3(grid), dim3(128), 0, stream, out_perm, row_of_slot, weights, out_shared, y, T,
                    k, d, S);
}

}  // namespace moe
