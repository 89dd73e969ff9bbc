// Auxiliary-loss-free balancing step ("From One Giant FFN to 384 Tiny Experts", section 6, the
// bias-update rule): once per step, every expert whose load over the batch is above the balanced
// level T*k/E loses gamma from its selection bias, every expert below it gains gamma, and one exactly
// at it keeps its bias.  The comparison is made exactly in integers as counts[e] * E against T * k.
// E <= 512 experts: one block, one thread per expert.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__global__ void update_bias_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias, int E,
                                   long long balanced_times_E, float gamma) {
  pdl_begin();
  const int e = threadIdx.x;
  if (e >= E) return;
  const long long load_times_E = (long long)counts[e] * E;
  const float b = bias[e];
  if (load_times_E > balanced_times_E)
    bias[e] = __fsub_rn(b, gamma);
  else if (load_times_E < balanced_times_E)
    bias[e] = __fadd_rn(b, gamma);
}

}  // namespace

cudaError_t launch_update_bias(const int32_t* counts, float* bias, int E, long long balanced_times_E, float gamma,
                               cudaStream_t stream) {
  const int threads = (E + 31) / 32 * 32;
  return launch_pdl(update_bias_kernel, dim3(1), dim3(threads), 0, stream, counts, bias, E, balanced_times_E, gamma);
}

}  // namespace moe
