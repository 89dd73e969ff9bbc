// moe_dispatch_static: the dispatch of moe_dispatch for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: for example a plugin that a host framework hands only
// its input and output buffers (the framework owns every byte of device memory), or a latency-bound
// loop where an allocation's implicit device synchronisation is not allowed.  Such callers cannot
// provide the workspace that moe_dispatch takes.  This entry point runs the same three kernels with
// their scratch (the per-block expert histograms and row bases) in a fixed array of device memory
// that belongs to the library itself: kStaticScratchInts 32-bit integers (4 MiB), reserved on every
// GPU that loads the library until the process exits.
//
// Rules of use:
// * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
//   device current, and caches it; make that first call before any stream capture.
// * Every call shares the one array, which keeps whatever the last call left in it.  Each kernel
//   writes every scratch entry it later reads, so nothing needs clearing, but calls whose kernels
//   overlap on the GPU (two streams, or two host threads) race on the array and must not be issued.
// * Sizes beyond the array -- ceil(T*k / 128) * E > kStaticScratchInts / 2 -- are rejected with
//   MOE_ERR_UNSUPPORTED before anything is launched.
// * Out-of-range expert indices are clamped, as in moe_dispatch, but not reported: there is no
//   workspace error word to record them in.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr long kStaticScratchInts = 1L << 20;  // 4 MiB: histograms and bases, half each
constexpr int kMaxDevices = 64;

// The library's own scratch.  In host code `g_dispatch_scratch` names a host-side stand-in, not
// device memory: only the address from cudaGetSymbolAddress may be handed to a kernel.
static __device__ __align__(256) int32_t g_dispatch_scratch[kStaticScratchInts];

int32_t* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch on the current device, looked up once per device.
int32_t* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_dispatch_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = static_cast<int32_t*>(ptr);
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" moe_status moe_dispatch_static(const moe_layer_desc* desc, int T, const int32_t* indices,
                                          const moe_bf16* x, int32_t* counts, int32_t* offsets,
                                          int32_t* row_of_slot, int32_t* tok_of_row, moe_bf16* x_perm,
                                          moe_stream_t stream) {
  if (desc == nullptr || desc->n_experts <= 0 || desc->n_experts > 512 || desc->topk <= 0 || desc->topk > 8 ||
      desc->dim <= 0 || desc->dim % 128 != 0)
    return MOE_ERR_INVALID;
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID;
  if (T > 0 && (indices == nullptr || x == nullptr || row_of_slot == nullptr || tok_of_row == nullptr))
    return MOE_ERR_INVALID;   // x_perm may be NULL: the permutation only
  if (T > 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_perm)) & 15u) != 0)
    return MOE_ERR_INVALID;
  const int E = desc->n_experts;
  const long S = (long)T * desc->topk;
  const long nblk = moe::dispatch_blocks(S);
  if (nblk * E > kStaticScratchInts / 2) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  int32_t* scratch = scratch_on_current_device();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  int32_t* hist = scratch;
  int32_t* base = scratch + kStaticScratchInts / 2;
  const cudaError_t err = moe::launch_dispatch(indices, (int)S, desc->topk, E,
                                               reinterpret_cast<const __nv_bfloat16*>(x), desc->dim, hist, base,
                                               counts, offsets, row_of_slot, tok_of_row,
                                               reinterpret_cast<__nv_bfloat16*>(x_perm), nullptr, s);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
