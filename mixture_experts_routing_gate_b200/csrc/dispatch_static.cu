// moe_dispatch_static: the dispatch of moe_dispatch for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: for example a plugin that a host framework hands only
// its input and output buffers (the framework owns every byte of device memory), or a latency-bound
// loop where an allocation's implicit device synchronisation is not allowed.  Such callers cannot
// provide the workspace that moe_dispatch takes.  This entry point runs the same two kernels with
// their scratch (the histogram blocks' finishing ticket, the per-block expert histograms and row
// bases) in a fixed array of device memory that belongs to the library itself: kStaticScratchInts
// 32-bit integers (1 MiB), reserved on every GPU that loads the library until the process exits.
//
// Rules of use:
// * Every call looks up the array's device address on the current device (cudaGetSymbolAddress,
//   with that device current) before it launches anything; the first call on a device may
//   initialise the module there, so make it before any stream capture.
// * Every call shares the one array, which keeps whatever the last call left in it.  Each call
//   clears the ticket (an asynchronous 4-byte memset on its stream) and its kernels write every
//   other scratch entry before reading it, but calls whose kernels overlap on the GPU (two streams,
//   or two host threads) race on the array and must not be issued.
// * Sizes beyond the array -- n_coarse * E > kStaticCap, where n_coarse = dispatch_plan(T*k).n_coarse
//   (about 64 for up to 2^19 slots, T*k / 8192 beyond) -- are rejected with MOE_ERR_UNSUPPORTED
//   before anything is launched.
// * Out-of-range expert indices are clamped, as in moe_dispatch, but not reported: there is no
//   workspace error word to record them in.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr long kStaticScratchInts = 1L << 18;   // 1 MiB
constexpr long kStaticHead = 64;                // the ticket, padded to 256 bytes
constexpr long kStaticCap = (kStaticScratchInts - kStaticHead) / 2;   // ints of hist, and of base

// The library's own scratch.  In host code `g_dispatch_scratch` names a host-side stand-in, not
// device memory: only the address from cudaGetSymbolAddress may be handed to a kernel.
static __device__ __align__(256) int32_t g_dispatch_scratch[kStaticScratchInts];

}  // namespace

extern "C" moe_status moe_dispatch_static(const moe_layer_desc* desc, int T, const int32_t* indices,
                                          const moe_bf16* x, int32_t* counts, int32_t* offsets,
                                          int32_t* row_of_slot, int32_t* tok_of_row, moe_bf16* x_perm,
                                          moe_stream_t stream) {
  moe::NvtxRange nvtx("moe_dispatch_static");
  const moe_status st = moe::check_layer_desc(desc);   // the same descriptors as moe_dispatch
  if (st != MOE_OK) return st;
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID;
  if (T > 0 && (indices == nullptr || x == nullptr || row_of_slot == nullptr || tok_of_row == nullptr))
    return MOE_ERR_INVALID;   // x_perm may be NULL: the permutation only
  if (T > 0 && ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_perm)) & 15u) != 0)
    return MOE_ERR_INVALID;
  const int E = desc->n_experts;
  const long S = (long)T * desc->topk;
  if ((long)moe::dispatch_plan(S, desc->topk, 148).n_coarse * E > kStaticCap) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_dispatch_scratch) != cudaSuccess || addr == nullptr) return MOE_ERR_CUDA;
  int32_t* scratch = static_cast<int32_t*>(addr);
  int* ticket = scratch;
  int32_t* hist = scratch + kStaticHead;
  int32_t* base = hist + kStaticCap;
  if (cudaMemsetAsync(ticket, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  const moe::RowCopy rc = moe::row_copy_bf16(reinterpret_cast<const __nv_bfloat16*>(x), desc->dim,
                                             reinterpret_cast<__nv_bfloat16*>(x_perm));
  const cudaError_t err = moe::launch_dispatch(indices, (int)S, desc->topk, E, rc, hist, base, ticket, counts, offsets,
                                               row_of_slot, tok_of_row, nullptr, s);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
