// The C ABI of libmoe (declared in include/moe.h): argument checks, the workspace layout, TMA
// tensor maps, and the launch sequences of every entry point.  Nothing here computes layer values;
// every step runs in the kernels of router.cu, dispatch.cu, expert_gemm.cu and combine.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_PDL");
    return v == nullptr || v[0] != '0';
  }();
  return on;
}

}  // namespace moe

namespace {

using moe::NvtxRange;

using moe::ErrorWord;

constexpr size_t kAlign = 1024;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
constexpr size_t kPreparedHeader = 1024;   // prepared router weight: flag word, then the three planes

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------------------------
// layer checks
// ---------------------------------------------------------------------------------------------
moe_status check_desc(const moe_layer_desc* d) {
  if (d == nullptr) return MOE_ERR_INVALID;
  if (d->dim <= 0 || d->n_experts <= 0 || d->n_groups <= 0 || d->n_limited_groups <= 0 || d->topk <= 0 ||
      d->inter_dim <= 0)
    return MOE_ERR_INVALID;
  if (d->n_experts % d->n_groups != 0) return MOE_ERR_INVALID;
  if (d->n_limited_groups > d->n_groups) return MOE_ERR_INVALID;
  if (d->topk > d->n_limited_groups * (d->n_experts / d->n_groups)) return MOE_ERR_INVALID;
  if (d->score_func < MOE_SCORE_SIGMOID || d->score_func > MOE_SCORE_SOFTMAX) return MOE_ERR_INVALID;
  if (d->n_shared != 1) return MOE_ERR_UNSUPPORTED;
  if (d->dim % 128 != 0 || d->inter_dim % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (d->n_experts % 16 != 0 || d->n_experts > 512) return MOE_ERR_UNSUPPORTED;
  if (d->n_experts > 256 && d->n_experts % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (d->topk > 8 || d->n_groups > 32) return MOE_ERR_UNSUPPORTED;
  if (!(d->swiglu_limit >= 0.f) || (d->weight_in_expert != 0 && d->weight_in_expert != 1)) return MOE_ERR_INVALID;
  if ((d->options & ~(MOE_OPT_ROUTER_ONE_CTA | MOE_OPT_GEMM_ONE_CTA | MOE_OPT_FUSED_GATHER |
                      MOE_OPT_MXFP4_BF16_ACTIVATIONS)) != 0)
    return MOE_ERR_INVALID;
  if (d->token_chunk != 0 && d->token_chunk != 96 && d->token_chunk != 128 && d->token_chunk != 224 &&
      d->token_chunk != 256)
    return MOE_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(d->gate_prepared) & 15u) != 0) return MOE_ERR_INVALID;
  return MOE_OK;
}

}  // namespace

namespace moe {
moe_status check_layer_desc(const moe_layer_desc* d) { return check_desc(d); }
}  // namespace moe

namespace {

// ---------------------------------------------------------------------------------------------
// workspace layout: every region starts on a 1 KiB boundary
// ---------------------------------------------------------------------------------------------
// The block-scaled MXFP4 path keeps E4M3 codes and their scales in the regions of x_perm and h (codes
// first, the scales 1 KiB-aligned after them) and the quantised x in a region of its own.
struct WsLayout {
  size_t err, flag, planes, indices, weights, counts, offsets, row_of_slot, tok_of_row, w_perm, hist, base,
      chunk_prefix, x_perm, h, out_perm, out_shared, xq, total;
  size_t xp_scales, h_scales, xq_scales;   // offsets of the scales inside x_perm, h and xq
};

WsLayout ws_layout(const moe_layer_desc& d, int T) {
  const size_t E = d.n_experts, D = d.dim, I = d.inter_dim, S = (size_t)T * d.topk;
  // histogram blocks: the histogram kernel's (independent of the SM count) or the cluster router's
  // (up to 8 per 128-token tile) when moe_forward fuses the histogram into it
  const size_t nblk = std::max((size_t)moe::dispatch_plan((long)S, d.topk, 148).n_coarse, ((size_t)T + 127) / 128 * 8);
  WsLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  L.err = take(sizeof(ErrorWord));
  L.flag = take(sizeof(int));
  L.planes = take(3 * E * D * 2);
  L.indices = take(S * 4);
  L.weights = take(S * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.row_of_slot = take(S * 4);
  L.tok_of_row = take(S * 4);
  L.w_perm = take(S * 4);
  L.hist = take(nblk * E * 4);
  L.base = take(nblk * E * 4);
  L.chunk_prefix = take((E + 2) * 4);
  const auto codes_and_scales = [](size_t n) { return align_up(n) + align_up(n / 32); };
  L.x_perm = take(std::max(S * D * 2, codes_and_scales(S * D)));
  L.xp_scales = L.x_perm + align_up(S * D);
  L.h = take(std::max((S + T) * I * 2, codes_and_scales((S + T) * I)));
  L.h_scales = L.h + align_up((S + T) * I);
  L.out_perm = take(S * D * 2);
  L.out_shared = take((size_t)T * D * 2);
  L.xq = take(codes_and_scales((size_t)T * D));
  L.xq_scales = L.xq + align_up((size_t)T * D);
  L.total = o;
  return L;
}

template <typename Ptr>
Ptr* at(void* ws, size_t off) {
  return reinterpret_cast<Ptr*>(static_cast<uint8_t*>(ws) + off);
}

moe_status check_ws(const moe_layer_desc& d, int T, void* ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return MOE_ERR_WORKSPACE;
  if (ws_bytes < ws_layout(d, T).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// ---------------------------------------------------------------------------------------------
// device properties and tensor maps
// ---------------------------------------------------------------------------------------------
int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [rows, cols] bf16 matrix, boxes of [box_rows, 64] (128 bytes wide, 128-byte swizzle).
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows, row_bytes] packed E2M1 codes, boxes of 128 rows x 32 bytes (64 codes), unswizzled.
bool make_map_fp4(CUtensorMap* map, const void* base, uint64_t rows, uint64_t row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {32, (cuuint32_t)moe::kGemmBM};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows, K/32] UE8M0 block scales, boxes of 128 rows x 16 bytes (the scales of 8 K steps).
bool make_map_scales(CUtensorMap* map, const void* base, uint64_t rows, uint64_t row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {16, (cuuint32_t)moe::kGemmBM};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed E2M1 codes [rows, K elements] (two per byte) as the block-scaled MMAs read them: TMA spreads
// each 16 codes over 16 bytes of shared memory (type 16U4_ALIGN16B); boxes of 128 rows x 128 elements
// (the type's fixed inner box), 128-byte swizzle.  Base 32-byte aligned, K % 128 == 0.
bool make_map_e2m1(CUtensorMap* map, const void* base, uint64_t rows, uint64_t K) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K / 2};
  const cuuint32_t box[2] = {128, (cuuint32_t)moe::kGemmBM};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major [rows, cols] bytes in boxes of box_rows x box_cols bytes (128-byte swizzle when
// box_cols == 128: E4M3 token rows as the MMA reads them; none for the 16-byte scale boxes).
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                      \
  do {                                     \
    const moe_status _s = (expr);          \
    if (_s != MOE_OK) return _s;           \
  } while (0)

// ---------------------------------------------------------------------------------------------
// launch sequences (arguments already checked)
// ---------------------------------------------------------------------------------------------
// Hash-routed selection handed to the cluster router (mode 1: token-id table, mode 2: 2-gram hash).
// Dispatch's histogram fused into the cluster router (moe_forward): the buffers it fills, and the
// slots per histogram block it used (0 when the gate ran another kernel and dispatch must count).
struct FusedHist {
  int32_t* hist = nullptr;
  int32_t* base = nullptr;
  int32_t* counts = nullptr;
  int32_t* offsets = nullptr;
  int* ticket = nullptr;
  int coarse = 0;
};

struct HashSelect {
  int mode = 0;
  int vocab = 0;
  const int32_t* token_ids = nullptr;
  const int32_t* prev_ids = nullptr;
  const int32_t* tid2eid = nullptr;
  const int64_t* primes = nullptr;
};

bool router_single_forced(const moe_layer_desc& d) { return (d.options & MOE_OPT_ROUTER_ONE_CTA) != 0; }

#ifdef MOE_TEST_HOOKS
// Failure-detection test hook, compiled only into the test build of the library (libmoe_testhooks.so):
// while set, the CTA-pair expert GEMMs' producers issue no loads, so every consumer's bounded wait runs
// out, records MOE_ERR_TIMEOUT and the kernels return.
int g_test_stall = 0;
#endif
int test_stall_flag() {
#ifdef MOE_TEST_HOOKS
  return g_test_stall;
#else
  return 0;
#endif
}

// The tcgen05 router: logits of all experts, then group-limited top-k, or (hs != null) the hash
// selection, which only the split-K cluster router implements.
moe_status run_gate(const moe_layer_desc& d, int T, const moe_bf16* x, const float* w_gate, const float* bias,
                    const float* logit_offset, float* weights, int32_t* indices, void* ws, cudaStream_t stream,
                    const HashSelect* hs = nullptr, FusedHist* fh = nullptr) {
  const WsLayout L = ws_layout(d, T);
  const int E = d.n_experts;
  // the bf16 planes of w_gate and their flag: prepared once by moe_gate_prepare, else split per call
  const int* flag;
  const __nv_bfloat16* planes;
  if (d.gate_prepared != nullptr) {
    flag = static_cast<const int*>(d.gate_prepared);
    planes = reinterpret_cast<const __nv_bfloat16*>(static_cast<const uint8_t*>(d.gate_prepared) + kPreparedHeader);
  } else {
    int* f = at<int>(ws, L.flag);
    __nv_bfloat16* pl = at<__nv_bfloat16>(ws, L.planes);
    MOE_TRY(cuda_status(cudaMemsetAsync(f, 0, sizeof(int), stream)));
    MOE_TRY(cuda_status(moe::launch_gate_planes(w_gate, pl, (long)E * d.dim, f, num_sms(), stream)));
    flag = f;
    planes = pl;
  }
  moe::RouterParams p{};
  p.T = T; p.d = d.dim; p.E = E; p.G = d.n_groups; p.g = d.n_limited_groups; p.k = d.topk;
  p.score_func = d.score_func; p.renorm = d.renorm; p.route_scale = d.route_scale;
  p.n_split = E > 256 ? 2 : 1;
  p.n_half = E / p.n_split;
  p.tmem_cols = 32;
  while (p.tmem_cols < E) p.tmem_cols <<= 1;
  const size_t stage = 128 * 128 + (size_t)E * 128;
  p.stages = (int)((200 * 1024) / stage);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) return MOE_ERR_UNSUPPORTED;
  p.bias = bias; p.logit_offset = logit_offset; p.plane_flag = flag;
  p.weights = weights; p.indices = indices; p.ew = at<ErrorWord>(ws, L.err);
  if (hs != nullptr) {
    p.sel_mode = hs->mode; p.vocab = hs->vocab;
    p.token_ids = hs->token_ids; p.prev_ids = hs->prev_ids; p.tid2eid = hs->tid2eid;
    for (int j = 0; hs->primes != nullptr && j < d.topk; ++j) p.primes[j] = (unsigned long long)hs->primes[j];
  }
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, T, d.dim, 128)) return MOE_ERR_CUDA;
  if (!make_map(&mw, planes, 3 * (uint64_t)E, d.dim, p.n_half)) return MOE_ERR_CUDA;

  // The split-K cluster router, where its epilogue's lane layout fits (E = 16 x {1,2,4,8,16,24}, G
  // dividing 16); MOE_OPT_ROUTER_ONE_CTA selects the one-CTA-per-tile router.
  if (!router_single_forced(d) && moe::router_cluster_supported(E, hs != nullptr ? 1 : d.n_groups)) {
    const int tiles = (T + 127) / 128, nk = d.dim / 64;
    int ks = 8;
    while (ks > 1 && ((long)tiles * ks > num_sms() || ks > nk)) ks >>= 1;
    p.ksplit = ks;
    p.e_pad = E + 4;   // rows 16 bytes apart in bank terms: conflict-free 16-byte stores down a column
    const size_t recv = (size_t)128 * p.e_pad * sizeof(float);
    const size_t region = p.stages * stage > recv ? p.stages * stage : recv;
    p.region_bytes = (int)((region + 1023) / 1024 * 1024);
    if (fh != nullptr) {
      p.hist = fh->hist; p.base = fh->base; p.counts = fh->counts; p.offsets = fh->offsets; p.ticket = fh->ticket;
    }
    if (moe::router_cluster_smem_bytes(p) <= 227 * 1024) {
      MOE_TRY(cuda_status(moe::launch_router_cluster(mx, mw, p, stream)));
      if (fh != nullptr) fh->coarse = (128 / ks) * d.topk;
      return MOE_OK;
    }
    p.hist = nullptr;
  }
  if (hs != nullptr) return MOE_ERR_UNSUPPORTED;   // callers check hash_on_tensor_cores first
  p.nsplit = E % 64 == 0 ? 4 : (E % 32 == 0 ? 2 : 1);
  const size_t epi = moe::router_epilogue_bytes(p.nsplit, d.n_groups, d.topk);
  const size_t region = p.stages * stage > epi ? p.stages * stage : epi;
  p.region_bytes = (int)((region + 1023) / 1024 * 1024);
  return cuda_status(moe::launch_router(mx, mw, p, stream));
}

// Whether the hash gates run on the cluster router (all logits on the tensor cores, then the table's
// experts picked out), or one warp per token computes just the k dot products.
bool hash_on_tensor_cores(const moe_layer_desc& d, int T) {
  if (router_single_forced(d) || !moe::router_cluster_supported(d.n_experts, 1)) return false;
  const size_t stage = 128 * 128 + (size_t)d.n_experts * 128;
  const size_t recv = (size_t)128 * (d.n_experts + 4) * sizeof(float);
  const size_t region = std::max<size_t>(std::min<size_t>(8, (200 * 1024) / stage) * stage, recv);
  return 1024 + region + 4096 <= 227 * 1024 && T > 0;
}

// tid2eid != null: the token-id table; otherwise the 2-gram hash of (prev_ids, token_ids) with primes.
moe_status run_hash_gate(const moe_layer_desc& d, int T, const int32_t* token_ids, const int32_t* tid2eid, int vocab,
                         const moe_bf16* x, const float* w_gate, float* weights, int32_t* indices, void* ws,
                         cudaStream_t stream, const int32_t* prev_ids = nullptr, const int64_t* primes = nullptr,
                         FusedHist* fh = nullptr) {
  if (hash_on_tensor_cores(d, T)) {
    HashSelect hs;
    hs.mode = tid2eid != nullptr ? 1 : 2;
    hs.vocab = vocab; hs.token_ids = token_ids; hs.prev_ids = prev_ids; hs.tid2eid = tid2eid; hs.primes = primes;
    return run_gate(d, T, x, w_gate, nullptr, nullptr, weights, indices, ws, stream, &hs, fh);
  }
  const WsLayout L = ws_layout(d, T);
  moe::HashGateParams p{};
  p.T = T; p.d = d.dim; p.E = d.n_experts; p.k = d.topk; p.vocab = vocab;
  p.score_func = d.score_func; p.renorm = d.renorm; p.route_scale = d.route_scale;
  p.token_ids = token_ids; p.tid2eid = tid2eid; p.prev_ids = prev_ids;
  for (int j = 0; primes != nullptr && j < d.topk; ++j) p.primes[j] = (unsigned long long)primes[j];
  p.x = reinterpret_cast<const __nv_bfloat16*>(x); p.w_gate = w_gate;
  p.weights = weights; p.indices = indices; p.ew = at<ErrorWord>(ws, L.err);
  return cuda_status(moe::launch_hash_gate(p, stream));
}

moe_status run_dispatch_rows(const moe_layer_desc& d, int T, const int32_t* indices, const moe::RowCopy& rc,
                             int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* tok_of_row, void* ws,
                             cudaStream_t stream, const float* weights = nullptr, float* w_perm = nullptr) {
  const WsLayout L = ws_layout(d, T);
  const int S = T * d.topk;
  ErrorWord* ew = at<ErrorWord>(ws, L.err);
  return cuda_status(moe::launch_dispatch(indices, S, d.topk, d.n_experts, rc, at<int32_t>(ws, L.hist),
                                          at<int32_t>(ws, L.base), &ew->dispatch_ticket, counts, offsets, row_of_slot,
                                          tok_of_row, ew, stream, weights, w_perm));
}

moe_status run_dispatch(const moe_layer_desc& d, int T, const int32_t* indices, const moe_bf16* x, int32_t* counts,
                        int32_t* offsets, int32_t* row_of_slot, int32_t* tok_of_row, moe_bf16* x_perm, void* ws,
                        cudaStream_t stream, const float* weights = nullptr, float* w_perm = nullptr) {
  const moe::RowCopy rc = moe::row_copy_bf16(reinterpret_cast<const __nv_bfloat16*>(x), d.dim,
                                             reinterpret_cast<__nv_bfloat16*>(x_perm));
  return run_dispatch_rows(d, T, indices, rc, counts, offsets, row_of_slot, tok_of_row, ws, stream, weights, w_perm);
}

// The quantised rows of x (codes and scales in the workspace's xq region) as the scatter's copy
// into the x_perm region.
moe::RowCopy row_copy_mx(const moe_layer_desc& d, int T, void* ws) {
  const WsLayout L = ws_layout(d, T);
  moe::RowCopy rc{};
  rc.nseg = 2;
  rc.bytes[0] = d.dim;
  rc.bytes[1] = d.dim / 32;
  rc.src[0] = at<uint8_t>(ws, L.xq);
  rc.src[1] = at<uint8_t>(ws, L.xq_scales);
  rc.dst[0] = at<uint8_t>(ws, L.x_perm);
  rc.dst[1] = at<uint8_t>(ws, L.xp_scales);
  return rc;
}

// The CTA-pair kernels need I % 256 == 0 (up projections) and d % 256 == 0 (down projection);
// MOE_OPT_GEMM_ONE_CTA selects the single-CTA kernels for every shape (bf16 weights only: MXFP4 runs
// on the pair kernels alone).
bool single_cta_forced(const moe_layer_desc& d, bool fp4) { return !fp4 && (d.options & MOE_OPT_GEMM_ONE_CTA) != 0; }

// Rows per box of the CTA-pair kernels' wide token-row maps (the narrow maps hold 16 rows; the
// double-wide ones twice this).
constexpr uint32_t kWideBoxRows = 64;

// Whether the up-projection kernel can gather the token rows of x itself (tile::gather4 loads on the
// CTA-pair kernel), and whether the forward lets it instead of having dispatch write x_perm first.
// The forward keeps the separate gather unless MOE_OPT_FUSED_GATHER is set: on the V3-shaped prefill
// layer the gathered up projection measured about 20 % slower than the one that streams x_perm in
// 16-row boxes, more than the gather kernel it saves.
bool gather_supported(const moe_layer_desc& d, bool fp4) { return !single_cta_forced(d, fp4) && d.inter_dim % 256 == 0; }

bool fused_gather(const moe_layer_desc& d, bool fp4) {
  return (d.options & MOE_OPT_FUSED_GATHER) != 0 && gather_supported(d, fp4);
}

// fp4 != null: MXFP4 weights (w1 / w3 / w2 unused); the CTA-pair kernels only (I % 256 == 0, d % 256 == 0,
// checked by the entry points).  gather_rows != null: the routed B rows of the up projections are rows
// gather_rows[r] of x (x_perm unused); the CTA-pair kernel only.
moe_status run_experts(const moe_layer_desc& d, int T, const moe_bf16* x_perm, const int32_t* offsets,
                       const float* row_weights, const moe_bf16* x, const moe_bf16* w1, const moe_bf16* w3,
                       const moe_bf16* w2, moe_bf16* out_perm, moe_bf16* out_shared, void* ws, cudaStream_t stream,
                       const moe_mxfp4_weights* fp4 = nullptr, const int32_t* gather_rows = nullptr) {
  const WsLayout L = ws_layout(d, T);
  const int E = d.n_experts, D = d.dim, I = d.inter_dim, S = T * d.topk;
  int32_t* prefix = at<int32_t>(ws, L.chunk_prefix);
  __nv_bfloat16* H = at<__nv_bfloat16>(ws, L.h);
  ErrorWord* ew = at<ErrorWord>(ws, L.err);
  const bool single = single_cta_forced(d, fp4 != nullptr);
  const bool fp4_weights = fp4 != nullptr;
  const int test_stall = test_stall_flag();   // always 0 outside the test build
  // Token chunks of up to 256 rows when experts expect at least 16 rows each: an expert of 129..256
  // rows then streams its weights once instead of once per 128-row chunk (the MMA's N follows the
  // chunk's rows, rounded up to 32, so a short chunk wastes little); 128 otherwise, where the second
  // TMEM accumulator buffer lets the epilogue overlap the next tile.  The down projection holds two
  // 128-row weight tiles per CTA (one when d is an odd multiple of 256).
  const bool big = (long)S >= 16L * E;
  // Two w2 tiles per CTA (512 output features per pair tile) even though their accumulators then
  // fill TMEM: one tile per CTA with double-buffered accumulators measured 6-12 % slower.
  const int down_mode = D % 512 == 0 ? moe::kGemmPair : moe::kGemmSingle;
  const bool pair_up = !single && I % 256 == 0;
  const bool pair_down = !single && D % 256 == 0;
  int bn = (pair_up && pair_down && big) ? 256 : 128;
  if (pair_up && pair_down && d.token_chunk != 0) bn = d.token_chunk;   // the caller's chunk size
  MOE_TRY(cuda_status(moe::launch_expert_tiles(offsets, E, T, S, bn, prefix, ew, stream)));

  const int sms = num_sms();
  const long chunk_bound = (S + bn - 1) / bn + E + (T + bn - 1) / bn;

  // up projections + SwiGLU: A = w1 / w3 rows [(E+1) I, d], B = x_perm (routed) or x (shared)
  {
    CUtensorMap ma0, ma1, mbr, mbs;
    const uint32_t brows = pair_up ? 16 : 32;
    if (fp4 != nullptr) {
      if (!make_map_fp4(&ma0, fp4->w1, (uint64_t)(E + 1) * I, D / 2)) return MOE_ERR_CUDA;
      if (!make_map_fp4(&ma1, fp4->w3, (uint64_t)(E + 1) * I, D / 2)) return MOE_ERR_CUDA;
    } else {
      if (!make_map(&ma0, w1, (uint64_t)(E + 1) * I, D, moe::kGemmBM)) return MOE_ERR_CUDA;
      if (!make_map(&ma1, w3, (uint64_t)(E + 1) * I, D, moe::kGemmBM)) return MOE_ERR_CUDA;
    }
    if (pair_up && gather_rows != nullptr) {
      if (!make_map(&mbr, x, T, D, 1)) return MOE_ERR_CUDA;
    } else {
      if (x_perm == nullptr) return MOE_ERR_INVALID;
      if (!make_map(&mbr, x_perm, S, D, brows)) return MOE_ERR_CUDA;
    }
    if (!make_map(&mbs, x, T, D, brows)) return MOE_ERR_CUDA;
    moe::GemmParams p{};
    p.chunk_prefix = prefix; p.offsets = offsets; p.E = E; p.T = T; p.S = S;
    p.K = D; p.M_total = I; p.bn = bn;
    p.swiglu_limit = d.swiglu_limit; p.row_weight = row_weights; p.test_stall = test_stall;
    p.gather_rows = pair_up ? gather_rows : nullptr;
    p.shared_b_row = 0; p.out_routed = H; p.out_shared = H + (size_t)S * I; p.ew = ew;
    CUtensorMap ms0, ms1;
    if (fp4 != nullptr) {
      if (!make_map_scales(&ms0, fp4->w1_scale, (uint64_t)(E + 1) * I, D / 32)) return MOE_ERR_CUDA;
      if (!make_map_scales(&ms1, fp4->w3_scale, (uint64_t)(E + 1) * I, D / 32)) return MOE_ERR_CUDA;
    }
    if (pair_up) {
      p.m_rows = 2 * moe::kGemmBM; p.m_tiles = I / p.m_rows;
      const long tiles = chunk_bound * p.m_tiles;
      const int clusters = (int)(tiles < sms / 2 ? tiles : sms / 2);
      // the same token rows in 128- and 64-row boxes, for whole blocks of a tile (fewer TMA operations)
      CUtensorMap mbrw, mbsw, mbrx, mbsx;
      p.b_wide = p.gather_rows != nullptr ? 0 : kWideBoxRows;
      if (p.b_wide > 0) {
        if (!make_map(&mbrw, x_perm, S, D, kWideBoxRows)) return MOE_ERR_CUDA;
        if (!make_map(&mbsw, x, T, D, kWideBoxRows)) return MOE_ERR_CUDA;
        if (!make_map(&mbrx, x_perm, S, D, 2 * kWideBoxRows)) return MOE_ERR_CUDA;
        if (!make_map(&mbsx, x, T, D, 2 * kWideBoxRows)) return MOE_ERR_CUDA;
      }
      MOE_TRY(cuda_status(moe::launch_expert_gemm_pair(moe::kGemmSwiGLU, ma0, ma1, mbr, mbs, p, clusters, stream,
                                                       fp4_weights ? &ms0 : nullptr, fp4_weights ? &ms1 : nullptr,
                                                       p.b_wide > 0 ? &mbrw : nullptr, p.b_wide > 0 ? &mbsw : nullptr,
                                                       p.b_wide > 0 ? &mbrx : nullptr, p.b_wide > 0 ? &mbsx : nullptr)));
    } else {
      p.m_tiles = I / moe::kGemmBM; p.m_rows = moe::kGemmBM;
      p.stages = moe::expert_gemm_stages(moe::kGemmSwiGLU);
      const long tiles = chunk_bound * p.m_tiles;
      const int grid = (int)(tiles < sms ? tiles : sms);
      MOE_TRY(cuda_status(moe::launch_expert_gemm(moe::kGemmSwiGLU, ma0, ma1, mbr, mbs, p, grid, stream)));
    }
  }
  // down projection: A = w2 rows [(E+1) d, I], B = H rows [S + T, I]
  {
    CUtensorMap ma0, mb;
    if (fp4 != nullptr) {
      if (!make_map_fp4(&ma0, fp4->w2, (uint64_t)(E + 1) * D, I / 2)) return MOE_ERR_CUDA;
    } else {
      if (!make_map(&ma0, w2, (uint64_t)(E + 1) * D, I, moe::kGemmBM)) return MOE_ERR_CUDA;
    }
    if (!make_map(&mb, H, (uint64_t)S + T, I, pair_down ? 16 : 32)) return MOE_ERR_CUDA;
    moe::GemmParams p{};
    p.chunk_prefix = prefix; p.offsets = offsets; p.E = E; p.T = T; p.S = S;
    p.K = I; p.M_total = D; p.bn = bn;
    p.shared_b_row = S; p.test_stall = test_stall;
    p.out_routed = reinterpret_cast<__nv_bfloat16*>(out_perm);
    p.out_shared = reinterpret_cast<__nv_bfloat16*>(out_shared);
    p.ew = ew;
    CUtensorMap ms0;
    if (fp4 != nullptr && !make_map_scales(&ms0, fp4->w2_scale, (uint64_t)(E + 1) * D, I / 32)) return MOE_ERR_CUDA;
    if (pair_down) {
      p.m_rows = (down_mode == moe::kGemmSingle ? 2 : 4) * moe::kGemmBM; p.m_tiles = D / p.m_rows;
      const long tiles = chunk_bound * p.m_tiles;
      const int clusters = (int)(tiles < sms / 2 ? tiles : sms / 2);
      CUtensorMap mbw, mbx;
      p.b_wide = kWideBoxRows;
      if (!make_map(&mbw, H, (uint64_t)S + T, I, kWideBoxRows)) return MOE_ERR_CUDA;
      if (!make_map(&mbx, H, (uint64_t)S + T, I, 2 * kWideBoxRows)) return MOE_ERR_CUDA;
      MOE_TRY(cuda_status(moe::launch_expert_gemm_pair(down_mode, ma0, ma0, mb, mb, p, clusters, stream,
                                                       fp4_weights ? &ms0 : nullptr, fp4_weights ? &ms0 : nullptr,
                                                       &mbw, &mbw, &mbx, &mbx)));
    } else {
      const int mode = (D / moe::kGemmBM) % 2 == 0 ? moe::kGemmPair : moe::kGemmSingle;
      p.m_rows = mode == moe::kGemmPair ? 2 * moe::kGemmBM : moe::kGemmBM; p.m_tiles = D / p.m_rows;
      p.stages = moe::expert_gemm_stages(mode);
      const long tiles = chunk_bound * p.m_tiles;
      const int grid = (int)(tiles < sms ? tiles : sms);
      MOE_TRY(cuda_status(moe::launch_expert_gemm(mode, ma0, ma0, mb, mb, p, grid, stream)));
    }
  }
  return MOE_OK;
}

// MXFP4 weights on the block-scaled tensor cores: E4M3 activations with UE8M0 scales, already in the
// workspace (routed rows: codes at L.x_perm, scales at L.xp_scales; x: L.xq, L.xq_scales).  h is
// written as codes + scales into the h region; out_perm / out_shared are bf16.
moe_status run_experts_mx(const moe_layer_desc& d, int T, const int32_t* offsets, const float* row_weights,
                          const moe_mxfp4_weights* fp4, moe_bf16* out_perm, moe_bf16* out_shared, void* ws,
                          cudaStream_t stream) {
  const WsLayout L = ws_layout(d, T);
  const int E = d.n_experts, D = d.dim, I = d.inter_dim, S = T * d.topk;
  int32_t* prefix = at<int32_t>(ws, L.chunk_prefix);
  ErrorWord* ew = at<ErrorWord>(ws, L.err);
  // token chunks of 224 rows, or of 96 when no group can hold more (T <= 96: the tensor core's N and
  // the token loads shrink, and the accumulators get two buffers), unless the caller chose; batches
  // of at most 64 tokens run one CTA per tile (64-row chunks), whose MMA threads issue twice as often
  // per SM as a pair's
  const bool solo = d.token_chunk == 0 && T <= moe::kMxSoloChunk;
  const int bn = solo ? moe::kMxSoloChunk
                      : (d.token_chunk != 0 ? d.token_chunk
                                            : (T <= moe::kMxTwoBufChunk ? moe::kMxTwoBufChunk : moe::kMxMaxChunk));
  const int cta_per_tile = solo ? 1 : 2;
  MOE_TRY(cuda_status(moe::launch_expert_tiles(offsets, E, T, S, bn, prefix, ew, stream)));
  const int sms = num_sms();
  const long chunk_bound = (S + bn - 1) / bn + E + (T + bn - 1) / bn;
  uint8_t* xp = at<uint8_t>(ws, L.x_perm);
  uint8_t* xp_s = at<uint8_t>(ws, L.xp_scales);
  uint8_t* xq = at<uint8_t>(ws, L.xq);
  uint8_t* xq_s = at<uint8_t>(ws, L.xq_scales);
  uint8_t* hq = at<uint8_t>(ws, L.h);
  uint8_t* hs = at<uint8_t>(ws, L.h_scales);
  const uint64_t RI = (uint64_t)(E + 1) * I, RD = (uint64_t)(E + 1) * D;
  // up projections + SwiGLU: A = w1 / w3 codes [(E+1) I, d], B = E4M3 rows of x_perm (routed) or x
  {
    moe::MxMaps m;
    if (!make_map_e2m1(&m.a0, fp4->w1, RI, D) || !make_map_e2m1(&m.a1, fp4->w3, RI, D)) return MOE_ERR_CUDA;
    m.sa0 = fp4->w1_scale;
    m.sa1 = fp4->w3_scale;
    if (!make_map_u8(&m.b_routed, xp, S, D, 16, 128) || !make_map_u8(&m.bw_routed, xp, S, D, 64, 128)) return MOE_ERR_CUDA;
    if (!make_map_u8(&m.b_shared, xq, T, D, 16, 128) || !make_map_u8(&m.bw_shared, xq, T, D, 64, 128)) return MOE_ERR_CUDA;
    m.sb_routed = xp_s; m.sb_routed_rows = S;
    m.sb_shared = xq_s; m.sb_shared_rows = T;
    moe::GemmParams p{};
    p.chunk_prefix = prefix; p.offsets = offsets; p.E = E; p.T = T; p.S = S;
    p.K = D; p.M_total = I; p.bn = bn; p.m_rows = cta_per_tile * moe::kGemmBM; p.m_tiles = I / p.m_rows;
    p.solo = solo ? 1 : 0;
    p.swiglu_limit = d.swiglu_limit; p.row_weight = row_weights; p.test_stall = test_stall_flag();
    p.shared_b_row = 0;
    p.q_routed = hq; p.q_shared = hq + (size_t)S * I; p.s_routed = hs; p.s_shared = hs + (size_t)S * (I / 32);
    p.ew = ew;
    const long units = chunk_bound * p.m_tiles, most = sms / cta_per_tile;
    const int ctas = cta_per_tile * (int)(units < most ? units : most);
    MOE_TRY(cuda_status(moe::launch_expert_gemm_mx(moe::kGemmSwiGLU, m, p, ctas, stream)));
  }
  // down projection: A = w2 codes [(E+1) d, I], B = E4M3 rows of h [S + T, I] (shared rows from S)
  {
    moe::MxMaps m;
    if (!make_map_e2m1(&m.a0, fp4->w2, RD, I)) return MOE_ERR_CUDA;
    m.a1 = m.a0;
    m.sa0 = m.sa1 = fp4->w2_scale;
    if (!make_map_u8(&m.b_routed, hq, (uint64_t)S + T, I, 16, 128) ||
        !make_map_u8(&m.bw_routed, hq, (uint64_t)S + T, I, 64, 128))
      return MOE_ERR_CUDA;
    m.b_shared = m.b_routed; m.bw_shared = m.bw_routed;
    m.sb_routed = m.sb_shared = hs;
    m.sb_routed_rows = m.sb_shared_rows = S + T;
    moe::GemmParams p{};
    p.chunk_prefix = prefix; p.offsets = offsets; p.E = E; p.T = T; p.S = S;
    p.K = I; p.M_total = D; p.bn = bn; p.m_rows = 2 * cta_per_tile * moe::kGemmBM; p.m_tiles = D / p.m_rows;
    p.solo = solo ? 1 : 0;
    p.shared_b_row = S; p.test_stall = test_stall_flag();
    p.out_routed = reinterpret_cast<__nv_bfloat16*>(out_perm);
    p.out_shared = reinterpret_cast<__nv_bfloat16*>(out_shared);
    p.ew = ew;
    const long units = chunk_bound * p.m_tiles, most = sms / cta_per_tile;
    const int ctas = cta_per_tile * (int)(units < most ? units : most);
    MOE_TRY(cuda_status(moe::launch_expert_gemm_mx(moe::kGemmPair, m, p, ctas, stream)));
  }
  return MOE_OK;
}

// E4M3 codes and scales of bf16 rows [R, d] into the workspace at (codes, scales).
moe_status quantize_rows(const moe_layer_desc& d, const moe_bf16* x, long R, void* ws, size_t codes, size_t scales,
                         cudaStream_t stream) {
  return cuda_status(moe::launch_quantize_rows(reinterpret_cast<const __nv_bfloat16*>(x), R, d.dim, at<uint8_t>(ws, codes),
                                               at<uint8_t>(ws, scales), num_sms(), stream));
}


moe_status run_combine(const moe_layer_desc& d, int T, const moe_bf16* out_perm, const int32_t* row_of_slot,
                       const float* weights, const moe_bf16* out_shared, moe_bf16* y, cudaStream_t stream) {
  return cuda_status(moe::launch_combine(reinterpret_cast<const __nv_bfloat16*>(out_perm), row_of_slot, weights,
                                         reinterpret_cast<const __nv_bfloat16*>(out_shared),
                                         reinterpret_cast<__nv_bfloat16*>(y), T, d.topk, d.dim, T * d.topk, num_sms(),
                                         stream));
}

// MXFP4 weights run on the CTA-pair kernels only, with K % 512 == 0 for both GEMMs (rows of block scales
// a multiple of 16 bytes, the TMA stride rule): I % 512 == 0 and d % 512 == 0; every pointer 16-byte
// aligned (the TMA base-address rule).
bool mx_activations(const moe_layer_desc& d, const moe_mxfp4_weights* fp4) {
  return fp4 != nullptr && (d.options & MOE_OPT_MXFP4_BF16_ACTIVATIONS) == 0;
}

// token_chunk: 96 or 224 for the block-scaled kernels (E4M3 activations), 128 or 256 for the others.
bool token_chunk_fits(const moe_layer_desc& d, const moe_mxfp4_weights* fp4) {
  if (d.token_chunk == 0) return true;
  const bool mx = mx_activations(d, fp4);
  return mx ? (d.token_chunk == moe::kMxTwoBufChunk || d.token_chunk == moe::kMxMaxChunk)
            : (d.token_chunk == 128 || d.token_chunk == 256);
}

moe_status check_mxfp4(const moe_layer_desc& d, int T, const moe_mxfp4_weights* w) {
  if (d.inter_dim % 512 != 0 || d.dim % 512 != 0) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  const void* ptrs[6] = {w->w1, w->w1_scale, w->w3, w->w3_scale, w->w2, w->w2_scale};
  for (const void* q : ptrs)
    if (q == nullptr || !aligned16(q)) return MOE_ERR_INVALID;
  // the block-scaled path reads the codes through 16U4_ALIGN16B tensor maps: 32-byte aligned bases
  if (mx_activations(d, w) && ((reinterpret_cast<uintptr_t>(w->w1) | reinterpret_cast<uintptr_t>(w->w3) |
                                reinterpret_cast<uintptr_t>(w->w2)) & 31u) != 0)
    return MOE_ERR_INVALID;
  return MOE_OK;
}

// Trial division; the 2-gram hash's primes lie below 2^32, so at most 65536 divisions each.
bool is_prime(int64_t q) {
  if (q < 2) return false;
  for (int64_t f = 2; f * f <= q; ++f)
    if (q % f == 0) return false;
  return true;
}

// The checks shared by the expert-FFN entry points: routed rows from x_perm (tok_of_row null) or
// gathered from x by tok_of_row (x_perm null); bf16 weights w1 / w3 / w2 or MXFP4 weights fp4.
moe_status expert_ffn_entry(const moe_layer_desc* desc, int T, const moe_bf16* x_perm, const int32_t* tok_of_row,
                            const int32_t* offsets, const float* row_weights, const moe_bf16* x, const moe_bf16* w1,
                            const moe_bf16* w3, const moe_bf16* w2, const moe_mxfp4_weights* fp4, moe_bf16* out_perm,
                            moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_desc(desc));
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (!token_chunk_fits(*desc, fp4)) return MOE_ERR_UNSUPPORTED;
  if (fp4 != nullptr) MOE_TRY(check_mxfp4(*desc, T, fp4));
  if (tok_of_row != nullptr && !gather_supported(*desc, fp4 != nullptr)) return MOE_ERR_UNSUPPORTED;
  const void* rows = tok_of_row != nullptr ? static_cast<const void*>(tok_of_row) : x_perm;
  if (T > 0 && (rows == nullptr || offsets == nullptr || x == nullptr || out_perm == nullptr || out_shared == nullptr))
    return MOE_ERR_INVALID;
  if (T > 0 && fp4 == nullptr && (w1 == nullptr || w3 == nullptr || w2 == nullptr)) return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x_perm) || !aligned16(x) || !aligned16(out_perm) || !aligned16(out_shared)))
    return MOE_ERR_INVALID;
  if (T > 0 && fp4 == nullptr && (!aligned16(w1) || !aligned16(w3) || !aligned16(w2))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (mx_activations(*desc, fp4)) {
    // E4M3 activations: x quantised once, the routed rows quantised from x_perm or gathered (already
    // quantised) from x through tok_of_row
    const WsLayout L = ws_layout(*desc, T);
    const int S = T * desc->topk;
    MOE_TRY(quantize_rows(*desc, x, T, ws, L.xq, L.xq_scales, s));
    if (tok_of_row != nullptr) {
      MOE_TRY(cuda_status(moe::launch_gather_rows(row_copy_mx(*desc, T, ws), tok_of_row, S, T, num_sms(), s)));
    } else {
      MOE_TRY(quantize_rows(*desc, x_perm, S, ws, L.x_perm, L.xp_scales, s));
    }
    return run_experts_mx(*desc, T, offsets, row_weights, fp4, out_perm, out_shared, ws, s);
  }
  return run_experts(*desc, T, x_perm, offsets, row_weights, x, w1, w3, w2, out_perm, out_shared, ws, s, fp4,
                     tok_of_row);
}

moe_status forward_impl(const moe_layer_desc* desc, int T, const moe_bf16* x, const int32_t* token_ids,
                        const int32_t* tid2eid, int vocab, const float* w_gate, const float* bias,
                        const float* logit_offset, const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                        const moe_mxfp4_weights* fp4, moe_bf16* y, float* weights_out, int32_t* indices_out,
                        int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_desc(desc));
  const bool hashed = token_ids != nullptr || tid2eid != nullptr;
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (hashed && (token_ids == nullptr || tid2eid == nullptr || vocab <= 0)) return MOE_ERR_INVALID;
  if (hashed && desc->score_func == MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if (!token_chunk_fits(*desc, fp4)) return MOE_ERR_UNSUPPORTED;
  if (fp4 != nullptr) MOE_TRY(check_mxfp4(*desc, T, fp4));
  if (T > 0 && (x == nullptr || w_gate == nullptr || y == nullptr)) return MOE_ERR_INVALID;
  if (T > 0 && fp4 == nullptr && (w1 == nullptr || w3 == nullptr || w2 == nullptr)) return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x) || !aligned16(w_gate) || !aligned16(y))) return MOE_ERR_INVALID;
  if (T > 0 && fp4 == nullptr && (!aligned16(w1) || !aligned16(w3) || !aligned16(w2))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (counts_out != nullptr) return cuda_status(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * desc->n_experts, s));
    return MOE_OK;
  }
  const moe_layer_desc& d = *desc;
  const WsLayout L = ws_layout(d, T);
  float* weights = weights_out ? weights_out : at<float>(ws, L.weights);
  int32_t* indices = indices_out ? indices_out : at<int32_t>(ws, L.indices);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_of_slot = at<int32_t>(ws, L.row_of_slot);
  int32_t* tok_of_row = at<int32_t>(ws, L.tok_of_row);
  moe_bf16* x_perm = at<moe_bf16>(ws, L.x_perm);
  moe_bf16* out_perm = at<moe_bf16>(ws, L.out_perm);
  moe_bf16* out_shared = at<moe_bf16>(ws, L.out_shared);
  // the cluster router also counts dispatch's histogram (fh.coarse > 0 after the gate): then dispatch
  // is the scatter alone
  FusedHist fh;
  fh.hist = at<int32_t>(ws, L.hist); fh.base = at<int32_t>(ws, L.base); fh.counts = counts; fh.offsets = offsets;
  fh.ticket = &at<ErrorWord>(ws, L.err)->dispatch_ticket;
  {
    NvtxRange r("gate");
    if (hashed)
      MOE_TRY(run_hash_gate(d, T, token_ids, tid2eid, vocab, x, w_gate, weights, indices, ws, s, nullptr, nullptr, &fh));
    else
      MOE_TRY(run_gate(d, T, x, w_gate, bias, logit_offset, weights, indices, ws, s, nullptr, &fh));
  }
  float* w_perm = d.weight_in_expert ? at<float>(ws, L.w_perm) : nullptr;
  const int S = T * d.topk;
  ErrorWord* ew = at<ErrorWord>(ws, L.err);
  auto dispatch = [&](const moe::RowCopy& rc) -> moe_status {
    if (fh.coarse > 0)
      return cuda_status(moe::launch_dispatch_scatter(indices, S, d.topk, d.n_experts, rc, fh.coarse, fh.base, offsets,
                                                      row_of_slot, tok_of_row, ew, s, w_perm ? weights : nullptr,
                                                      w_perm));
    return run_dispatch_rows(d, T, indices, rc, counts, offsets, row_of_slot, tok_of_row, ws, s,
                             w_perm ? weights : nullptr, w_perm);
  };
  if (mx_activations(d, fp4)) {
    // E4M3 activations: x quantised once; dispatch copies the quantised rows (codes and scales)
    {
      NvtxRange r("dispatch");
      MOE_TRY(quantize_rows(d, x, T, ws, L.xq, L.xq_scales, s));
      MOE_TRY(dispatch(row_copy_mx(d, T, ws)));
    }
    {
      NvtxRange r("experts");
      MOE_TRY(run_experts_mx(d, T, offsets, w_perm, fp4, out_perm, out_shared, ws, s));
    }
    NvtxRange r("combine");
    return run_combine(d, T, out_perm, row_of_slot, w_perm ? nullptr : weights, out_shared, y, s);
  }
  const bool fuse = fused_gather(d, fp4 != nullptr);
  {
    NvtxRange r("dispatch");
    MOE_TRY(dispatch(moe::row_copy_bf16(reinterpret_cast<const __nv_bfloat16*>(x), d.dim,
                                        reinterpret_cast<__nv_bfloat16*>(fuse ? nullptr : x_perm))));
  }
  {
    NvtxRange r("experts");
    MOE_TRY(run_experts(d, T, fuse ? nullptr : x_perm, offsets, w_perm, x, w1, w3, w2, out_perm, out_shared, ws, s,
                        fp4, fuse ? tok_of_row : nullptr));
  }
  NvtxRange r("combine");
  return run_combine(d, T, out_perm, row_of_slot, w_perm ? nullptr : weights, out_shared, y, s);
}

}  // namespace

// =============================================================================================
// exported entry points
// =============================================================================================
extern "C" {

size_t moe_workspace_bytes(const moe_layer_desc* desc, int T) {
  if (check_desc(desc) != MOE_OK || T < 0) return 0;
  return ws_layout(*desc, T).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < sizeof(ErrorWord)) return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(ErrorWord), reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_gate_prepared_bytes(const moe_layer_desc* desc) {
  if (check_desc(desc) != MOE_OK) return 0;
  return kPreparedHeader + align_up(3 * (size_t)desc->n_experts * desc->dim * 2);
}

moe_status moe_gate_prepare(const moe_layer_desc* desc, const float* w_gate, void* prepared, moe_stream_t stream) {
  NvtxRange nvtx("moe_gate_prepare");
  MOE_TRY(check_desc(desc));
  if (w_gate == nullptr || prepared == nullptr || !aligned16(w_gate) || !aligned16(prepared)) return MOE_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* flag = static_cast<int*>(prepared);
  auto* planes = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(prepared) + kPreparedHeader);
  MOE_TRY(cuda_status(cudaMemsetAsync(flag, 0, sizeof(int), s)));
  return cuda_status(moe::launch_gate_planes(w_gate, planes, (long)desc->n_experts * desc->dim, flag, num_sms(), s));
}

moe_status moe_gate(const moe_layer_desc* desc, int T, const moe_bf16* x, const float* w_gate, const float* bias,
                    const float* logit_offset, float* weights, int32_t* indices, void* ws, size_t ws_bytes,
                    moe_stream_t stream) {
  NvtxRange nvtx("moe_gate");
  MOE_TRY(check_desc(desc));
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (T > 0 && (x == nullptr || w_gate == nullptr || weights == nullptr || indices == nullptr)) return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x) || !aligned16(w_gate))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  return run_gate(*desc, T, x, w_gate, bias, logit_offset, weights, indices, ws,
                  reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_hash_gate(const moe_layer_desc* desc, int T, const int32_t* token_ids, const int32_t* tid2eid,
                         int vocab, const moe_bf16* x, const float* w_gate, float* weights, int32_t* indices, void* ws,
                         size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_hash_gate");
  MOE_TRY(check_desc(desc));
  if (T < 0 || vocab <= 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (desc->score_func == MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (token_ids == nullptr || tid2eid == nullptr || x == nullptr || w_gate == nullptr ||
                weights == nullptr || indices == nullptr))
    return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x) || !aligned16(w_gate))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  return run_hash_gate(*desc, T, token_ids, tid2eid, vocab, x, w_gate, weights, indices, ws,
                       reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_ngram_gate(const moe_layer_desc* desc, int T, const int32_t* prev_ids, const int32_t* token_ids,
                          const int64_t* primes, int vocab, const moe_bf16* x, const float* w_gate, float* weights,
                          int32_t* indices, void* ws, size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_ngram_gate");
  MOE_TRY(check_desc(desc));
  if (T < 0 || vocab <= 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (desc->score_func == MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if (primes == nullptr) return MOE_ERR_INVALID;
  for (int j = 0; j < desc->topk; ++j) {
    if (primes[j] <= vocab || primes[j] >= (int64_t(1) << 32) || !is_prime(primes[j])) return MOE_ERR_INVALID;
    for (int i = 0; i < j; ++i)
      if (primes[i] == primes[j]) return MOE_ERR_INVALID;
  }
  if (T > 0 && (prev_ids == nullptr || token_ids == nullptr || x == nullptr || w_gate == nullptr ||
                weights == nullptr || indices == nullptr))
    return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x) || !aligned16(w_gate))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  if (T == 0) return MOE_OK;
  return run_hash_gate(*desc, T, token_ids, nullptr, vocab, x, w_gate, weights, indices, ws,
                       reinterpret_cast<cudaStream_t>(stream), prev_ids, primes);
}

moe_status moe_update_bias(const moe_layer_desc* desc, int T, const int32_t* counts, float* bias, float gamma,
                           moe_stream_t stream) {
  NvtxRange nvtx("moe_update_bias");
  MOE_TRY(check_desc(desc));
  if (T < 0 || !std::isfinite(gamma) || gamma < 0.f) return MOE_ERR_INVALID;
  if (counts == nullptr || bias == nullptr) return MOE_ERR_INVALID;
  const long long balanced_times_E = (long long)T * desc->topk;
  return cuda_status(moe::launch_update_bias(counts, bias, desc->n_experts, balanced_times_E, gamma,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const moe_layer_desc* desc, int T, const int32_t* indices, const moe_bf16* x, int32_t* counts,
                        int32_t* offsets, int32_t* row_of_slot, int32_t* tok_of_row, moe_bf16* x_perm, void* ws,
                        size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_dispatch");
  MOE_TRY(check_desc(desc));
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID;
  if (T > 0 && (indices == nullptr || x == nullptr || row_of_slot == nullptr || tok_of_row == nullptr))
    return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID;
  MOE_TRY(check_ws(*desc, T, ws, ws_bytes));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    MOE_TRY(cuda_status(cudaMemsetAsync(counts, 0, sizeof(int32_t) * desc->n_experts, s)));
    return cuda_status(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (desc->n_experts + 1), s));
  }
  return run_dispatch(*desc, T, indices, x, counts, offsets, row_of_slot, tok_of_row, x_perm, ws, s);
}

moe_status moe_expert_ffn(const moe_layer_desc* desc, int T, const moe_bf16* x_perm, const int32_t* offsets,
                          const float* row_weights, const moe_bf16* x, const moe_bf16* w1, const moe_bf16* w3,
                          const moe_bf16* w2, moe_bf16* out_perm, moe_bf16* out_shared, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  NvtxRange nvtx("moe_expert_ffn");
  return expert_ffn_entry(desc, T, x_perm, nullptr, offsets, row_weights, x, w1, w3, w2, nullptr, out_perm, out_shared,
                          ws, ws_bytes, stream);
}

moe_status moe_expert_ffn_gather(const moe_layer_desc* desc, int T, const int32_t* tok_of_row, const int32_t* offsets,
                                 const float* row_weights, const moe_bf16* x, const moe_bf16* w1, const moe_bf16* w3,
                                 const moe_bf16* w2, moe_bf16* out_perm, moe_bf16* out_shared, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_expert_ffn_gather");
  return expert_ffn_entry(desc, T, nullptr, tok_of_row, offsets, row_weights, x, w1, w3, w2, nullptr, out_perm,
                          out_shared, ws, ws_bytes, stream);
}

moe_status moe_combine(const moe_layer_desc* desc, int T, const moe_bf16* out_perm, const int32_t* row_of_slot,
                       const float* weights, const moe_bf16* out_shared, moe_bf16* y, moe_stream_t stream) {
  NvtxRange nvtx("moe_combine");
  MOE_TRY(check_desc(desc));
  if (T < 0 || (long)T * desc->topk > INT32_MAX / 2) return MOE_ERR_INVALID;
  if (T > 0 && (out_perm == nullptr || row_of_slot == nullptr || y == nullptr)) return MOE_ERR_INVALID;
  if (T > 0 && (!aligned16(out_perm) || !aligned16(y) || (out_shared != nullptr && !aligned16(out_shared))))
    return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  return run_combine(*desc, T, out_perm, row_of_slot, weights, out_shared, y, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_forward(const moe_layer_desc* desc, int T, const moe_bf16* x, const int32_t* token_ids,
                       const int32_t* tid2eid, int vocab, const float* w_gate, const float* bias,
                       const float* logit_offset, const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                       moe_bf16* y, float* weights_out, int32_t* indices_out, int32_t* counts_out, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_forward");
  return forward_impl(desc, T, x, token_ids, tid2eid, vocab, w_gate, bias, logit_offset, w1, w3, w2, nullptr, y,
                      weights_out, indices_out, counts_out, ws, ws_bytes, stream);
}

moe_status moe_forward_mxfp4(const moe_layer_desc* desc, int T, const moe_bf16* x, const int32_t* token_ids,
                             const int32_t* tid2eid, int vocab, const float* w_gate, const float* bias,
                             const float* logit_offset, const moe_mxfp4_weights* weights_mxfp4, moe_bf16* y,
                             float* weights_out, int32_t* indices_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  NvtxRange nvtx("moe_forward_mxfp4");
  if (weights_mxfp4 == nullptr) return MOE_ERR_INVALID;
  return forward_impl(desc, T, x, token_ids, tid2eid, vocab, w_gate, bias, logit_offset, nullptr, nullptr, nullptr,
                      weights_mxfp4, y, weights_out, indices_out, counts_out, ws, ws_bytes, stream);
}

moe_status moe_expert_ffn_mxfp4(const moe_layer_desc* desc, int T, const moe_bf16* x_perm, const int32_t* offsets,
                                const float* row_weights, const moe_bf16* x, const moe_mxfp4_weights* weights_mxfp4,
                                moe_bf16* out_perm, moe_bf16* out_shared, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  NvtxRange nvtx("moe_expert_ffn_mxfp4");
  if (weights_mxfp4 == nullptr) return MOE_ERR_INVALID;
  return expert_ffn_entry(desc, T, x_perm, nullptr, offsets, row_weights, x, nullptr, nullptr, nullptr, weights_mxfp4,
                          out_perm, out_shared, ws, ws_bytes, stream);
}

moe_status moe_expert_ffn_mxfp4_gather(const moe_layer_desc* desc, int T, const int32_t* tok_of_row,
                                       const int32_t* offsets, const float* row_weights, const moe_bf16* x,
                                       const moe_mxfp4_weights* weights_mxfp4, moe_bf16* out_perm,
                                       moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream) {
  NvtxRange nvtx("moe_expert_ffn_mxfp4_gather");
  if (weights_mxfp4 == nullptr) return MOE_ERR_INVALID;
  return expert_ffn_entry(desc, T, nullptr, tok_of_row, offsets, row_weights, x, nullptr, nullptr, nullptr,
                          weights_mxfp4, out_perm, out_shared, ws, ws_bytes, stream);
}

moe_status moe_get_error(void* ws, moe_stream_t stream, int32_t* info) {
  if (ws == nullptr) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int host[2] = {0, 0};
  if (cudaMemcpy(host, ws, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (info != nullptr) *info = host[1];
  if (host[0] != 0) {
    if (cudaMemset(ws, 0, sizeof(host)) != cudaSuccess) return MOE_ERR_CUDA;
    return static_cast<moe_status>(host[0]);
  }
  return MOE_OK;
}

#ifdef MOE_TEST_HOOKS
// Test build only (not declared in include/moe.h): 1 makes the CTA-pair expert GEMMs stall, 0 restores them.
void moe_test_set_stall(int on) { g_test_stall = on; }
#endif

const char* moe_status_str(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID: return "MOE_ERR_INVALID: bad argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape not implemented";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call or launch failed";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: out-of-range token id or expert index (clamped)";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a kernel wait ran out of time";
    case MOE_ERR_IO: return "MOE_ERR_IO: a file could not be opened, read or written";
  }
  return "unknown moe_status";
}

}  // extern "C"
