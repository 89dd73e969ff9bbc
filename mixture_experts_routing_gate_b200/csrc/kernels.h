// Parameter blocks and declarations of the libmoe kernels (host and device side).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moe.h"

namespace moe {

// Programmatic dependent launch: every kernel of the library may be launched while its predecessor
// on the stream drains (each kernel begins with pdl_begin(), which waits for that predecessor to
// complete before any global memory is touched).  MOE_PDL=0 in the environment turns it off; the
// variable is read once, at the library's first launch, never per call.
bool pdl_enabled();

// The layer-descriptor checks shared by every entry point (moe_api.cu).
moe_status check_layer_desc(const moe_layer_desc* d);

// An NVTX range over one entry point or stage (no cost without an attached profiler), so that a
// timeline tool shows the layer's stages by name.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Fills attr[0] with the programmatic-serialization attribute when it is enabled; returns the count.
inline unsigned pdl_attr(cudaLaunchAttribute* attr) {
  if (!pdl_enabled()) return 0;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  return 1;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = pdl_attr(attr);
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct ErrorWord;

constexpr int kMaxRouteTopk = 8;

struct RouterParams {
  int T, d, E, G, g, k;
  int score_func, renorm;
  float route_scale;
  int n_half;      // experts per MMA (E, or E/2 when E > 256)
  int n_split;     // 1 or 2 MMAs per K step
  int stages;      // pipeline depth
  int tmem_cols;   // power of two >= E
  int nsplit;      // expert column ranges per token in the epilogue (1, 2 or 4)
  int region_bytes;  // shared memory for the pipeline stages, reused by the epilogue
  int ksplit;        // cluster router: CTAs per 128-token tile (split of the K loop), 1, 2, 4 or 8
  int e_pad;         // cluster router: row pitch (floats) of the partial-logit exchange buffer
  int sel_mode;      // cluster router: 0 group-limited top-k; 1 token-id table; 2 2-gram hash
  int vocab;         //   hash modes: token ids lie in [0, vocab)
  const int32_t* token_ids;  // [T] (hash modes)
  const int32_t* prev_ids;   // [T] (2-gram hash)
  const int32_t* tid2eid;    // [vocab, k] (table mode)
  unsigned long long primes[kMaxRouteTopk];  // 2-gram hash: expert j = (prev * primes[j] + id) mod E
  const float* bias;          // [E] or null
  const float* logit_offset;  // [E] or null
  const int* plane_flag;      // device: non-zero when the router weight needs three bf16 planes
  float* weights;             // [T, k]
  int32_t* indices;           // [T, k]
  ErrorWord* ew;
  // cluster router, when non-null: dispatch's histogram fused into the epilogue -- each CTA writes
  // the expert histogram of its owned tokens' slots as row blockIdx.x of hist (its tokens are
  // [blockIdx.x * 128 / ksplit, ...): blocks of (128 / ksplit) * k slots), and the CTA that takes the
  // last ticket turns the rows into base, counts and offsets (dispatch_scan.cuh)
  int32_t* hist;              // [gridDim, E]
  int32_t* base;              // [gridDim, E]
  int32_t* counts;            // [E]
  int32_t* offsets;           // [E + 1]
  int* ticket;                // zero between calls
};

struct HashGateParams {
  int T, d, E, k, vocab, score_func, renorm;
  float route_scale;
  const int32_t* token_ids;
  const int32_t* tid2eid;   // [vocab, k]; null for the 2-gram hash
  const int32_t* prev_ids;  // [T] previous token of each position (2-gram hash) or null
  unsigned long long primes[kMaxRouteTopk];  // 2-gram hash: expert j = (prev * primes[j] + id) mod E
  const __nv_bfloat16* x;
  const float* w_gate;
  float* weights;
  int32_t* indices;
  ErrorWord* ew;
};

struct GemmParams {
  const int* chunk_prefix;  // [E+2]: token chunks of groups 0..E (E = shared expert), prefix summed
  const int* offsets;       // [E+1]: first row of each routed expert
  int E, T, S;              // routed experts, tokens, routed rows (T*k)
  int K;                    // reduction length (d for the up projections, I for the down projection)
  int m_tiles;              // weight-row tiles per expert (each m_rows rows)
  int m_rows;               // weight rows per tile: 128 (SwiGLU, single) or 256 (pair)
  int M_total;              // output features per row (I or d)
  int stages;
  int bn;                   // token rows per chunk (128, or 256 for the CTA-pair kernels)
  int shared_b_row;         // first B row of the shared expert in its tensor map
  float swiglu_limit;       // > 0: clamp of the SwiGLU branches
  const float* row_weight;  // [S] or null: weight of each routed row, applied to h
  int b_wide;               // CTA-pair kernels: > 0 = rows per box of the wide B maps, which come with
                            // double-wide ones (whole boxes of a tile's token rows come from them,
                            // the rest from the 16-row maps); 0 = none
  const int* gather_rows;   // [S] or null (up projections of the CTA-pair kernel): token of each routed
                            // row; the routed B rows are then gathered from x (B map: x, one-row box)
  int solo;                 // block-scaled kernels: 1 = one CTA per tile (M = 128), 0 = CTA pairs
  int test_stall;           // failure-detection test hook (set only by the test build of the library):
                            // the producer issues no loads, so every consumer's bounded wait runs out
                            // and reports MOE_ERR_TIMEOUT
  __nv_bfloat16* out_routed;  // [S, M_total]
  __nv_bfloat16* out_shared;  // [T, M_total]
  uint8_t* q_routed;          // block-scaled up projection: E4M3 codes of h, routed rows [S, M_total]
  uint8_t* q_shared;          //   and shared-expert rows [T, M_total]
  uint8_t* s_routed;          //   UE8M0 scales of h per 32 features, [S, M_total / 32]
  uint8_t* s_shared;          //   and [T, M_total / 32]
  ErrorWord* ew;
};

constexpr int kGemmBN = 128;   // token tile (the MMA's N); a tile holds 1..128 rows of one expert
constexpr int kGemmBM = 128;   // weight rows per tile (the MMA's M)
constexpr int kGemmThreads = 192;
constexpr int kGemmSingle = 0;  // one 128-row weight tile per token chunk
constexpr int kGemmSwiGLU = 1;  // w1 and w3 tiles of the same rows, SwiGLU epilogue
constexpr int kGemmPair = 2;    // two adjacent 128-row weight tiles

// Host-side launchers, one per kernel; each returns the launch's cudaError_t.
cudaError_t launch_gate_planes(const float* w, __nv_bfloat16* planes, long n, int* inexact_flag, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_router(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                          cudaStream_t stream);
size_t router_smem_bytes(const RouterParams& p);
// The split-K cluster router: E = 16 * per_lane with per_lane in {1, 2, 4, 8, 16, 24}, 16 % G == 0.
bool router_cluster_supported(int E, int G);
size_t router_cluster_smem_bytes(const RouterParams& p);
cudaError_t launch_router_cluster(const CUtensorMap& map_x, const CUtensorMap& map_w, const RouterParams& p,
                                  cudaStream_t stream);
size_t router_epilogue_bytes(int nsplit, int G, int k);
cudaError_t launch_hash_gate(const HashGateParams& p, cudaStream_t stream);

// bias[e] -= gamma when counts[e] * E > T * k, += gamma when below, in place.
cudaError_t launch_update_bias(const int32_t* counts, float* bias, int E, long long balanced_times_E, float gamma,
                               cudaStream_t stream);

// How dispatch cuts S = T * k slots: n_coarse histogram blocks of `coarse` slots, and n_fine
// scatter blocks of fine_tokens tokens.  Its scratch: hist and base, n_coarse * E ints each.
struct DispatchPlan {
  int coarse, n_coarse, fine_tokens, n_fine;
};
DispatchPlan dispatch_plan(long S, int k, int num_sms);

// What the scatter copies per token: nseg segments (0: the permutation only), segment g being a row
// of bytes[g] bytes (a multiple of 16) of src[g] (row index = token) stored to rows of dst[g] (row
// index = the slot's permuted row); e.g. the bf16 row of x into x_perm, or the E4M3 codes and the
// scales of the quantised row.
struct RowCopy {
  int nseg;
  int bytes[2];
  const uint8_t* src[2];
  uint8_t* dst[2];
};
// The scatter alone, on per-block bases of `coarse` slots each computed before (by the histogram
// kernel, or by the cluster router's fused histogram).
cudaError_t launch_dispatch_scatter(const int32_t* indices, int S, int k, int E, const RowCopy& rc, int coarse,
                                    const int32_t* base, const int32_t* offsets, int32_t* row_of_slot,
                                    int32_t* tok_of_row, ErrorWord* ew, cudaStream_t stream, const float* weights,
                                    float* w_perm);


// weights [S] / w_perm [S] (both or neither): w_perm[row_of_slot[s]] = weights[s].  *ticket must be 0
// before the first call (every call leaves it 0).
cudaError_t launch_dispatch(const int32_t* indices, int S, int k, int E, const RowCopy& rc, int32_t* hist,
                            int32_t* base, int* ticket, int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                            int32_t* tok_of_row, ErrorWord* ew, cudaStream_t stream, const float* weights = nullptr,
                            float* w_perm = nullptr);
// rc.dst[g] row r = rc.src[g] row tok_of_row[r] for r < S (tokens clamped into [0, T)).
cudaError_t launch_gather_rows(const RowCopy& rc, const int32_t* tok_of_row, int S, int T, int num_sms,
                               cudaStream_t stream);

// RowCopy of bf16 rows of x [T, d] into x_perm (or none when x_perm is null).
inline RowCopy row_copy_bf16(const __nv_bfloat16* x, int d, __nv_bfloat16* x_perm) {
  RowCopy rc{};
  if (x_perm == nullptr) return rc;
  rc.nseg = 1;
  rc.bytes[0] = d * 2;
  rc.src[0] = reinterpret_cast<const uint8_t*>(x);
  rc.dst[0] = reinterpret_cast<uint8_t*>(x_perm);
  return rc;
}

cudaError_t launch_expert_tiles(const int32_t* offsets, int E, int T, int S, int bn, int32_t* chunk_prefix,
                                ErrorWord* ew, cudaStream_t stream);
// mode: kGemmSwiGLU for the up projections, kGemmPair / kGemmSingle for the down projection.
cudaError_t launch_expert_gemm(int mode, const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                               const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared, const GemmParams& p,
                               int grid, cudaStream_t stream);
size_t expert_gemm_smem_bytes(int mode, int E, int stages);
// The CTA-pair variant of kGemmSwiGLU (I % 256 == 0), kGemmPair (d % 512 == 0) and kGemmSingle
// (d % 256 == 0); p.m_rows is the pair tile's weight rows (256 or 512) and p.m_tiles = M_total / p.m_rows.
// MXFP4 weights (kGemmSwiGLU and kGemmPair, K % 512 == 0): map_a0 / map_a1 cover the packed E2M1 codes
// ([rows, K/2] bytes, boxes of 128 rows x 32 bytes) and map_s0 / map_s1 (non-null) their block scales
// ([rows, K/32] bytes, boxes of 128 rows x 16 bytes).
cudaError_t launch_expert_gemm_pair(int mode, const CUtensorMap& map_a0, const CUtensorMap& map_a1,
                                    const CUtensorMap& map_b_routed, const CUtensorMap& map_b_shared,
                                    const GemmParams& p, int max_clusters, cudaStream_t stream,
                                    const CUtensorMap* map_s0 = nullptr, const CUtensorMap* map_s1 = nullptr,
                                    const CUtensorMap* map_bw_routed = nullptr,
                                    const CUtensorMap* map_bw_shared = nullptr,
                                    const CUtensorMap* map_bx_routed = nullptr,
                                    const CUtensorMap* map_bx_shared = nullptr);
size_t expert_gemm_pair_smem_bytes(int mode, int E, int bn, bool fp4 = false);
int expert_gemm_stages(int mode);

// Tensor maps of the block-scaled (MXFP4 weights x E4M3 activations) CTA-pair GEMMs.
struct MxMaps {
  CUtensorMap a0, a1;              // E2M1 weights (16U4_ALIGN16B: 16 codes per 16-byte slot in shared memory),
                                   // boxes of 128 rows x 128 elements, 128-byte swizzle
  CUtensorMap b_routed, b_shared;  // E4M3 token rows [rows, K], boxes of 16 rows x 128 bytes
  CUtensorMap bw_routed, bw_shared;  // the same in 64-row boxes
  // UE8M0 scales, row-major [rows, K/32] (16-byte aligned; read with plain loads by the scale warp)
  const uint8_t* sa0;              // of the a0 weight rows
  const uint8_t* sa1;              // of the a1 weight rows
  const uint8_t* sb_routed;        // of the routed token rows
  const uint8_t* sb_shared;        // of the shared expert's token rows
  int sb_routed_rows, sb_shared_rows;  // rows of those two (a tile's padding rows are clamped into them)
};
// mode kGemmSwiGLU (w1 / w3, h written as E4M3 codes + scales) or kGemmPair (two w2 tiles per CTA, bf16
// out); p.bn <= kMxMaxChunk, K % 512 == 0.
constexpr int kMxMaxChunk = 224;
constexpr int kMxTwoBufChunk = 96;   // chunks of at most this many rows get two accumulator buffers
constexpr int kMxSoloChunk = 64;     // the single-CTA form's chunk rows (decode-sized batches)
cudaError_t launch_expert_gemm_mx(int mode, const MxMaps& maps, const GemmParams& p, int max_ctas,
                                  cudaStream_t stream);
size_t expert_gemm_mx_smem_bytes(int E);
// E4M3 codes [R, d] and UE8M0 scales [R, d/32] of bf16 rows x [R, d] (blocks of 32 along a row; the
// least scale 2^e with 448 * 2^e >= the block's largest magnitude).
cudaError_t launch_quantize_rows(const __nv_bfloat16* x, long R, int d, uint8_t* codes, uint8_t* scales,
                                 int num_sms, cudaStream_t stream);

cudaError_t launch_combine(const __nv_bfloat16* out_perm, const int32_t* row_of_slot, const float* weights,
                           const __nv_bfloat16* out_shared, __nv_bfloat16* y, int T, int k, int d, int S, int num_sms,
                           cudaStream_t stream);

}  // namespace moe
