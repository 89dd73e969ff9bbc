/*
 * libmoe -- the forward pass of a DeepSeek-style mixture-of-experts layer on NVIDIA B200 (sm_100a).
 *
 * Plain C ABI: no C++ or framework types cross it.  Every device pointer is a pointer into the
 * current CUDA device's global memory; host pointers are marked "host".  The caller owns every
 * buffer; the library never allocates.  Scratch memory comes from a caller-provided workspace of
 * at least moe_workspace_bytes() bytes.  All device work is enqueued asynchronously on `stream`
 * (a cudaStream_t; NULL means the legacy default stream) and no call blocks the host except
 * moe_get_error().
 *
 * Layout: every matrix is row-major and contiguous.  bf16 tensors hold raw IEEE bfloat16 bit
 * patterns (moe_bf16).  Device pointers handed to the tensor-memory-accelerator paths (x, x_perm,
 * w1, w3, w2, out_perm, out_shared, y) must be 16-byte aligned; the library checks this.
 *
 * Errors: argument errors (bad sizes, NULL or misaligned pointers, unsupported shapes) return a
 * status before anything is launched.  A failed launch returns MOE_ERR_CUDA.  Bad data found by a
 * kernel (a token id outside the vocabulary, an expert index outside [0, E), an MXFP4 scale outside
 * [2, 252]) is clamped so that no access leaves its buffer, and is recorded in the workspace's
 * error word, which moe_get_error() reads.  Every wait inside a kernel is bounded (about two
 * seconds): one that runs out records MOE_ERR_TIMEOUT and the kernel returns.  No kernel traps.
 *
 * Notation: T tokens, d = dim, E routed experts, G expert groups, k experts per token,
 * I = inter_dim; the single shared expert is stored after the routed ones, as expert E.
 * "Slot" s = t*k + j is the j-th expert choice of token t.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;              /* raw bfloat16 bits */
typedef struct CUstream_st* moe_stream_t; /* the same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,      /* bad argument: NULL/misaligned pointer, negative or inconsistent size */
  MOE_ERR_UNSUPPORTED = 2,  /* valid layer, but a shape this build does not implement */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  MOE_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than moe_workspace_bytes() */
  MOE_ERR_DEVICE = 5,       /* a kernel saw an out-of-range token id or expert index (clamped) */
  MOE_ERR_TIMEOUT = 6,      /* a kernel's pipeline wait ran out of time and the kernel returned */
  MOE_ERR_IO = 7            /* a file could not be opened, read or written (host calls only) */
} moe_status;

typedef enum {
  MOE_SCORE_SIGMOID = 0,        /* s = 1 / (1 + exp(-l)) */
  MOE_SCORE_SQRT_SOFTPLUS = 1,  /* s = sqrt(log(1 + exp(l))) */
  MOE_SCORE_SOFTMAX = 2         /* s = softmax over the E experts (never renormalised) */
} moe_score_func;

/*
 * The layer's hyper-parameters ("DeepSeek-V3.2-Exp - Routing weights", gate-init excerpt:
 * dim, n_activated_experts, n_expert_groups, n_limited_groups, score_func, route_scale,
 * n_routed_experts; "DeepSeek V4.1 - Add shared", class MoE: moe_inter_dim, n_shared_experts == 1).
 */
typedef struct {
  int dim;               /* d: hidden size; multiple of 128 */
  int n_experts;         /* E routed experts; multiple of 16, at most 512 (multiple of 32 above 256) */
  int n_groups;          /* G >= 1 dividing E; with a bias, each group needs >= 2 experts */
  int n_limited_groups;  /* groups kept per token, 1 <= n_limited_groups <= G */
  int topk;              /* k experts per token, 1 <= k <= 8 and k <= n_limited_groups * E / G */
  int inter_dim;         /* I: intermediate size of every expert (routed and shared); multiple of 128 */
  int n_shared;          /* shared experts; must be 1 */
  moe_score_func score_func;
  float route_scale;     /* multiplies the gate weights */
  int renorm;            /* 1: divide the chosen experts' scores by their sum (sigmoid, sqrt-softplus) */
  float swiglu_limit;    /* > 0: cap the gate branch above at this and clamp the value branch to
                            [-limit, limit] in every expert ("From One Giant FFN to 384 Tiny Experts",
                            section 11.4); 0: no clamp */
  int weight_in_expert;  /* 1: moe_forward hands each routed row its gate weight inside the expert
                            (h is scaled before the down projection, "DeepSeek V4.1 - Add shared":
                            expert(x[idx], weights[...])) and the combine sums unweighted outputs;
                            0: the combine weights the expert outputs */
  int options;           /* bitwise OR of MOE_OPT_* below; 0 selects the default kernels.  The
                            options change which kernels run, not the values they compute (except
                            MOE_OPT_MXFP4_BF16_ACTIVATIONS, which keeps bf16 activations). */
  int token_chunk;       /* token rows per chunk of the CTA-pair expert GEMMs, or 0 to choose from
                            the shape.  bf16 tensor-core kernels: 128 or 256 (0: 256 when experts
                            average >= 16 rows, else 128).  Block-scaled MXFP4 kernels (E4M3
                            activations): 96 or 224 (0: 96 when T <= 96, else 224; chunks of 96
                            get two accumulator buffers).  Another value is MOE_ERR_INVALID, a
                            valid value of the other family MOE_ERR_UNSUPPORTED. */
  const void* gate_prepared;  /* NULL, or device memory written by moe_gate_prepare from this
                            layer's router weight: the tensor-core gates then read its bf16 planes
                            instead of splitting w_gate on every call (the caller re-prepares
                            whenever w_gate changes; w_gate is still passed, and still read by the
                            one-warp-per-token hash gate) */
} moe_layer_desc;

/* Kernel choices (moe_layer_desc.options).  Any other bit is MOE_ERR_INVALID. */
#define MOE_OPT_ROUTER_ONE_CTA 1  /* gates: one CTA per 128 tokens instead of the split-K cluster
                                     router; hash gates: one warp per token */
#define MOE_OPT_GEMM_ONE_CTA 2    /* experts: single-CTA GEMMs instead of CTA pairs (bf16 weights
                                     only; MXFP4 weights always run on CTA pairs) */
#define MOE_OPT_FUSED_GATHER 4    /* moe_forward: the up projection gathers the routed rows of x
                                     itself (as moe_expert_ffn_gather) and dispatch writes no x_perm
                                     (bf16 weights, and MXFP4 weights with bf16 activations) */
#define MOE_OPT_MXFP4_BF16_ACTIVATIONS 8  /* MXFP4 entry points: keep the activations in bf16 and decode
                                     the weights to bf16 on the SMs (the kind::f16 kernels) instead of
                                     the default E4M3 activations on the block-scaled tensor cores.
                                     Unlike the other options this one changes the values computed. */

/* Bytes of workspace needed by any entry point below for a batch of T tokens. */
size_t moe_workspace_bytes(const moe_layer_desc* desc, int T);

/* Clears the workspace's control words (the error word and dispatch's block counter, which every
 * call leaves at zero).  Call once after allocating a workspace, before any other call uses it
 * (asynchronous). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The router weight prepared once for the tensor-core gates: w_gate [E, d] fp32 split exactly into
 * three bf16 planes (hi + mid + lo = w, each the bf16 rounding of what the planes before it leave)
 * and a flag word saying whether any mid plane entry is non-zero (if none is, the gates run one
 * bf16 pass, else three).  prepared: device memory of moe_gate_prepared_bytes(desc) bytes, 16-byte
 * aligned, owned by the caller; point desc->gate_prepared at it for the calls that use it.
 * Asynchronous on `stream`.  MOE_ERR_INVALID for a NULL or misaligned pointer.
 */
size_t moe_gate_prepared_bytes(const moe_layer_desc* desc);
moe_status moe_gate_prepare(const moe_layer_desc* desc, const float* w_gate, void* prepared, moe_stream_t stream);

/*
 * Gate.forward ("DeepSeek-V3.2-Exp - Routing weights", gate-forward excerpt; affinity
 * sqrt(softplus) from "From One Giant FFN to 384 Tiny Experts", section 11.2):
 *   l = x . w_gate^T in fp32 (+ logit_offset[e] when given), s = affinity(l),
 *   b = s + bias (selection only), group-limited top-k on b, weights = s at the chosen experts,
 *   divided by their sum when desc->renorm, times route_scale.
 * x [T, d] bf16; w_gate [E, d] fp32; bias [E] fp32 or NULL; logit_offset [E] fp32 or NULL.
 * Outputs: weights [T, k] fp32; indices [T, k] int32, each row in descending selection score
 * (equal scores: lower expert index first).  Router weights holding bf16-exact values take one
 * bf16 tensor-core pass; general fp32 router weights are split exactly into three bf16 parts.
 */
moe_status moe_gate(const moe_layer_desc* desc, int T, const moe_bf16* x, const float* w_gate,
                    const float* bias, const float* logit_offset, float* weights, int32_t* indices,
                    void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Hash-routed gate ("From One Giant FFN to 384 Tiny Experts", section 11.1; table from
 * "How was DeepSeek V4's tid2eid derived?"): indices[t, j] = tid2eid[token_ids[t], j] in table
 * order; weights = affinity(x . w_gate[e]) at those experts, renormalised when desc->renorm,
 * times route_scale.  No bias, no groups.
 * token_ids [T] int32 in [0, vocab); tid2eid [vocab, k] int32 in [0, E); x [T, d] bf16;
 * w_gate [E, d] fp32.  Outputs as for moe_gate.
 */
moe_status moe_hash_gate(const moe_layer_desc* desc, int T, const int32_t* token_ids,
                         const int32_t* tid2eid, int vocab, const moe_bf16* x, const float* w_gate,
                         float* weights, int32_t* indices, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/*
 * 2-gram hash gate ("How was DeepSeek V4's tid2eid derived?", section "An extreme case"): for the
 * pair (a, b) = (prev_ids[t], token_ids[t]), expert j is (a * primes[j] + b) mod E, computed exactly
 * in 64-bit unsigned arithmetic; a row may name the same expert more than once.  Weights as for
 * moe_hash_gate, a repeated expert's affinity counted once per occurrence in the renormalisation.
 * prev_ids, token_ids [T] int32 on the device, in [0, vocab): prev_ids[t] is the token before t in
 * its sequence (at a sequence start the caller supplies one, e.g. a begin-of-sequence id).
 * primes [k] HOST int64: k distinct primes with vocab < primes[j] < 2^32 (MOE_ERR_INVALID
 * otherwise, checked on the host before any launch).  x, w_gate and outputs as for moe_hash_gate;
 * out-of-range ids are clamped and reported as MOE_ERR_DEVICE through moe_get_error.
 */
moe_status moe_ngram_gate(const moe_layer_desc* desc, int T, const int32_t* prev_ids,
                          const int32_t* token_ids, const int64_t* primes, int vocab,
                          const moe_bf16* x, const float* w_gate, float* weights, int32_t* indices,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Greedy tid2eid builder, HOST ONLY ("How was DeepSeek V4's tid2eid derived?", the greedy rule
 * under eq. 2): tokens are visited by descending frequency p (equal p: lower token id first);
 * each takes the k experts of least current load (equal loads: lower expert index first), written
 * in that order to its row, and each of them gains p_i / k (fp64).
 * p [m] host fp64; tid2eid [m, k] host int32 (out); loads [n_experts] host fp64 (out) or NULL.
 * Returns MOE_ERR_INVALID for m < 0, k < 1, k > n_experts or NULL pointers.
 */
moe_status moe_build_tid2eid(const double* p, int m, int n_experts, int k, int32_t* tid2eid,
                             double* loads);

/*
 * Randomised greedy tid2eid builder, HOST ONLY ("How was DeepSeek V4's tid2eid derived?", the
 * paragraph after the reference implementation): one greedy pass as in moe_build_tid2eid per
 * visiting order, where orders [runs, m] host int32 holds in row r a permutation of the token ids
 * 0..m-1 (the caller draws them at random); keeps the table of least max_vio = n_experts * max f - 1
 * (equal max_vio: the earlier run).
 * Outputs: tid2eid [m, k] host int32 and loads [n_experts] host fp64 (or NULL) of the kept run;
 * max_vio [runs] host fp64 (or NULL) of every run, so that a caller can keep several of the best;
 * kept (host, or NULL) the index of the kept run.  MOE_ERR_INVALID for runs < 1, a row of orders
 * that is not a permutation, or the conditions of moe_build_tid2eid.
 */
moe_status moe_build_tid2eid_best(const double* p, int m, int n_experts, int k, const int32_t* orders,
                                  int runs, int32_t* tid2eid, double* loads, double* max_vio,
                                  int32_t* kept);

/*
 * tid2eid tables on disk, HOST ONLY.  The pages have no counterpart to these calls: a table is built
 * once per vocabulary and frequency vector ("How was DeepSeek V4's tid2eid derived?") and then used
 * by every forward, so it is kept in a file next to the weights.  Layout, little-endian: the 8 bytes
 * "MOETID01"; int32 m, k, n_experts and a reserved 0; the uint64 FNV-1a hash of the bytes of the m
 * fp64 frequencies p the table was built from (0 when saved without p); then m*k int32 expert ids,
 * row-major.
 *   moe_tid2eid_save   writes tid2eid [m, k] (host) and, when p [m] (host) is given, its hash.  Every
 *                      id must lie in [0, n_experts), else MOE_ERR_INVALID before anything is written.
 *   moe_tid2eid_header reads m, k and n_experts of a file (host ints) so that the caller can size
 *                      the table.
 *   moe_tid2eid_load   reads the table into tid2eid [m, k] (host).  MOE_ERR_INVALID when the file is
 *                      not such a table (magic, length), when its m, k or n_experts differ from the
 *                      arguments, when p is given and the file does not carry its hash (a table built
 *                      for other frequencies, or saved without them), or when an id lies outside
 *                      [0, n_experts); tid2eid is then left untouched.  p may be NULL to skip the check.
 * MOE_ERR_IO when the file cannot be opened, read or written.
 */
moe_status moe_tid2eid_save(const char* path, const int32_t* tid2eid, int m, int k, int n_experts,
                            const double* p);
moe_status moe_tid2eid_header(const char* path, int* m, int* k, int* n_experts);
moe_status moe_tid2eid_load(const char* path, int32_t* tid2eid, int m, int k, int n_experts,
                            const double* p);

/*
 * Dispatch ("DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt: bincount and x[idx]):
 *   counts[e] = #slots choosing e; offsets = exclusive prefix sum (offsets[E] = T*k);
 *   slots are laid out expert by expert, in slot order inside each expert (stable);
 *   row_of_slot[s] = the row of slot s; tok_of_row[r] = the token of row r; x_perm[r] = x[tok_of_row[r]].
 * indices [T, k] int32; x [T, d] bf16.  Outputs: counts [E], offsets [E+1], row_of_slot [T*k],
 * tok_of_row [T*k] int32; x_perm [T*k, d] bf16, or NULL to skip writing it (for
 * moe_expert_ffn_gather, which reads the rows of x through tok_of_row instead).
 */
moe_status moe_dispatch(const moe_layer_desc* desc, int T, const int32_t* indices, const moe_bf16* x,
                        int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* tok_of_row,
                        moe_bf16* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Dispatch without a workspace, for callers that cannot allocate device memory: for example a
 * plugin that a host framework hands only its input and output buffers (the framework owns all
 * device memory), or a loop where an allocation's implicit device synchronisation is not allowed.
 * The pages have no counterpart to this call: it is moe_dispatch with its scratch (a block counter,
 * per-block histograms and row bases) in a fixed 1 MiB array of library-owned device memory, which
 * every GPU that loads the library holds until the process exits.  It allocates nothing itself.
 * Arguments, outputs, layouts and accepted descriptors as for moe_dispatch, without ws.  Rules:
 *   - n_coarse * E must not exceed 131040, else MOE_ERR_UNSUPPORTED before any launch; n_coarse is
 *     the number of histogram blocks, max(1, ceil(T*k / 1024)) up to 64 blocks (T*k <= 65536), about
 *     64 up to T*k = 524288, and ceil(T*k / 8192) beyond (so at E = 512, T*k up to 2088960);
 *   - every call looks up the array's device address with the call's device current; the first call
 *     on a device may initialise the library's module there, so make it before any stream capture;
 *   - every call shares the array and keeps what the last call left in it: each call clears the
 *     block counter with a 4-byte cudaMemsetAsync on `stream`, and its kernels write the rest before
 *     reading it; calls whose kernels overlap on the GPU (other streams, other host threads) race on
 *     the array and must not be issued;
 *   - out-of-range expert indices are clamped as in moe_dispatch but not reported (no error word).
 */
moe_status moe_dispatch_static(const moe_layer_desc* desc, int T, const int32_t* indices, const moe_bf16* x,
                               int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* tok_of_row,
                               moe_bf16* x_perm, moe_stream_t stream);

/*
 * The experts ("From One Giant FFN to 384 Tiny Experts", section 1, SwiGLU): for every routed
 * expert e, on its rows x_perm[offsets[e] : offsets[e+1]], and for the shared expert on all of x:
 *   h = bf16( silu(x . w1[e]^T) * (x . w3[e]^T) ),  out = bf16( h . w2[e]^T ),
 * with fp32 accumulation on the tensor cores.
 * With desc->swiglu_limit > 0 the gate branch is first capped above at the limit and the value
 * branch clamped to [-limit, limit]; with row_weights non-NULL, routed row r's h is multiplied by
 * row_weights[r] before its rounding (the shared expert's rows by 1).
 * x_perm [T*k, d] bf16; offsets [E+1] int32 (device, as written by moe_dispatch); row_weights [T*k]
 * fp32 or NULL; x [T, d] bf16; w1, w3 [E+1, I, d] bf16; w2 [E+1, d, I] bf16 (shared expert at index E).
 * Outputs: out_perm [T*k, d] bf16 (row r = expert output of row r); out_shared [T, d] bf16.
 */
moe_status moe_expert_ffn(const moe_layer_desc* desc, int T, const moe_bf16* x_perm,
                          const int32_t* offsets, const float* row_weights, const moe_bf16* x, const moe_bf16* w1,
                          const moe_bf16* w3, const moe_bf16* w2, moe_bf16* out_perm,
                          moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn with the dispatch gather x_perm[r] = x[tok_of_row[r]] ("DeepSeek-V3.2-Exp - Routing
 * weights", moe-forward excerpt: x[idx]) done by the up-projection kernel's own loads: routed row r
 * is read from row tok_of_row[r] of x, so x_perm is never written.  tok_of_row [T*k] int32 (device,
 * as written by moe_dispatch; values outside [0, T) are clamped).  Results are bit-identical to
 * moe_expert_ffn on the x_perm that moe_dispatch writes.  Needs inter_dim % 256 == 0 (the CTA-pair
 * kernel), else MOE_ERR_UNSUPPORTED.  Other arguments as for moe_expert_ffn.
 * It saves the T*k*d*2 bytes of x_perm and the gather's pass over them, at a cost: on a B200 the
 * gathered up projection of the V3-shaped prefill layer ran about 20 % slower than moe_expert_ffn's,
 * more than the gather it replaces, so moe_forward keeps the separate gather.
 */
moe_status moe_expert_ffn_gather(const moe_layer_desc* desc, int T, const int32_t* tok_of_row,
                                 const int32_t* offsets, const float* row_weights, const moe_bf16* x,
                                 const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2, moe_bf16* out_perm,
                                 moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Combine ("DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt; "DeepSeek V4.1 - Add
 * shared"): y[t] = bf16( sum_j weights[t, j] * out_perm[row_of_slot[t*k + j]] + out_shared[t] ),
 * accumulated in fp32 (slot order, shared term last).  One thread owns each output element, so
 * the result does not depend on scheduling.  out_shared may be NULL (no shared term); weights may be
 * NULL, for expert outputs that already carry their weights (desc->weight_in_expert).
 * out_perm [T*k, d] bf16; row_of_slot [T*k] int32; weights [T, k] fp32; y [T, d] bf16 (out).
 */
moe_status moe_combine(const moe_layer_desc* desc, int T, const moe_bf16* out_perm,
                       const int32_t* row_of_slot, const float* weights, const moe_bf16* out_shared,
                       moe_bf16* y, moe_stream_t stream);

/*
 * MoE.forward: gate (or hash gate when token_ids and tid2eid are both given), dispatch, experts,
 * combine, all on `stream` with no host synchronisation.  Intermediate tensors live in `ws`.
 * Optional outputs (NULL to skip): weights_out [T, k] fp32, indices_out [T, k] int32,
 * counts_out [E] int32.  y [T, d] bf16.  The results equal those of the stage calls in sequence
 * (moe_gate / moe_hash_gate, moe_dispatch, moe_expert_ffn, moe_combine) bit for bit; when the gate
 * runs on the split-K cluster router, that router also counts dispatch's histogram, so dispatch is
 * one launch fewer.  desc->gate_prepared applies as for moe_gate.
 */
moe_status moe_forward(const moe_layer_desc* desc, int T, const moe_bf16* x, const int32_t* token_ids,
                       const int32_t* tid2eid, int vocab, const float* w_gate, const float* bias,
                       const float* logit_offset, const moe_bf16* w1, const moe_bf16* w3,
                       const moe_bf16* w2, moe_bf16* y, float* weights_out, int32_t* indices_out,
                       int32_t* counts_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Auxiliary-loss-free balancing step ("From One Giant FFN to 384 Tiny Experts", section 6, the bias
 * update run once per training step): with the balanced load T * topk / E, bias[e] -= gamma where
 * counts[e] is above it, bias[e] += gamma where below, unchanged where equal (compared exactly as
 * counts[e] * E against T * topk); fp32, in place, on `stream`.
 * counts [E] int32 on the device: slots routed to each expert over the T tokens of the batch (the
 * counts of moe_dispatch, or moe_forward's counts_out); bias [E] fp32 on the device.  gamma >= 0 and
 * finite (the page's V3 schedule: 0.001, then 0).  Needs no workspace.
 */
moe_status moe_update_bias(const moe_layer_desc* desc, int T, const int32_t* counts, float* bias,
                           float gamma, moe_stream_t stream);

/*
 * MXFP4 expert weights ("From One Giant FFN to 384 Tiny Experts", section 11.6: expert weights in
 * the OCP MXFP4 format, E2M1 elements in 1x32 blocks, each block sharing one power-of-two scale).
 * Each matrix of moe_expert_ffn is replaced by its codes and scales, stacked over the E routed
 * experts and the shared expert (index E) as there:
 *   w1, w3   [E+1, I, d/2] bytes: row r of expert e holds elements 2j (low nibble) and 2j+1 (high
 *            nibble) of its d inputs in byte j; each nibble is an E2M1 code (bit 3 sign, bits 2-1
 *            exponent with bias 1, bit 0 mantissa: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6);
 *   w1_scale, w3_scale [E+1, I, d/32] bytes: UE8M0 scale of elements 32b..32b+31 of the row, the
 *            block's values being code value * 2^(scale - 127);
 *   w2 [E+1, d, I/2] and w2_scale [E+1, d, I/32]: the same for the down projection.
 * Scales must lie in [2, 252] (every decoded value is then a normal bf16 number); others are
 * clamped into it and reported as MOE_ERR_DEVICE with info 0x10000 + scale.  All six pointers are
 * device memory, 16-byte aligned.
 */
typedef struct moe_mxfp4_weights {
  const uint8_t* w1;
  const uint8_t* w1_scale;
  const uint8_t* w3;
  const uint8_t* w3_scale;
  const uint8_t* w2;
  const uint8_t* w2_scale;
} moe_mxfp4_weights;

/*
 * moe_expert_ffn with MXFP4 weights: every expert computes with its decoded weights, which are exact
 * in bf16, so the arithmetic (bf16 operands, fp32 accumulation, bf16 h and outputs, clamp and row
 * weights) is that of moe_expert_ffn holding the decoded weights.  Needs inter_dim % 512 == 0 and
 * dim % 512 == 0 (MOE_ERR_UNSUPPORTED otherwise).  Other arguments as for moe_expert_ffn.
 */
moe_status moe_expert_ffn_mxfp4(const moe_layer_desc* desc, int T, const moe_bf16* x_perm,
                                const int32_t* offsets, const float* row_weights, const moe_bf16* x,
                                const moe_mxfp4_weights* weights_mxfp4, moe_bf16* out_perm,
                                moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_expert_ffn_mxfp4 reading routed rows through tok_of_row, as moe_expert_ffn_gather does. */
moe_status moe_expert_ffn_mxfp4_gather(const moe_layer_desc* desc, int T, const int32_t* tok_of_row,
                                       const int32_t* offsets, const float* row_weights, const moe_bf16* x,
                                       const moe_mxfp4_weights* weights_mxfp4, moe_bf16* out_perm,
                                       moe_bf16* out_shared, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_forward with MXFP4 expert weights (as for moe_expert_ffn_mxfp4); other arguments as for
 * moe_forward.
 */
moe_status moe_forward_mxfp4(const moe_layer_desc* desc, int T, const moe_bf16* x,
                             const int32_t* token_ids, const int32_t* tid2eid, int vocab,
                             const float* w_gate, const float* bias, const float* logit_offset,
                             const moe_mxfp4_weights* weights_mxfp4, moe_bf16* y, float* weights_out,
                             int32_t* indices_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * Synchronises `stream`, then returns the first error a kernel recorded in `ws` since the last
 * call (MOE_OK if none) and clears it.  *info (host, may be NULL) receives the offending value.
 */
moe_status moe_get_error(void* ws, moe_stream_t stream, int32_t* info);

/* A static, human-readable name for a status. */
const char* moe_status_str(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
