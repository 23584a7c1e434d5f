/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE SwiGLU FFN layer library (libmoe.so).
 *
 * The layer: given routed tokens (top-k expert ids and gate weights per token),
 * reorder the routed rows by expert, run every expert's SwiGLU FFN on its rows
 * as one grouped GEMM pair, and sum each token's top-k results back in token
 * order, weighted by its gate weights.
 *
 * Sources (pages the method is taken from):
 *   [PTO]   "PTO MoE算子实战dispatch/combine如何与计算流水线重叠实现性能倍增",
 *           sections "MoE dispatch/combine 为什么慢" (reorder by expert -> expert
 *           FFN -> top-k weighted accumulation) and "MegaMoE 融合算子七阶段"
 *           (FrontReorder, Dispatch, GMM1, SwiGLU, GMM2, Combine, Unpermute).
 *   [GG]    "Grouped GEMM 为什么适合 MoE？从碎片小矩阵到通信友好的算子设计",
 *           sections "Grouped GEMM 到底解决什么问题" (C_i = A_i x B_i with
 *           per-problem sizes; a fixed set of CTAs pulls tiles from one queue),
 *           "1. Tiling", "2. Double-buffer pipeline", "Fused GemmAdd" (fp32
 *           epilogue arithmetic, one cast on output).
 *   [COMET] "COMET: Fine-grained Computation-communication Overlapping for
 *           Mixture-of-Experts" (paper review), sections 4.1 (shared-tensor
 *           decomposition and rescheduling) and 4.2 (thread-block specialisation,
 *           adaptive thread-block count n_c chosen from profiled metadata).
 *
 * Conventions for every call
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; the
 *     caller allocates and owns all buffers.  The library allocates no device
 *     memory and keeps no device state between calls.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream) and does not synchronise.
 *   - Errors that the host can see (null pointers, bad sizes, misalignment,
 *     unsupported shapes, short workspace) return before anything is launched;
 *     moe_last_error() then gives a one-line message (thread-local).
 *   - Errors that only the device can see (an expert id out of [0, E), a wait
 *     that ran out of time) are recorded in the status word at the start of the
 *     workspace; read it with moe_get_device_status().  Kernels never trap.
 *   - bf16 tensors are row-major with the stated shapes and dense rows; every
 *     base pointer must be 16-byte aligned.  Integers are int32, weights fp32.
 *   - R = M * topk is the number of routed rows.  Flat routed index i = t*topk+k.
 *   - M = 0 is legal: nothing is launched and MOE_OK is returned.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, negative size, topk > E, ...      */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* H or F not a multiple of 64, E > MOE_MAX_EXPERTS */
  MOE_ERR_BAD_EXPERT_ID = 3,      /* device: some topk_ids entry is outside [0, E)   */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,
  MOE_ERR_TIMEOUT = 5,            /* device: a bounded wait ran out                   */
  MOE_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed                */
  MOE_ERR_MISALIGNED = 7,         /* a base pointer is not 16-byte aligned            */
  MOE_ERR_BAD_INDEX = 8           /* device: a permutation entry is outside [0, R)    */
} moe_status;

/* Largest expert count the kernels accept. */
#define MOE_MAX_EXPERTS 1024

/* Epilogue of moe_grouped_gemm ([GG] "Fused GemmAdd": the accumulator is kept in
 * fp32 and transformed before the single cast to bf16 on output). */
typedef enum moe_epilogue {
  /* C[s, n] = bf16(acc[s, n]);  C is [R, N]. */
  MOE_EPI_STORE = 0,
  /* B = W1 holds gate columns [0, N/2) and up columns [N/2, N);
   * C[s, j] = bf16(silu(acc[s, j]) * acc[s, N/2 + j]),  silu(v) = v / (1 + e^-v);
   * C is [R, N/2].  ([PTO] "MegaMoE 融合算子七阶段": SwiGLU consumes GMM1's
   * output as soon as it is produced.) */
  MOE_EPI_SWIGLU = 1,
  /* C[perm[s], n] = w_sorted[s] * acc[s, n]: the gate-weighted row goes straight
   * to its token-major slot i = t*topk + k; C is FP32 [R, N].  It stays in fp32
   * because moe_combine sums it once more: one bf16 rounding fewer on the path
   * to the layer output. */
  MOE_EPI_WEIGHT_SCATTER = 2
} moe_epilogue;

/* Which call a workspace is sized for. */
typedef enum moe_op {
  MOE_OP_PLAN = 0,
  MOE_OP_DISPATCH = 1,
  MOE_OP_GROUPED_GEMM = 2,
  MOE_OP_COMBINE = 3,
  MOE_OP_FFN_FUSED = 4,
  MOE_OP_ROUTE = 5,
  MOE_OP_FFN_FP8 = 6,  /* moe_ffn_fused_fp8 */
  MOE_OP_GEMM_MX = 7,  /* moe_grouped_gemm_mx: M = R, H = N, F = K */
  MOE_OP_FFN_MX = 8    /* moe_ffn_fused_mx */
} moe_op;

/* Version of this ABI (incremented on any incompatible change). */
int moe_abi_version(void);

/* Bytes of device workspace `op` needs for this shape (always >= 256; the first
 * 256 bytes are a control block: the device status word and the grouped GEMM's
 * tile queue; the plan also keeps per-chunk expert histograms after it, 256 *
 * (E + 1) int32).  The workspace must be 256-byte aligned.  Its contents need no
 * initialisation except that the control block must read 0 before the first
 * call (zero the buffer once, or call moe_get_device_status once, which clears
 * it); every call leaves the tile queue at zero again.  A workspace serves one
 * call at a time: calls that overlap on the GPU need workspaces of their own. */
size_t moe_workspace_size(moe_op op, int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk);

/*
 * moe_route -- the router in front of the layer (the grouped GEMM article's
 * introduction: the router hands each token to some experts; the pages define
 * no more, so this is the plainest reading):
 *   topk_ids[t, :] = the topk experts with the largest logits[t, :], largest
 *                    first, ties to the lower expert index
 *   topk_w[t, k]   = exp(l_k) / sum_j exp(l_j) over the chosen logits l_k
 *   logits fp32 [M, E] (finite), topk_ids int32 [M, topk], topk_w fp32 [M, topk].
 * Selection compares the given fp32 values exactly; the softmax runs in fp32.
 * topk <= min(E, 32), E <= MOE_MAX_EXPERTS.
 */
moe_status moe_route(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* topk_ids,
                     float* topk_w, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_plan -- routing plan ([PTO] "MegaMoE 融合算子七阶段", FrontReorder; [GG]
 * "Grouped GEMM 到底解决什么问题": per-problem sizes passed as arrays).
 *   topk_ids  int32 [M, topk]   expert of each routed row
 *   topk_w    fp32  [M, topk]   gate weight of each routed row (may be NULL if
 *                               w_sorted is NULL)
 *   counts    int32 [E]         out: rows routed to each expert
 *   offsets   int32 [E+1]       out: exclusive prefix sum, offsets[E] = R
 *   perm      int32 [R]         out: perm[s] = i, the flat routed row held in
 *                               expert-ordered slot s; stable: within one expert
 *                               the slots follow ascending i
 *   inv_perm  int32 [R]         out: inv_perm[perm[s]] = s (may be NULL)
 *   w_sorted  fp32  [R]         out: w_sorted[s] = topk_w[perm[s]] (may be NULL)
 * Duplicate ids within a token are legal and counted twice.  If any id is out of
 * [0, E), the device status becomes MOE_ERR_BAD_EXPERT_ID, counts and offsets
 * are all zero and perm/inv_perm are the identity (safe for later calls).
 */
moe_status moe_plan(const int32_t* topk_ids, const float* topk_w, int64_t M, int32_t E,
                    int32_t topk, int32_t* counts, int32_t* offsets, int32_t* perm,
                    int32_t* inv_perm, float* w_sorted, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * moe_route_plan -- moe_route and moe_plan in one call, the routing front end
 * fused with the plan's first pass ([PTO] "MegaMoE 融合算子七阶段": FrontReorder
 * directly behind the router): one kernel routes every token (as moe_route) and
 * counts its routed rows per expert into per-chunk histograms in the workspace;
 * a second kernel scans them into offsets and scatters the stable permutation.
 *   logits fp32 [M, E]; out: topk_ids int32 [M, topk], topk_w fp32 [M, topk]
 *   (exactly as moe_route writes them), counts [E], offsets [E+1], perm [R],
 *   inv_perm [R] (may be NULL), w_sorted [R] (may be NULL): exactly as moe_plan
 *   writes them for those ids and weights.
 * Workspace: moe_workspace_size(MOE_OP_PLAN, ...).  topk <= min(E, 32).
 */
moe_status moe_route_plan(const float* logits, int64_t M, int32_t E, int32_t topk,
                          int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv_perm, float* w_sorted, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * moe_dispatch -- permute ([PTO] Dispatch; [COMET] 3.2, layer 0 token dispatch):
 *   xp[s, :] = x[perm[s] / topk, :]          x bf16 [M, H], xp bf16 [R, H]
 * A pure copy of bf16 bits.  H must be a multiple of 8.  A perm entry outside
 * [0, R) writes a zero row and records MOE_ERR_BAD_INDEX.
 */
moe_status moe_dispatch(const void* x, const int32_t* perm, int64_t M, int64_t H, int32_t topk,
                        void* xp, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_grouped_gemm -- one persistent tcgen05 kernel for every expert's GEMM
 * ([GG] "Grouped GEMM 到底解决什么问题"):
 *   for every expert e and row s in [offsets[e], offsets[e+1]):
 *     acc[s, n] = sum_k A[s, k] * B[e, k, n]     (fp32 accumulate)
 *   then the epilogue `epi` writes C (see moe_epilogue).
 *   A bf16 [R, K] (rows in expert order), B bf16 [E, K, N] row-major (N
 *   contiguous), offsets int32 [E+1] as written by moe_plan.
 *   w_sorted, perm: used by MOE_EPI_WEIGHT_SCATTER only (else may be NULL).
 * K and N must be multiples of 64 (for SWIGLU, N/2 must be a multiple of 64).
 */
moe_status moe_grouped_gemm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                            int64_t R, int64_t K, int64_t N, moe_epilogue epi,
                            const float* w_sorted, const int32_t* perm, void* C, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * moe_combine -- top-k reduction back to token order ([PTO] "MoE dispatch/combine
 * 为什么慢": topK 加权累加; Combine + Unpermute):
 *   out[t, :] = bf16( sum_{k=0}^{topk-1} wk * fp32(y[row(t, k), :]) )   (k ascending)
 *   row(t, k) = inv_perm[t*topk + k] if inv_perm != NULL (y in expert order),
 *               t*topk + k           if inv_perm == NULL (y token-major, as
 *                                    written by MOE_EPI_WEIGHT_SCATTER)
 *   wk = topk_w[t*topk + k] if topk_w != NULL, else 1.
 *   y [R, H] is bf16 (y_fp32 = 0) or fp32 (y_fp32 = 1); out bf16 [M, H];
 *   H a multiple of 8.  An index outside [0, R) contributes zero and records
 *   MOE_ERR_BAD_INDEX.
 */
moe_status moe_combine(const void* y, int32_t y_fp32, const int32_t* inv_perm,
                       const float* topk_w, int64_t M, int64_t H, int32_t topk, void* out,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * moe_ffn_fused -- the whole layer:
 *   out[t, :] = sum_k topk_w[t, k] * FFN_{topk_ids[t, k]}(x[t, :])
 *   FFN_e(v) = (silu(v . W1[e][:, :F]) * (v . W1[e][:, F:])) . W2[e]
 *   x bf16 [M, H], W1 bf16 [E, H, 2F], W2 bf16 [E, F, H], out bf16 [M, H].
 * It runs plan -> dispatch -> GEMM1 with the SwiGLU epilogue -> GEMM2 with the
 * gate-weight scatter epilogue -> combine.  counts [E], offsets [E+1] and perm
 * [R] receive the plan (as moe_plan).  The intermediates (expert-ordered x and
 * the SwiGLU activations in bf16, the gate-weighted expert outputs in fp32)
 * live in the workspace (moe_workspace_size(MOE_OP_FFN_FUSED, ...)).
 *   n_c: thread blocks given to the memory stages (dispatch / combine) while the
 *   GEMM blocks run, [COMET] 4.2.1-4.2.2.  0 runs the stages as consecutive
 *   kernels; n_c >= 1 runs plan, then ONE persistent cooperative kernel with one
 *   CTA per SM, of which n_c only dispatch and combine while the rest run the
 *   GEMM tiles with six further memory warps each, handing off through
 *   per-m-tile and per-token ready counters;
 *   -1 takes the value from the library's profiled table for this shape.
 *   n_c must be below 65 and below the SM count.
 * H and F must be multiples of 64.
 */
moe_status moe_ffn_fused(const void* x, const void* W1, const void* W2, const int32_t* topk_ids,
                         const float* topk_w, int64_t M, int64_t H, int64_t F, int32_t E,
                         int32_t topk, int32_t n_c, void* out, int32_t* counts,
                         int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * moe_combine_add -- moe_combine with the Fused GemmAdd epilogue ([GG] "Fused
 * GemmAdd": Y = cast(alpha * Acc_fp32 + beta * Add_fp32), the addition done in
 * fp32 before the one cast):
 *   out[t, :] = bf16( alpha * sum_k wk * fp32(y[row(t, k), :]) + beta * fp32(add[t, :]) )
 * with row(t, k), wk, y and y_fp32 as in moe_combine; add bf16 [M, H] (e.g. the
 * residual stream), 16-byte aligned.  add is read only when beta != 0 (it may
 * then be NULL); add may be the same buffer as out.  alpha = 1 and beta = 0
 * give exactly moe_combine's result.
 */
moe_status moe_combine_add(const void* y, int32_t y_fp32, const int32_t* inv_perm,
                           const float* topk_w, const void* add, float alpha, float beta,
                           int64_t M, int64_t H, int32_t topk, void* out, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * moe_ffn_fused_add -- the layer with the Fused GemmAdd epilogue ([GG] "Fused
 * GemmAdd"), e.g. the residual connection around the MoE layer:
 *   out[t, :] = bf16( alpha * sum_k topk_w[t, k] * FFN_{topk_ids[t, k]}(x[t, :])
 *                     + beta * add[t, :] )
 * The addition happens in fp32 inside the combine, before the single bf16 cast
 * (no extra pass over out).  add bf16 [M, H], read only when beta != 0; it may be
 * x itself (out = x + layer(x) with alpha = beta = 1) or the same buffer as out.
 * Other arguments, the workspace (moe_workspace_size(MOE_OP_FFN_FUSED, ...)) and
 * the errors are those of moe_ffn_fused; the stages run as consecutive kernels
 * (as moe_ffn_fused with n_c = 0).  alpha = 1 and beta = 0 give exactly
 * moe_ffn_fused's result.
 */
moe_status moe_ffn_fused_add(const void* x, const void* W1, const void* W2,
                             const int32_t* topk_ids, const float* topk_w, const void* add,
                             float alpha, float beta, int64_t M, int64_t H, int64_t F, int32_t E,
                             int32_t topk, void* out, int32_t* counts, int32_t* offsets,
                             int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/* Size of the library's own device scratch used by moe_ffn_fused_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * moe_ffn_fused_noalloc -- the same layer as moe_ffn_fused, for callers that
 * cannot allocate device memory.  The pages have no counterpart of this call.
 *
 * Who needs it: a host program that is handed only its input and output
 * buffers (a C or plugin caller with no device allocator of its own), or a
 * process whose device memory was reserved up front by another allocator, has
 * no way to provide the workspace moe_ffn_fused asks for -- a cudaMalloc would
 * fail, or would stall the device at a bad moment.  This call takes no
 * workspace and allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library routine).  Its intermediates live in a fixed device array of
 * MOE_NOALLOC_SCRATCH_BYTES (64 MiB) inside the library, which every GPU that
 * loads the library holds until the process exits.
 *
 * Arguments are those of moe_ffn_fused without n_c and workspace (the stages
 * run as consecutive kernels on `stream`), plus
 *   status  int32 [1] device pointer (may be NULL): receives this call's device
 *           status word (a moe_status; MOE_ERR_BAD_EXPERT_ID etc.).
 * Host-side checks and their status codes are those of moe_ffn_fused (shape
 * checks first, then the scratch limit, then pointers).  When the device status
 * is not MOE_OK (e.g. an expert id out of range), `out` is undefined: it may
 * hold values computed from an earlier call's intermediates.
 * Limit: the intermediates of R = M*topk rows need
 *   256 + 256*(E+1)*4 + R*H*2 + R*F*2 + R*H*4 + R*4 bytes (each part rounded
 *   up to 256);
 * a shape that needs more than MOE_NOALLOC_SCRATCH_BYTES is rejected with
 * MOE_ERR_WORKSPACE_TOO_SMALL before anything is launched (e.g. H=7168, F=4096,
 * topk=8 fits up to M=163 tokens; H=4096, F=14336, topk=2 up to M=630).
 * The first call on a device looks up the array's device address (with that
 * device current) and remembers it; make that first call before any stream
 * capture.  Every call shares the one array and it keeps the previous call's
 * contents: calls that overlap on the GPU (on different streams, or from
 * different threads without ordering) race on it and must be serialised by the
 * caller.
 */
moe_status moe_ffn_fused_noalloc(const void* x, const void* W1, const void* W2,
                                 const int32_t* topk_ids, const float* topk_w, int64_t M,
                                 int64_t H, int64_t F, int32_t E, int32_t topk, void* out,
                                 int32_t* counts, int32_t* offsets, int32_t* perm,
                                 int32_t* status, void* stream);

/* ---------------------------------------------------------------- FP8 (E4M3)
 * The down projection on 8-bit floats ([PTO] "MegaMoE 融合算子七阶段": SwiGLU
 * consumes each GMM1 segment and quantises it, so that GMM2 runs on quantised
 * activations).  E4M3 is the 8-bit float with 4 exponent bits (bias 7), 3
 * mantissa bits, no infinities, largest finite 448.  A quantised value is
 * q = nearest E4M3 to (v / scale) computed in fp32, ties to even, saturating at
 * 448; scale = (largest |v| of its group) / 448 in fp32, 1 for an all-zero
 * group, so that v ~= scale * q and the group's largest element maps to +-448.
 */

/* moe_quantize_weights_e4m3 -- offline, once per weight tensor:
 *   W bf16 [E, K, N] row-major (the layout of W2, N contiguous)
 *   Wq  E4M3 bytes [E, N, K] (K contiguous: the K-major operand of the FP8 GEMM)
 *   scale fp32 [E, N]: one scale per (expert, output column), over K.
 * K and N must be multiples of 16.  All pointers device, caller-owned. */
moe_status moe_quantize_weights_e4m3(const void* W, int32_t E, int64_t K, int64_t N, void* Wq,
                                     float* scale, void* stream);

/* moe_quantize_rows_e4m3 -- per-row quantisation of a bf16 matrix:
 *   A bf16 [R, K] -> Aq E4M3 bytes [R, K], scale fp32 [R] (one per row).
 * K must be a multiple of 64 and at most 32768.  Workspace as for
 * MOE_OP_GROUPED_GEMM (the status word).  Rows are independent.  R = 0 is a
 * no-op. */
moe_status moe_quantize_rows_e4m3(const void* A, int64_t R, int64_t K, void* Aq, float* scale,
                                  void* ws, size_t ws_bytes, void* stream);

/* moe_grouped_gemm_e4m3 -- grouped GEMM on E4M3 operands (tcgen05 kind::f8f6f4,
 * fp32 accumulate), the FP8 counterpart of moe_grouped_gemm with the
 * MOE_EPI_WEIGHT_SCATTER epilogue:
 *   for every expert e and row s in [offsets[e], offsets[e+1]):
 *     C[d, n] = w * a_scale[s] * b_scale[e, n] * sum_k Aq[s, k] * BqT[e, n, k]
 *   with d = perm[s], w = w_sorted[s] (perm == NULL: d = s; w_sorted == NULL:
 *   w = 1).  Aq [R, K] and BqT [E, N, K] as written by the two quantisers
 *   (K contiguous), C fp32 [R, N].  K and N must be multiples of 64.  Workspace
 *   as for MOE_OP_GROUPED_GEMM.  A perm entry outside [0, R) skips that row and
 *   records MOE_ERR_BAD_INDEX; offsets inconsistent with R record it too and
 *   compute nothing; a wait that runs out records MOE_ERR_TIMEOUT. */
moe_status moe_grouped_gemm_e4m3(const void* Aq, const float* a_scale, const void* BqT,
                                 const float* b_scale, const int32_t* offsets, int32_t E,
                                 int64_t R, int64_t K, int64_t N, const float* w_sorted,
                                 const int32_t* perm, float* C, void* ws, size_t ws_bytes,
                                 void* stream);

/* moe_ffn_fused_fp8 -- the layer with an FP8 down projection:
 *   plan -> dispatch -> GEMM1 + SwiGLU (bf16 h, as moe_ffn_fused) -> h
 *   quantised per row -> FP8 GEMM2 against W2q / w2_scale (from
 *   moe_quantize_weights_e4m3 on W2 [E, F, H]) with the gate-weight scatter ->
 *   combine.  Arguments as moe_ffn_fused (without n_c); the workspace is
 *   moe_workspace_size(MOE_OP_FFN_FP8, ...).  F at most 32768. */
moe_status moe_ffn_fused_fp8(const void* x, const void* W1, const void* W2q,
                             const float* w2_scale, const int32_t* topk_ids, const float* topk_w,
                             int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk, void* out,
                             int32_t* counts, int32_t* offsets, int32_t* perm, void* ws,
                             size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- block-scaled FP8 (MX)
 * The down projection on E4M3 with one scale per block of 32 values along the
 * contraction ([PTO] "MegaMoE 融合算子七阶段": SwiGLU quantises each GMM1 segment
 * it consumes; a block scale needs only the block, so GEMM1's epilogue quantises
 * h as it computes it).  A block of 32 consecutive values along K shares the
 * scale 2^e, e the smallest integer with (largest |v| of the block) <= 448 * 2^e,
 * clamped to [-127, 127] (-127 for an all-zero block); the scale is stored as the
 * byte e + 127 (E8M0); the elements are q = nearest E4M3 to v * 2^-e, ties to
 * even.  The GEMM multiplies E4M3 blocks on the tensor core
 * (tcgen05.mma kind::mxf8f6f4.block_scale), each block product scaled by
 * 2^(ea + eb), and accumulates in fp32.
 */

/* moe_quantize_weights_mx -- offline, once per weight tensor:
 *   W bf16 [E, K, N] row-major (the layout of W2, N contiguous)
 *   BqT E4M3 bytes [E, N, K] (K contiguous), sf bytes [E, N, K / 32] (the
 *   scale code of column n, K block b at sf[(e * N + n) * K / 32 + b]).
 * K must be a multiple of 32, N of 16.  All pointers device, caller-owned. */
moe_status moe_quantize_weights_mx(const void* W, int32_t E, int64_t K, int64_t N, void* BqT,
                                   uint8_t* sf, void* stream);

/* moe_quantize_rows_mx -- A bf16 [R, K] -> Aq E4M3 bytes [R, K] and sf bytes
 * [R, K / 32] (row-major).  K must be a multiple of 32.  Rows are independent;
 * R = 0 is a no-op. */
moe_status moe_quantize_rows_mx(const void* A, int64_t R, int64_t K, void* Aq, uint8_t* sf,
                                void* stream);

/* moe_grouped_gemm_swiglu_mx -- GEMM1 + SwiGLU as moe_grouped_gemm with
 * MOE_EPI_SWIGLU (A bf16 [R, K], B bf16 [E, K, N2] gate | up), with h quantised
 * in blocks of 32 columns inside the epilogue instead of stored in bf16:
 *   hq E4M3 bytes [R, N2 / 2], h_sf bytes [R, N2 / 64] (row-major).
 * h is computed in fp32 from the fp32 accumulator.  N2 must be a multiple of
 * 128, K of 64.  Workspace as for MOE_OP_GROUPED_GEMM.  Error behaviour as
 * moe_grouped_gemm. */
moe_status moe_grouped_gemm_swiglu_mx(const void* A, const void* B, const int32_t* offsets,
                                      int32_t E, int64_t R, int64_t K, int64_t N2, void* hq,
                                      uint8_t* h_sf, void* ws, size_t ws_bytes, void* stream);

/* moe_grouped_gemm_mx -- grouped GEMM on block-scaled E4M3 operands with the
 * gate-weight scatter epilogue:
 *   for every expert e and row s in [offsets[e], offsets[e+1]):
 *     C[d, n] = w * sum over K blocks b of 2^(a_sf[s, b] - 127) * 2^(b_sf[e, n, b] - 127)
 *                                       * sum_{k in b} Aq[s, k] * BqT[e, n, k]
 *   with d = perm[s], w = w_sorted[s] (perm == NULL: d = s; w_sorted == NULL:
 *   w = 1).  Aq [R, K] and a_sf [R, K / 32] as written by moe_quantize_rows_mx
 *   (or moe_grouped_gemm_swiglu_mx), BqT [E, N, K] and b_sf [E, N, K / 32] as
 *   written by moe_quantize_weights_mx; C fp32 [R, N].  K must be a multiple of
 *   32, N of 64.  Workspace: moe_workspace_size(MOE_OP_GEMM_MX, R, N, K, E, 1)
 *   (the scales are rearranged there into the groups the tensor core reads).
 *   A perm entry outside [0, R) skips that row and records MOE_ERR_BAD_INDEX;
 *   offsets inconsistent with R record it too and compute nothing. */
moe_status moe_grouped_gemm_mx(const void* Aq, const uint8_t* a_sf, const void* BqT,
                               const uint8_t* b_sf, const int32_t* offsets, int32_t E, int64_t R,
                               int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                               float* C, void* ws, size_t ws_bytes, void* stream);

/* moe_ffn_fused_mx -- the layer with a block-scaled E4M3 down projection:
 *   plan -> dispatch -> GEMM1 + SwiGLU with h quantised in the epilogue (codes
 *   and scales written to the workspace; no bf16 h) -> MX GEMM2 against
 *   (W2q, w2_sf) from moe_quantize_weights_mx on W2 [E, F, H], with the
 *   gate-weight scatter -> combine.  Arguments as moe_ffn_fused (without n_c);
 *   the workspace is moe_workspace_size(MOE_OP_FFN_MX, ...). */
moe_status moe_ffn_fused_mx(const void* x, const void* W1, const void* W2q, const uint8_t* w2_sf,
                            const int32_t* topk_ids, const float* topk_w, int64_t M, int64_t H,
                            int64_t F, int32_t E, int32_t topk, void* out, int32_t* counts,
                            int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes,
                            void* stream);

/* Synchronises `stream`, returns the device status word of `ws` (a moe_status)
 * and clears the control block (status word MOE_OK, tile queue zero).  Returns
 * MOE_ERR_CUDA if the stream reports an error. */
moe_status moe_get_device_status(void* ws, void* stream);

/* Time limit, in nanoseconds, of every bounded device-side wait (default 2 s).
 * In the single-kernel layer (moe_ffn_fused with n_c > 0) the limit counts time
 * without progress anywhere in the kernel, not the total wait. */
void moe_set_wait_timeout_ns(uint64_t ns);

/* Test hook for failure detection (no GPU fault is ever injected):
 *   kind 0           off (default)
 *   kind 1, index m  the single-kernel layer never publishes m-tile m as
 *                    dispatched, so the GEMM tiles waiting for it run into the
 *                    wait limit and the call ends with MOE_ERR_TIMEOUT in the
 *                    device status, leaving the context usable.
 * Process-wide; returns MOE_ERR_INVALID_ARG for an unknown kind. */
moe_status moe_set_fault_injection(int32_t kind, int32_t index);

/* Stage timing for moe_ffn_fused and moe_ffn_fused_mx (measurement only; the
 * pages have no counterpart).  events: NULL (off, the default) or an array of 6
 * cudaEvent_t handles created by the caller; the caller keeps ownership and must
 * keep them alive while set.  While set, each such call on this thread records
 * events[0] on its stream before the plan and events[i + 1] after stage i
 * (plan, dispatch, GEMM1 + SwiGLU, GEMM2 + scatter, combine), so that the
 * elapsed time between consecutive events is one stage's device time (in
 * moe_ffn_fused_mx the first stage also rearranges the weight scales).  In the
 * single-kernel layer (n_c > 0) events[2..5] are all recorded after the layer
 * kernel.  Recording an event between two kernels serialises them, so a
 * programmatic dependent launch between those kernels no longer overlaps.
 * Thread-local; returns MOE_OK. */
moe_status moe_set_stage_events(void* const* events);

/* Message of the last host-side error on this thread ("" if none). */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
