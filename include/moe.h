/*
 * moe.h — C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * The layer (DeepSeek-V3 technical report summary, xyznot.com, arXiv
 * 2412.19437, Method §2 "DeepSeekMoE with auxiliary-loss-free balancing"):
 *
 *   h'_t = u_t + sum_{i<=N_s} FFN_i^(s)(u_t) + sum_{i<=N_r} g_{i,t} FFN_i^(r)(u_t)
 *   s_{i,t} = Sigmoid(u_t . e_i)
 *   g'_{i,t} = s_{i,t} if s_{i,t} + b_i is among the K_r largest of {s_{j,t} + b_j}, else 0
 *   g_{i,t}  = S * g'_{i,t} / sum_j g'_{j,t}            (S: routed scale)
 *   end of step: b_i -= gamma if expert i is overloaded, += gamma if underloaded
 *
 * A forward pass is five calls on one stream:
 *   moe_route -> moe_permute -> moe_grouped_ffn (routed experts, then the
 *   shared expert as one more group) -> moe_combine, then moe_bias_update.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned and allocated by the
 *     caller; the library allocates no device memory. Scratch memory is passed
 *     in as `workspace` (size from the matching *_workspace_size call).
 *   - Tensors are dense row-major. bf16 tensors are raw 16-bit bfloat16.
 *     Buffers read or written in 16-byte vectors or by TMA must be 16-byte
 *     aligned (stated per argument); a misaligned pointer is rejected.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls
 *     are asynchronous: they enqueue kernels and return; nothing is
 *     synchronised and no device->host copy happens.
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code. Arguments are
 *     validated on the host before anything is enqueued; on error nothing is
 *     launched and outputs are untouched. MOE_ERR_CUDA keeps the CUDA error
 *     for moe_last_cuda_error(). A kernel whose internal bounded wait gives
 *     up (a broken pipeline, never a normal run) records a code that
 *     moe_get_device_status() reports after the stream has drained.
 *   - Tokens with index >= T, experts with no tokens and T = 0 are all valid:
 *     an empty batch produces zero counts and enqueues no expert work.
 *   - Device state: the grouped GEMMs hand out their tiles through one of 256
 *     device counters per GPU, taken round robin when the call enqueues and
 *     zeroed on the call's stream just before its kernel. Two launches share
 *     a counter only if 256 other GEMM launches were enqueued between them,
 *     so at most 256 GEMM launches may be in flight at once on one device. A
 *     launch captured into a CUDA graph keeps the counter it took: do not
 *     replay one graph on two streams at the same time (their launches would
 *     share counters and skip or repeat tiles).
 *
 * Supported shapes (others return MOE_ERR_UNSUPPORTED_SHAPE):
 *   d % 256 == 0, inter % 128 == 0, 1 <= top_k <= 8, top_k <= n_routed <= 256,
 *   1 <= G <= 1024 groups per grouped-FFN call.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Status codes. */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)       /* null/misaligned pointer, negative size, bad enum */
#define MOE_ERR_UNSUPPORTED_SHAPE (-2) /* shape outside the supported set above */
#define MOE_ERR_CUDA (-3)              /* a CUDA runtime/driver call failed */
#define MOE_ERR_DEVICE_TIMEOUT (-4)    /* a kernel's bounded wait ran out */
#define MOE_ERR_WORKSPACE (-5)         /* workspace NULL or smaller than required */

/* Gate form. SIGMOID_BIAS is the technical report's form (above).
 * SOFTMAX_TOPK is the form of the DeepSeekMoE forward listing on "DeepSeek
 * model architecture explained" (deepseekmodel.com): top-k over the raw
 * logits z = u.e (no sigmoid, no bias), then softmax over the k selected
 * logits, times the routed scale. */
typedef enum { MOE_GATE_SIGMOID_BIAS = 0, MOE_GATE_SOFTMAX_TOPK = 1 } moe_gate_kind;

/* Arithmetic type of the expert GEMM operands (see the FP8 section below). */
typedef enum { MOE_BF16 = 0, MOE_FP8_E4M3 = 1 } moe_dtype;

typedef void* moe_stream_t; /* cudaStream_t */

/* ------------------------------------------------------------------ route
 * Gate GEMM + affinity + bias-adjusted top-K + gate normalisation + load
 * histogram (technical report summary, Method §2: s_{i,t}, the g'_{i,t}
 * selection equation, the normalisation of g'; softmax form per the
 * deepseekmodel.com DeepSeekMoE forward listing).
 *
 *   u          [T, d] bf16, 16-B aligned. Token hidden states.
 *   centroids  [n_routed, d] bf16, 16-B aligned. e_i, one row per routed expert.
 *   bias       [n_routed] fp32 or NULL (= all zero). b_i; used for SELECTION
 *              only (the gate uses the unbiased s). Ignored for SOFTMAX_TOPK.
 *   routed_scale  S, multiplies every normalised gate.
 *   topk_idx   [T, top_k] int32 out. Selected experts in descending key
 *              order; equal keys: lower expert index first.
 *   topk_gate  [T, top_k] fp32 out. g of each selected expert (sums to S).
 *   expert_counts [n_routed] int32 out, OVERWRITTEN (not accumulated):
 *              number of (token, slot) pairs routed to each expert.
 * Logits are accumulated in fp32 on the tensor cores from the bf16 inputs;
 * sigmoid, keys and gates are fp32. Batches of 256 tokens or more run on CTA
 * pairs (256 tokens per cluster), smaller ones one CTA per 128 tokens; the
 * results follow from the logits the same way.
 */
MOE_API int moe_route(const void* u, const void* centroids, const float* bias, int T, int d,
                      int n_routed, int top_k, moe_gate_kind kind, float routed_scale,
                      int32_t* topk_idx, float* topk_gate, int32_t* expert_counts,
                      moe_stream_t stream);

/* Split-K form of moe_route for small batches (decode). moe_route gives each
 * CTA 128 tokens and the whole K = d, so a batch of a few hundred tokens runs
 * on one or two SMs, each reading all of the centroids. Here CTA (b, y) takes
 * token block b and the y-th slice of K and writes its fp32 partial logits
 * to the workspace; a second kernel adds the slices (fixed order) and does
 * the same selection, gates and counts as moe_route. Arguments as moe_route,
 * plus:
 *   workspace  device scratch, 16-B aligned, at least
 *              moe_route_splitk_workspace_size(T, d, n_routed) bytes; owned by
 *              the caller, overwritten, may be reused once the call's kernels
 *              have finished on the stream. NULL or too small ->
 *              MOE_ERR_WORKSPACE.
 * The logits are the same fp32 sums of bf16 products as moe_route's, added in
 * another order, so keys closer than the fp32 rounding of a sum may select
 * differently; every other result follows from the logits as in moe_route.
 * The slice count depends on T and d only.
 */
MOE_API size_t moe_route_splitk_workspace_size(int T, int d, int n_routed);
MOE_API int moe_route_splitk(const void* u, const void* centroids, const float* bias, int T,
                             int d, int n_routed, int top_k, moe_gate_kind kind,
                             float routed_scale, int32_t* topk_idx, float* topk_gate,
                             int32_t* expert_counts, void* workspace, size_t ws_bytes,
                             moe_stream_t stream);

/* ------------------------------------------------------------------ permute
 * Dispatch: copy each token's row into an expert-contiguous buffer, once per
 * selected expert (the per-expert grouping of tokens that the deepseekmodel.com
 * DeepSeekMoE listing does with a mask, written as explicit row numbers).
 * Rows of expert i occupy [expert_offsets[i], expert_offsets[i+1]); inside an
 * expert, rows are in ascending token order (stable).
 *
 *   u              [T, d] bf16, 16-B aligned.
 *   topk_idx       [T, top_k] int32 from moe_route (entries outside
 *                  [0, n_routed) are skipped and get pos = -1).
 *   expert_counts  [n_routed] int32 from moe_route.
 *   x_perm         [T*top_k, d] bf16 out, 16-B aligned.
 *   expert_offsets [n_routed + 1] int32 out: exclusive scan of the counts.
 *   pos            [T, top_k] int32 out: row of x_perm holding (t, slot k).
 *   src_token      [T*top_k] int32 out: token of each x_perm row.
 *   workspace      >= moe_permute_workspace_size(T, n_routed) bytes, 16-B aligned.
 */
MOE_API int moe_permute(const void* u, const int32_t* topk_idx, const int32_t* expert_counts,
                        int T, int d, int n_routed, int top_k, void* x_perm,
                        int32_t* expert_offsets, int32_t* pos, int32_t* src_token,
                        void* workspace, size_t ws_bytes, moe_stream_t stream);

MOE_API size_t moe_permute_workspace_size(int T, int n_routed);

/* moe_permute_shared: moe_permute that also copies u's rows once more, to
 * rows [T*top_k, T*top_k + T) of x_perm, so that the always-on shared expert
 * (one expert of the routed experts' inter, technical report summary, Method
 * §2: every token goes through it) runs as group n_routed of the same grouped
 * GEMMs as the routed experts: weights [n_routed + 1, ...] with the shared
 * expert last, and
 *   x_perm          [T*top_k + T, d] bf16 out, 16-B aligned.
 *   expert_offsets  [n_routed + 2] int32 out: entries 0..n_routed as
 *                   moe_permute; entry n_routed + 1 = T*top_k + T. The shared
 *                   group is [expert_offsets[n_routed], T*top_k + T): it starts
 *                   where the routed rows end, which is T*top_k unless routed
 *                   slots were skipped (topk_idx outside [0, n_routed)); the
 *                   rows in between are not written here, get computed by the
 *                   shared expert and are read by nothing.
 * After the down-projection of the n_routed + 1 groups, rows [T*top_k,
 * T*top_k + T) of its output are the shared expert's output for tokens 0..T-1
 * (moe_combine's shared_out). Other arguments and errors as moe_permute. */
MOE_API int moe_permute_shared(const void* u, const int32_t* topk_idx,
                               const int32_t* expert_counts, int T, int d, int n_routed,
                               int top_k, void* x_perm, int32_t* expert_offsets, int32_t* pos,
                               int32_t* src_token, void* workspace, size_t ws_bytes,
                               moe_stream_t stream);

/* moe_permute_index: the index half of moe_permute (expert_offsets, pos,
 * src_token, same definitions and arguments) without copying any row. For
 * the fused mode, where the up-projection gathers the token rows itself
 * (moe_expert_up_swiglu_gather). */
MOE_API int moe_permute_index(const int32_t* topk_idx, const int32_t* expert_counts, int T,
                              int n_routed, int top_k, int32_t* expert_offsets, int32_t* pos,
                              int32_t* src_token, void* workspace, size_t ws_bytes,
                              moe_stream_t stream);

/* moe_permute_noalloc: moe_permute without a workspace argument. The pages
 * have no counterpart: this entry point exists for callers that cannot
 * allocate device memory where they call the library — for example a plugin
 * whose host framework owns the whole device-memory budget and hands it no
 * allocator, or a latency-critical loop that must not call cudaMalloc (which
 * can synchronise the device). It allocates nothing and calls no allocating
 * routine; its scratch is a 256 KiB array in the library's own device memory,
 * reserved on every GPU that loads the library until the process exits.
 *
 * Same arguments, outputs and errors as moe_permute. Limit: ceil(T/128) *
 * n_routed <= 65536 (e.g. T <= 32768 with 256 experts); larger sizes return
 * MOE_ERR_UNSUPPORTED_SHAPE before anything is enqueued.
 * The first call on a device looks up the array's device address (one
 * cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture. Every call on a device shares the one array and
 * leaves its contents behind (nothing in it needs clearing: each call
 * overwrites every entry it reads), so calls that can overlap on the GPU —
 * concurrent streams, or several host threads on one device — race on it and
 * must be serialised by the caller.
 */
MOE_API int moe_permute_noalloc(const void* u, const int32_t* topk_idx,
                                const int32_t* expert_counts, int T, int d, int n_routed,
                                int top_k, void* x_perm, int32_t* expert_offsets, int32_t* pos,
                                int32_t* src_token, moe_stream_t stream);

/* ------------------------------------------------------------------ expert FFN
 * Grouped SwiGLU expert FFN (FFN_i^(r) and FFN_i^(s) of the technical report's
 * output equation; the pages do not define the FFN's inside — SwiGLU without
 * biases, FFN(x) = W2 (silu(W1 x) * (W3 x)), is this library's reading).
 *
 * Group g owns rows [group_offsets[g], group_offsets[g+1]) of x and its own
 * weights. group_offsets is a DEVICE array of G+1 int32, meant to be
 * non-decreasing with 0 <= group_offsets[0] and group_offsets[G] <= rows
 * (moe_permute's expert_offsets always are); rows outside every group are not
 * written. Being on the device it is not checked by the host, but every
 * kernel that reads it first clamps each entry into [0, rows] and raises it
 * to the largest entry before it, so a malformed array yields empty or
 * shortened groups and never a read or write outside x, y or the workspace.
 * The same holds for the group offsets of every grouped call below (expert
 * dgrad and wgrad, the FP8 GEMMs, the centroid gradient).
 *
 *   x      [rows, d] bf16, 16-B aligned.
 *   w13    [G, 2*inter, d] bf16, 16-B aligned: W1 and W3 of each group,
 *          row-interleaved in 16-row chunks ([W1 rows 0..15; W3 rows
 *          0..15; W1 rows 16..31; ...]); moe_pack_w13 builds it.
 *   w2     [G, d, inter] bf16, 16-B aligned.
 *   y      [rows, d] bf16 out, 16-B aligned.
 *   workspace >= moe_grouped_ffn_workspace_size(rows, inter, dtype): holds
 *          h = silu(x W1^T) * (x W3^T) as bf16 [rows, inter].
 * The shared expert(s) run as G = 1 with group_offsets = {0, T}, x = u and
 * the N_s shared experts' weights concatenated along inter.
 * dtype MOE_BF16: x, w13, w2 bf16; x_scales / w13_scales / w2_scales unused
 *   (pass NULL); workspace holds h as bf16 [rows, inter].
 * dtype MOE_FP8_E4M3: x, w13, w2 are E4M3 codes (1 byte) with fp32 scales
 *   x_scales [rows, d/128], w13_scales [G, 2, inter/128, d/128] (w13 packed by
 *   moe_pack_w13_fp8), w2_scales [G, d/128, inter/128] (see the FP8 section);
 *   y stays bf16; workspace holds h as E4M3 codes [rows, inter] + its
 *   scales [rows, inter/128] (quantised in the up-projection's epilogue).
 */
MOE_API int moe_grouped_ffn(const void* x, const float* x_scales, const int32_t* group_offsets,
                            int G, int rows, int d, int inter, const void* w13,
                            const float* w13_scales, const void* w2, const float* w2_scales,
                            moe_dtype dtype, void* y, void* workspace, size_t ws_bytes,
                            moe_stream_t stream);

MOE_API size_t moe_grouped_ffn_workspace_size(int rows, int inter, moe_dtype dtype);

/* moe_workspace_size: bytes of scratch one forward of the five calls needs if
 * its calls share one workspace (they run in stream order): the larger of
 * moe_permute_workspace_size(T, n_routed) and the grouped FFN's for the routed
 * rows (T*top_k, inter) and for the shared expert(s) (T, shared_inter). The
 * shared expert needs its own workspace if it runs beside the routed path on
 * another stream. d is accepted for symmetry with the other calls. */
MOE_API size_t moe_workspace_size(int T, int d, int n_routed, int top_k, int inter,
                                  int shared_inter, moe_dtype dtype);

/* The two halves of moe_grouped_ffn, for callers that keep h themselves.
 * moe_expert_up_swiglu:  h[rows, inter] = silu(x W1^T) * (x W3^T) per group.
 * moe_expert_down:       y[rows, d]     = h W2^T per group.
 * Same argument rules as moe_grouped_ffn; h is bf16, 16-B aligned. */
MOE_API int moe_expert_up_swiglu(const void* x, const int32_t* group_offsets, int G, int rows,
                                 int d, int inter, const void* w13, void* h,
                                 moe_stream_t stream);
/* moe_expert_up_swiglu_gather: moe_expert_up_swiglu whose x is not copied:
 * logical row r of x is row src_token[r] of u [T, d] (bf16, 16-B aligned),
 * read by the kernel itself (TMA gather, four rows per load). src_token,
 * group_offsets: from moe_permute_index. Removes the expert-contiguous copy
 * of the dispatch: the dispatch then moves no token rows. */
MOE_API int moe_expert_up_swiglu_gather(const void* u, int T, const int32_t* src_token,
                                        const int32_t* group_offsets, int G, int rows, int d,
                                        int inter, const void* w13, void* h,
                                        moe_stream_t stream);
MOE_API int moe_expert_down(const void* h, const int32_t* group_offsets, int G, int rows,
                            int inter, int d, const void* w2, void* y, moe_stream_t stream);

/* ------------------------------------------------------------------ FP8 variant
 * FP8 mixed precision of the technical report summary ("Main ideas", FP8
 * bullet): E4M3 operands, tile-wise 1x128 activation scaling, block-wise
 * 128x128 weight scaling, accumulation promoted to FP32 on the CUDA cores
 * every 128 elements of K; the scale of a tile or block is max|x| / 448
 * (block-quantisation pseudocode of "DeepSeek model architecture explained",
 * 448 = largest E4M3 value). Codes are decided in fp32: scale = amax / 448
 * (an all-zero tile gets 1) and x / scale are IEEE fp32 divisions, the
 * quotient is rounded to E4M3 to nearest-even, saturating at +-448. The
 * intermediate h is quantised in the up-projection's epilogue straight from
 * its fp32 value (it never goes to memory in a wider type).
 * E4M3 tensors are 1 byte per element, 16-B aligned; scales fp32, 4-B aligned.
 * The routing (moe_route) stays bf16: the expert indices must be exact.
 *
 * moe_quant_act_fp8: x [rows, cols] bf16 -> q [rows, cols] E4M3 and
 *   scales [rows, cols/128] (one per 1x128 tile). cols % 128 == 0.
 * moe_quant_weights_fp8: w [G, R, C] bf16 -> q [G, R, C] E4M3 and
 *   scales [G, R/128, C/128] (one per 128x128 block). R, C % 128 == 0.
 * moe_pack_w13_fp8: FP8 expert weights for the up-projection. Quantise W1 and
 *   W3 stacked as [G, 2, inter, d] (i.e. moe_quant_weights_fp8 with 2G groups:
 *   its scales [G, 2, inter/128, d/128] are the w13_scales the FP8 FFN takes),
 *   then pack the codes into w13 [G, 2*inter, d] with 64-row chunks
 *   interleaved (W1 rows 0..63, W3 rows 0..63, W1 rows 64..127, ...).
 *   inter % 64 == 0.
 * moe_permute_fp8: moe_permute with E4M3 rows out: each token's bf16 row of
 *   u [T, d] is quantised once (1x128 tiles, the rule above) and its codes
 *   and tile scales are written to each of its rows of x8 [T*top_k, d] and
 *   x_scales [T*top_k, d/128]; with u8 [T, d] and u_scales [T, d/128] given
 *   (both or neither), also to the token's own row there (the shared
 *   expert's input). Other arguments as moe_permute.
 * moe_expert_up_swiglu_fp8 / moe_expert_down_fp8: the two halves of
 *   moe_grouped_ffn in FP8. The first reads x8/x_scales and the packed w13 with
 *   w13_scales [G, 2, inter/128, d/128] and writes h = silu(a) * b quantised:
 *   codes h8 [rows, inter] (16-B aligned) and scales h_scales [rows,
 *   inter/128]; the second reads h8/h_scales and w2 with w2_scales [G, d/128,
 *   inter/128] and writes bf16 y.
 */
MOE_API int moe_quant_act_fp8(const void* x, int rows, int cols, void* q, float* scales,
                              moe_stream_t stream);
MOE_API int moe_quant_weights_fp8(const void* w, int G, int R, int C, void* q, float* scales,
                                  moe_stream_t stream);
MOE_API int moe_pack_w13_fp8(const void* w13_stacked, int G, int inter, int d, void* w13,
                             moe_stream_t stream);
MOE_API int moe_permute_fp8(const void* u, const int32_t* topk_idx, const int32_t* expert_counts,
                            int T, int d, int n_routed, int top_k, void* x8, float* x_scales,
                            void* u8, float* u_scales, int32_t* expert_offsets, int32_t* pos,
                            int32_t* src_token, void* workspace, size_t ws_bytes,
                            moe_stream_t stream);
MOE_API int moe_expert_up_swiglu_fp8(const void* x8, const float* x_scales,
                                     const int32_t* group_offsets, int G, int rows, int d,
                                     int inter, const void* w13, const float* w13_scales,
                                     void* h8, float* h_scales, moe_stream_t stream);
MOE_API int moe_expert_down_fp8(const void* h8, const float* h_scales,
                                const int32_t* group_offsets, int G, int rows, int inter, int d,
                                const void* w2, const float* w2_scales, void* y,
                                moe_stream_t stream);

/* ------------------------------------------------------------------ combine
 * out_t = residual_t + shared_t + sum_k topk_gate[t,k] * y_perm[pos[t,k]]
 * (the technical report's output equation h'_t). Sums in fp32, one rounding
 * to bf16; a gather per token, no atomics, deterministic.
 *
 *   y_perm     [T*top_k, d] bf16, 16-B aligned (moe_grouped_ffn output).
 *   pos        [T, top_k] int32 (moe_permute output; negative = skip).
 *   topk_gate  [T, top_k] fp32 (moe_route output).
 *   shared_out [T, d] bf16 or NULL (no shared expert).
 *   residual   [T, d] bf16 or NULL (the listing form without residual).
 *   out        [T, d] bf16 out, 16-B aligned. May alias residual.
 */
MOE_API int moe_combine(const void* y_perm, const int32_t* pos, const float* topk_gate,
                        const void* shared_out, const void* residual, int T, int d, int top_k,
                        void* out, moe_stream_t stream);

/* ------------------------------------------------------------------ fused scatter
 * The gate-weighted combine of the output equation h'_t (technical report
 * summary, Method §2) moved into the down-projection's epilogue: each routed
 * row leaves the GEMM already multiplied by its gate g_{i,t} and lands in the
 * row of its (token, slot) pair, so the combine only adds K rows that sit next
 * to each other. Deterministic: no atomics, the same fixed summation order.
 * One forward in this mode: moe_route, moe_permute, moe_slot_index,
 * moe_expert_up_swiglu, moe_expert_down_scatter, moe_combine_slots.
 *
 * moe_slot_index: dst_slot [rows] int32 out: dst_slot[pos[s]] = s for every
 *   pair s = t*top_k + k whose pos[s] (moe_permute's) lies in [0, rows); the
 *   other entries are set to -1. The inverse of pos.
 * moe_expert_down_scatter: moe_expert_down whose output row r goes to row
 *   dst_slot[r] of y_slots [T*top_k, d] bf16 (16-B aligned), multiplied in
 *   fp32 by topk_gate[dst_slot[r]] before the one bf16 rounding. Rows whose
 *   dst_slot lies outside [0, T*top_k) are not stored. Other arguments as
 *   moe_expert_down.
 * moe_combine_slots: out_t = residual_t + shared_t + sum over the slots k
 *   with pos[t,k] >= 0 of y_slots[t*top_k + k] (fp32 sums in slot order, one
 *   bf16 rounding). Arguments as moe_combine without topk_gate.
 */
MOE_API int moe_slot_index(const int32_t* pos, int T, int top_k, int rows, int32_t* dst_slot,
                           moe_stream_t stream);
MOE_API int moe_expert_down_scatter(const void* h, const int32_t* group_offsets, int G, int rows,
                                    int inter, int d, const void* w2, const int32_t* dst_slot,
                                    const float* topk_gate, int T, int top_k, void* y_slots,
                                    moe_stream_t stream);
MOE_API int moe_combine_slots(const void* y_slots, const int32_t* pos, const void* shared_out,
                              const void* residual, int T, int d, int top_k, void* out,
                              moe_stream_t stream);

/* moe_expert_down_scatter_combine: moe_expert_down_scatter followed, inside
 * the same kernel, by moe_combine_slots: the store that completes a token's
 * top_k slot rows over a block of 128 output features (a count per token and
 * block in the workspace) adds them to residual and shared_out and writes
 * out, with moe_combine_slots' arithmetic (fp32 in the order residual,
 * shared, slots 0..top_k-1; one bf16 rounding), so the two give the same
 * bits. y_slots is still written (the rows are read back from it).
 *   shared_out, residual  [T, d] bf16 or NULL, 16-B aligned; complete before
 *              the call is ordered on the stream (they are read during it).
 *   out        [T, d] bf16 out, 16-B aligned; must not alias y_slots.
 *   workspace  device scratch, 16-B aligned, at least
 *              moe_expert_down_scatter_combine_workspace_size(T, d) bytes
 *              (the counts, zeroed by the call); caller-owned. NULL or too
 *              small -> MOE_ERR_WORKSPACE.
 * Every (token, slot) pair must have a row (dst_slot covers all T*top_k
 * slots, as moe_permute + moe_slot_index give): a token with a slot that no
 * row maps to never completes, and its out row is not written. top_k <=
 * 8. Other arguments and errors as moe_expert_down_scatter.
 */
MOE_API size_t moe_expert_down_scatter_combine_workspace_size(int T, int d);
MOE_API int moe_expert_down_scatter_combine(const void* h, const int32_t* group_offsets, int G,
                                            int rows, int inter, int d, const void* w2,
                                            const int32_t* dst_slot, const float* topk_gate,
                                            int T, int top_k, void* y_slots,
                                            const void* shared_out, const void* residual,
                                            void* out, void* workspace, size_t ws_bytes,
                                            moe_stream_t stream);

/* ------------------------------------------------------------------ bias update
 * Auxiliary-loss-free balancing (technical report summary, Method §2): at the
 * end of a step, b_i <- b_i - gamma if expert i is overloaded and
 * b_i <- b_i + gamma if it is underloaded. Load is compared with the mean
 * T*top_k/n_routed exactly in integers (n_routed*c_i vs T*top_k); an expert
 * exactly at the mean is unchanged. bias is fp32 state, updated in place.
 * For data-parallel use, pass counts already summed over all ranks and the
 * global T.
 */
MOE_API int moe_bias_update(const int32_t* expert_counts, float* bias, int n_routed,
                            long long T, int top_k, float gamma, moe_stream_t stream);

/* ------------------------------------------------------------------ backward
 * The gradient of the layer forward above ("DeepSeek-V3 technical report",
 * Method §2, and the softmax-over-top-k variant of "DeepSeek model
 * architecture explained"). The pages give no backward equations and say
 * only that gradients are computed in BF16: these calls compute the exact
 * derivative of the forward with the top-K selection held fixed (no gradient
 * reaches the bias, which only selects), bf16 tensors in and out, fp32
 * accumulation. The calls of one backward step, in order:
 *
 *   forward (training)  moe_expert_up_swiglu_train also keeps ac
 *   1 moe_combine_backward      dgate, dy_perm          (from dout, y_perm)
 *   2 moe_expert_down_backward  dac = SwiGLU'(dy W2)     (routed; shared: G = 1)
 *   3 moe_expert_up_backward    dx = dac W13
 *   4 moe_expert_wgrad          dW2 = dy^T h,  dW13 = dac^T x
 *   5 moe_gate_backward         dz (selected logits), dz_perm
 *   6 moe_combine_dx            du
 *   7 moe_centroid_grad         de
 *
 * Shapes as for moe_grouped_ffn (d % 256 == 0, inter % 128 == 0, G <= 1024);
 * all tensors row-major, 16-B aligned, caller-owned; asynchronous on
 * `stream`; errors as for the forward calls.
 *
 * moe_expert_up_swiglu_train: moe_expert_up_swiglu that also writes the
 * pre-activations ac [rows, 2*inter] bf16 (x W13^T, in the packed W13 column
 * order: 16 columns of x W1^T, then the same 16 of x W3^T, ...), which the
 * backward of the SwiGLU needs. */
MOE_API int moe_expert_up_swiglu_train(const void* x, const int32_t* group_offsets, int G,
                                       int rows, int d, int inter, const void* w13, void* h,
                                       void* ac, moe_stream_t stream);

/* moe_combine_backward: for the routed term sum_k g_{t,k} y_{t,k} of h'_t,
 *   dgate[t,k] = dout_t . y_perm[pos[t,k]]   fp32 [T, top_k]
 *   dy_perm[pos[t,k]] = topk_gate[t,k] * dout_t   bf16 [T*top_k, d]
 * dout, y_perm, dy_perm bf16; pos, topk_gate as written by the forward. */
MOE_API int moe_combine_backward(const void* dout, const void* y_perm, const int32_t* pos,
                                 const float* topk_gate, int T, int d, int top_k, void* dy_perm,
                                 float* dgate, moe_stream_t stream);

/* moe_expert_down_backward: per group g, dh = dy W2_g ([rows, d] x [d, inter])
 * and the SwiGLU backward with the saved ac: da = dh * c * silu'(a),
 * dc = dh * silu(a), written as dac [rows, 2*inter] in ac's column order. */
MOE_API int moe_expert_down_backward(const void* dy, const void* ac, const int32_t* group_offsets,
                                     int G, int rows, int d, int inter, const void* w2, void* dac,
                                     moe_stream_t stream);

/* moe_expert_up_backward: per group g, dx = dac W13_g ([rows, 2*inter] x
 * [2*inter, d], the packed w13 of the forward), dx [rows, d] bf16. */
MOE_API int moe_expert_up_backward(const void* dac, const int32_t* group_offsets, int G,
                                   int rows, int d, int inter, const void* w13, void* dx,
                                   moe_stream_t stream);

/* moe_expert_wgrad: per group g, dw[g] = a[rows of g]^T b[rows of g], the
 * contraction over the group's rows; a [rows, m], b [rows, n] bf16, dw
 * [G, m, n] bf16 (overwritten; zero for a group without rows). m % 128 == 0,
 * n % 128 == 0. dW2 = moe_expert_wgrad(dy, h, m = d, n = inter); the packed
 * dW13 = moe_expert_wgrad(dac, x, m = 2*inter, n = d). Rows of a and b
 * outside every group but below `rows` must hold finite values. */
MOE_API int moe_expert_wgrad(const void* a, const void* b, const int32_t* group_offsets, int G,
                             int rows, int m, int n, void* dw, moe_stream_t stream);

/* moe_gate_backward: dL/dz of each selected logit z_{t,idx} = u_t . e_idx
 * from dgate. Sigmoid gate (g_k = S s_k / sum_j s_j, s = Sigmoid(z)
 * recomputed here from u and the centroids): dz_k = S/sum (dg_k - sum_j dg_j
 * s_j / sum) s_k (1 - s_k). Softmax gate (g = S softmax of the selected z):
 * dz_k = g_k (dg_k - sum_j g_j dg_j / S). dz fp32 [T, top_k]; dz_perm fp32
 * [T*top_k] receives dz[t,k] at row pos[t,k]. */
MOE_API int moe_gate_backward(const void* u, const void* centroids, const int32_t* topk_idx,
                              const float* topk_gate, const float* dgate, const int32_t* pos,
                              int T, int d, int n_routed, int top_k, moe_gate_kind kind,
                              float routed_scale, float* dz, float* dz_perm,
                              moe_stream_t stream);

/* moe_combine_dx: du_t = dout_t (residual; dout may be NULL for the form
 * without it) + dx_shared_t (may be NULL) + sum_k dx_perm[pos[t,k]]
 * + sum_k dz[t,k] e_{topk_idx[t,k]}, bf16 [T, d]. */
MOE_API int moe_combine_dx(const void* dout, const void* dx_perm, const int32_t* pos,
                           const void* dx_shared, const float* dz, const int32_t* topk_idx,
                           const void* centroids, int T, int d, int top_k, void* du,
                           moe_stream_t stream);

/* moe_centroid_grad: de_i = sum over the rows r of expert i of dz_perm[r] *
 * x_perm[r] (x_perm row r = u of the token routed there), bf16 [n_routed, d].
 * The rows are summed in chunks of 128 (so that a hot expert spreads over
 * many blocks), then the chunks in order: the result is reproducible.
 * workspace >= moe_centroid_grad_workspace_size(rows, n_routed, d) bytes,
 * 16-B aligned. n_routed < 1024. */
MOE_API int moe_centroid_grad(const void* x_perm, const float* dz_perm,
                              const int32_t* expert_offsets, int n_routed, int rows, int d,
                              void* de, void* workspace, size_t ws_bytes, moe_stream_t stream);
MOE_API size_t moe_centroid_grad_workspace_size(int rows, int n_routed, int d);

/* ------------------------------------------------------------------ expert parallelism
 * The routed experts split evenly over W ranks: rank p holds experts
 * [p*n_local, (p+1)*n_local), n_routed = W*n_local; the centroids, the bias
 * and the shared expert are replicated. Token rows travel by all-to-all
 * exchanges (DeepSeek-V3 technical report summary: "Problem setting and
 * motivation", the all-to-all cost of fine-grained routing; "Main ideas",
 * DualPipe bullet). One forward on each rank:
 *   moe_route, moe_permute (local tokens, all n_routed experts)
 *   counts exchange: rank p receives, from every rank q, the counts of q's
 *     rows for p's n_local experts -> recv_counts [W, n_local]
 *   moe_ep_plan (host)
 *   dispatch exchange: x_perm rows [offsets[p*n_local], offsets[(p+1)*n_local])
 *     go to rank p (send_splits[p] rows); recv_splits[q] rows arrive from q
 *   moe_gather_rows(x_recv, n_recv, regroup, n_recv, d, x_exp)
 *   moe_expert_up_swiglu(x_exp, group_offsets, n_local, n_recv, ...),
 *     moe_expert_down(..., y_exp)   (or moe_expert_up_swiglu_gather on
 *     x_recv with regroup as src_token, which skips the copy but is slower)
 *   moe_gather_rows(y_exp, n_recv, ungroup, n_recv, d, y_src)
 *   return exchange: y_src back with the splits swapped -> y_perm
 *   moe_combine (local tokens), as for one GPU.
 * The collectives are the caller's (NCCL in the binding).
 *
 * moe_ep_plan: HOST function on host arrays; launches nothing, touches no
 * device, may be called without a GPU.
 *   local_counts [W*n_local] int32: this rank's rows per expert (its
 *     moe_route counts).
 *   recv_counts [W, n_local] int32: recv_counts[q*n_local + e] = rows that
 *     rank q routes to this rank's local expert e.
 *   Out: send_splits[W], recv_splits[W] (rows to / from each rank);
 *     group_offsets [n_local+1] int32: expert-major offsets of the received
 *     rows; *n_recv = their number R. regroup [R] int32: for expert-major row
 *     j (expert e's rows from rank 0, then rank 1, ...; each rank's rows in
 *     its token order), its row in the received (source-major) buffer;
 *     ungroup [R] int32: the inverse. regroup/ungroup may be NULL (splits,
 *     offsets and R only); otherwise R must be <= recv_capacity.
 *   Errors: MOE_ERR_INVALID_ARG for a NULL required pointer, W or n_local
 *   < 1, a negative count, or R > recv_capacity with regroup/ungroup given;
 *   MOE_ERR_UNSUPPORTED_SHAPE for R >= 2^31. Nothing is written on error.
 *
 * moe_gather_rows: dst[i, :] = src[index[i], :] for i < n (bf16 rows of d
 *   elements; src [n_src, d], dst [n, d], 16-B aligned, d % 8 == 0; index
 *   [n] int32 device). An index outside [0, n_src) yields a zero row (src is
 *   never read out of bounds). HBM-bound: reads and writes n*d*2 bytes.
 */
MOE_API int moe_ep_plan(const int32_t* local_counts, const int32_t* recv_counts, int world,
                        int n_local, long long recv_capacity, long long* send_splits,
                        long long* recv_splits, int32_t* group_offsets, int32_t* regroup,
                        int32_t* ungroup, long long* n_recv);
MOE_API int moe_gather_rows(const void* src, int n_src, const int32_t* index, int n, int d,
                            void* dst, moe_stream_t stream);

/* ------------------------------------------------------------------ expert parallelism over peer memory
 * The same split of the experts over W ranks, with the token rows moved by
 * this library's own kernels through peer memory instead of all-to-all
 * collectives, and every step planned on the device (no host read):
 *   moe_route, moe_permute_index        this rank's tokens (no row copy)
 *   all-gather of the loads             all_counts [W, n_routed] int32 (the
 *                                       caller's collective, e.g. NCCL)
 *   moe_ep_plan_device                  where this rank's rows go
 *   moe_ep_dispatch_p2p                 rows stored into the owners' buffers
 *   barrier (caller)                    every rank's stores have landed
 *   moe_expert_up_swiglu, moe_expert_down   on x_recv, G = n_local, rows =
 *                                       its capacity, the plan's offsets
 *   barrier (caller)                    every owner's outputs are written
 *   moe_ep_combine_p2p                  each token's K outputs read back
 *   moe_bias_update(global_counts, ..., T summed over the ranks)
 * Rank q's receive buffer x_recv [capacity, d] is expert-major: expert e's
 * rows from rank 0, then from rank 1, ..., each in that rank's token order
 * (the order one GPU's stable dispatch gives the ranks' batches laid end to
 * end), so the result equals the single-GPU layer on that batch. The
 * buffers of the other ranks are reached through peer pointers (CUDA IPC,
 * moe_ipc_*); with one rank they are local. Plain peer loads and stores, no
 * TMA multicast.
 *
 * moe_ep_plan_device: one small kernel. all_counts [world, world*n_local]
 *   (row q = rank q's moe_route counts); writes dest_row [n_routed] (first row
 *   of this rank's rows for expert E in its owner's receive buffer),
 *   group_offsets [n_local + 1] (this rank's own receive buffer, expert-major)
 *   and global_counts [n_routed] (the loads summed over the ranks, plus
 *   add_counts [n_routed] when it is not NULL: an earlier micro-batch's
 *   global_counts, so that the last one holds the step's). A receive
 *   buffer that would need more than recv_capacity rows sets bit 16 of the
 *   device status word (moe_get_device_status then returns
 *   MOE_ERR_DEVICE_TIMEOUT); the rows past the capacity are not moved.
 *   world * n_local <= 256.
 * moe_ep_dispatch_p2p: token t's row of u goes to row dest_row[E] + pos[t,k]
 *   - expert_offsets[E] of peer_x[E / n_local], for each slot k with E =
 *   topk_idx[t,k]. peer_x: DEVICE array of `world` pointers to the ranks'
 *   receive buffers [recv_capacity, d] bf16 (16-B aligned), as mapped on this
 *   GPU. pos, expert_offsets: moe_permute_index's.
 * moe_ep_combine_p2p: moe_combine whose routed rows are read from
 *   peer_y[E / n_local] at the rows the dispatch wrote (peer_y: DEVICE array
 *   of `world` pointers to the ranks' expert output buffers [recv_capacity,
 *   d] bf16). out may alias residual.
 * moe_ipc_get_handle: the 64-byte CUDA IPC handle of the allocation that
 *   holds dev_ptr, and dev_ptr's byte offset in it (the allocation must come
 *   from cudaMalloc, e.g. PyTorch's default caching allocator; memory from
 *   the virtual-memory API, such as expandable segments, has no such handle
 *   and the call returns MOE_ERR_CUDA). moe_ipc_open_handle maps a handle
 *   from another process on this GPU (*base = the allocation's start; add
 *   the offset); moe_ipc_close_handle unmaps it.
 */
MOE_API int moe_ep_plan_device(const int32_t* all_counts, int world, int n_local, int rank,
                               long long recv_capacity, const int32_t* add_counts,
                               int32_t* dest_row, int32_t* group_offsets,
                               int32_t* global_counts, moe_stream_t stream);
MOE_API int moe_ep_dispatch_p2p(const void* u, const int32_t* topk_idx, const int32_t* pos,
                                const int32_t* expert_offsets, const int32_t* dest_row, int T,
                                int d, int n_routed, int top_k, int world, void* const* peer_x,
                                long long recv_capacity, moe_stream_t stream);
MOE_API int moe_ep_combine_p2p(const void* const* peer_y, const int32_t* topk_idx,
                               const int32_t* pos, const int32_t* expert_offsets,
                               const int32_t* dest_row, const float* topk_gate,
                               const void* shared_out, const void* residual, int T, int d,
                               int n_routed, int top_k, int world, long long recv_capacity,
                               void* out, moe_stream_t stream);
MOE_API int moe_ipc_get_handle(const void* dev_ptr, void* handle, long long* offset);
MOE_API int moe_ipc_open_handle(const void* handle, void** base);
MOE_API int moe_ipc_close_handle(void* base);

/* ------------------------------------------------------------------ helpers
 * moe_pack_w13: build the interleaved w13 [G, 2*inter, d] from w1 and w3
 * [G, inter, d] (all bf16, 16-B aligned; layout described at moe_grouped_ffn).
 */
MOE_API int moe_pack_w13(const void* w1, const void* w3, int G, int inter, int d, void* w13,
                         moe_stream_t stream);

/* Human-readable name of a status code (static storage). */
MOE_API const char* moe_strerror(int status);

/* The CUDA error code behind the calling thread's last MOE_ERR_CUDA (0 if none). */
MOE_API int moe_last_cuda_error(void);

/* Synchronises the current device, then writes the device status word of the
 * current device to *status; clears it if `clear`. Bits: 1, 2, 4 a pipeline
 * wait of a GEMM ran out (producer, MMA, epilogue), 8 the self-test below,
 * 16 an expert-parallel receive buffer was too small. 0 = none of these.
 * Returns MOE_ERR_DEVICE_TIMEOUT if the word was non-zero. */
MOE_API int moe_get_device_status(unsigned int* status, int clear);

/* Diagnostic for the failure-detection path: enqueues a one-thread kernel that
 * waits on a barrier nothing will complete, gives up after limit_ms
 * (1..10000) the way every pipeline wait of the library does, and ORs 8
 * into the device status word; moe_get_device_status() then
 * returns MOE_ERR_DEVICE_TIMEOUT. The device context stays usable. No
 * counterpart in the pages. */
MOE_API int moe_selftest_wait_timeout(int limit_ms, moe_stream_t stream);

/* Library version, major*10000 + minor*100 + patch. 0.2.0 (200) added, over
 * the forward's five calls of 0.1.0: the FP8 variant, the fused-gather
 * up-projection, the backward and the expert-parallel entry points. 0.3.0
 * (300): the fused scatter, expert parallelism over peer memory, the FP8
 * dispatch and up-projection quantising in place (their signatures
 * changed), device-side clamping of group offsets. */
MOE_API int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
