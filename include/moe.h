/*
 * libmoe -- forward pass of a DeepSeek-V3 / DeepSeek-V2-Lite mixture-of-experts
 * layer on one NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages state it:
 *   [MoE-walk]    zhiyuanblog.org "MoE 混合专家模型推理参数与前向传播详解":
 *                 §2.1 router, §2.2 stacked expert weights, §2.3 merged shared
 *                 experts, §3.1 routing, §3.2 token permutation, §3.3 grouped
 *                 SwiGLU experts and shared experts, §3.4 unpermute + combine.
 *   [V3-teardown] gsyq.cn "为什么要在本地拆解 DeepSeek-V3 的 MoE 与 MLA":
 *                 §3 router config (n_group, topk_group, norm_topk_prob,
 *                 routed_scaling_factor, sigmoid scoring; FP8 128x128 weight
 *                 blocks, dynamic activations), §4 route() and the load CV.
 *   [V3-digest]   xxqk.cn DeepSeek V3/R1/Janus-Pro digest, §2.2 aux-loss-free
 *                 bias and device-limited (group-limited) routing.
 *   [FP8-infer]   blog.hotdry.top DeepSeek-V3 FP8 inference post, FP8 section
 *                 (E4M3, 1x128 activation tiles, 128x128 weight blocks).
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers to dense row-major arrays, allocated
 *     and owned by the caller. The library allocates no memory. Its only
 *     mutable global state is the per-thread moe_last_cuda_error and the
 *     process-wide wait limit of moe_set_wait_limit_ns (a debugging knob,
 *     2 s unless changed); moe_permute_static_ws keeps its own array.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *     legacy default stream). Outputs are valid once the stream reaches it.
 *   - Arguments are checked on the host before any launch. On a non-OK
 *     return nothing has been launched or written, except MOE_ERR_CUDA,
 *     which reports a launch failure (see moe_last_cuda_error).
 *   - Every device pointer must be 16-byte aligned (MOE_ERR_ALIGNMENT).
 *   - `dev_status`, where taken, is an optional device int32 (NULL = off).
 *     Kernels never trap: a bounds check that fails or a bounded wait that
 *     runs out ORs a code into it (MOE_DEVSTAT_*) and the kernel returns.
 *     Read it with moe_read_device_status. After a wait runs out, the
 *     kernel's outputs are incomplete, but the CUDA context stays usable.
 *   - No C++ exception crosses this interface.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

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

#define MOE_ABI_VERSION 3

typedef int32_t moe_status;
#define MOE_OK                 0
#define MOE_ERR_INVALID_ARG    1  /* null pointer, bad size, k > E, ...      */
#define MOE_ERR_UNSUPPORTED    2  /* shape / dtype combination not built      */
#define MOE_ERR_ALIGNMENT      3  /* a pointer is not 16-byte aligned         */
#define MOE_ERR_CUDA           4  /* a CUDA launch or driver call failed      */
#define MOE_ERR_DEVICE_CHECK   5  /* device status: a bounds check failed     */
#define MOE_ERR_DEVICE_TIMEOUT 6  /* device status: a bounded wait ran out    */

/* bits ORed into *dev_status by kernels */
#define MOE_DEVSTAT_BAD_EXPERT_ID 0x1 /* a topk id outside [0, E)            */
#define MOE_DEVSTAT_TIMEOUT       0x2 /* an mbarrier wait exceeded its limit */

typedef int32_t moe_dtype;
#define MOE_F32  0
#define MOE_BF16 1
#define MOE_E4M3 2   /* float8 e4m3 "fn": bias 7, max 448, no inf */

typedef int32_t moe_scoring;
#define MOE_SOFTMAX 0
#define MOE_SIGMOID 1

/* ------------------------------------------------------------------------ *
 * moe_route -- gate projection + scoring + group-limited top-k + weights.
 * [MoE-walk] §2.1 and §3.1; [V3-teardown] §3-§4 route(); [V3-digest] §2.2.
 *
 *   logits = x @ gate^T                       (bf16 inputs, fp32 accumulate)
 *   scoring  softmax: p = softmax(logits) over all E experts
 *            sigmoid: s = sigmoid(logits)
 *   selection score  sel = s + sel_bias (sigmoid), p (softmax with groups or
 *            a bias), the logit itself (softmax, one group, no bias). The
 *            sigmoid and softmax are evaluated in double and rounded once to
 *            float; the bias add is one float add.
 *   if n_group > 1: experts [g*E/n_group, (g+1)*E/n_group) form group g; a
 *            group's score is the float sum of its two largest sel; only the
 *            topk_group best groups stay candidates (ties: lower group index).
 *   topk_ids = the k best sel among candidates, in slot order sel descending,
 *            expert index ascending (ties: lower expert index).
 *   topk_w   = unbiased s (or p) of those experts; if norm_topk_prob they are
 *            divided by their sum; then multiplied by routed_scaling_factor.
 *   expert_counts[e] = number of (t, j) with topk_ids[t][j] == e (zeroed by
 *            the call first).
 *
 * Arguments
 *   p             shapes and routing config (host pointer, read during call).
 *   x             [T, H] bf16, or NULL: then `logits` is an INPUT [T, E] fp32
 *                 and routing runs on those logits (no projection).
 *   gate_w        [E, H] bf16 (ignored when x == NULL).
 *   sel_bias      [E] fp32 selection-only bias, or NULL (= 0).
 *   logits        [T, E] fp32, required: written when x != NULL, read when
 *                 x == NULL.
 *   topk_ids      [T, k] int32 out;  topk_w [T, k] fp32 out.
 *   expert_counts [E] int32 out.
 * Work: with x, a tcgen05 gate GEMM on clusters of 2, 4 or 8 CTAs per 128
 * tokens (each CTA sums one slice of the hidden size; every logit is the
 * slices' partial sums added in order; the split depends on T and the SM
 * count only, so moe_gate_logits gives the same logits) and, in the same
 * launch where the shape allows (E = 8C, C in {2,4,8,16,32}, n_group | 8,
 * k <= 8), the routing of every token, eight threads per token. With
 * x == NULL, or from x for other shapes, the routing is its own launch
 * (eight threads per token where the shape allows, else one warp per token;
 * the same decisions either way).
 * Limits: 1 <= k <= 16, E % 16 == 0, 16 <= E <= 256, E % n_group == 0,
 *   n_group <= 32, topk_group <= n_group, k <= topk_group * E / n_group,
 *   H % 64 == 0 when x != NULL. Otherwise MOE_ERR_INVALID_ARG/UNSUPPORTED.
 * A token none of whose candidate experts has a score that compares (all
 *   NaN; with n_group > 1 the dropped groups' experts score -inf and still
 *   compare) gets ids -1 and weights 0, is counted nowhere, and flags
 *   MOE_DEVSTAT_BAD_EXPERT_ID in p->dev_status.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t T, H, E, k;
    int32_t n_group, topk_group;
    moe_scoring scoring;
    int32_t norm_topk_prob;          /* 0 / 1 */
    float routed_scaling_factor;
    int32_t* dev_status;             /* optional device status word */
} moe_route_params;

MOE_API moe_status moe_route(const moe_route_params* p, const void* x, const void* gate_w,
                     const float* sel_bias, float* logits, int32_t* topk_ids,
                     float* topk_w, int32_t* expert_counts, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_gate_logits -- the gate projection of moe_route alone.
 * [MoE-walk] §2.1: router_logits = hidden_states @ gate.weight^T.
 *
 *   logits [T, E] fp32 out = x [T, H] bf16 @ gate_w [E, H] bf16 ^T, computed
 *   exactly as moe_route computes them (same kernel, same summation order).
 * Followed by moe_route with x = NULL on the same logits it is moe_route in
 * two calls, so that other work (another stream's launch) can be ordered
 * between the projection and the routing.
 * Limits: H % 64 == 0, H >= 64, E % 16 == 0, 16 <= E <= 256.
 * dev_status: optional device status word (bounded waits report into it).
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_gate_logits(int32_t T, int32_t H, int32_t E, const void* x, const void* gate_w,
                                   float* logits, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_permute -- expand every token k times and order the copies by expert.
 * [MoE-walk] §3.2 and its worked example: segment e holds the tokens routed
 * to expert e in ASCENDING TOKEN ORDER; expert_offsets is
 * expert_first_token_offset with E + 1 entries (empty experts repeat).
 *
 *   expert_offsets [E+1] int32 out, expert_offsets[E] = T*k
 *   src_token      [T*k] int32 out, row -> token
 *   slot_to_row    [T*k] int32 out, t*k + j -> row (inv_permuted_idx)
 *   row_w          [T*k] fp32 out,  topk_w[t][j] at row slot_to_row[t*k+j]
 *                  (may be NULL, then topk_w may be NULL too)
 *   x / x_perm     x_dtype -> perm_dtype:
 *                  BF16 -> BF16: x [T, H] bf16 -> x_perm [T*k, H] bf16.
 *                  BF16 -> E4M3: x [T, H] bf16 is quantised here, per 1x128
 *                    tile along H ([FP8-infer] 1x128 activation tiles,
 *                    dynamic; the bytes of moe_quantize_rows): x_perm
 *                    [T*k, H] codes and x_perm_scale [T*k, H/128]; x_q /
 *                    x_q_scale [T, H] / [T, H/128] (optional, both or
 *                    neither) also receive the token's own codes and scales
 *                    (the shared expert's operand). H % 128 == 0.
 *                  E4M3 -> E4M3: x [T, H] codes with x_scale [T, H/128] ->
 *                    x_perm [T*k, H] codes and x_perm_scale [T*k, H/128].
 *                  E4M3 -> BF16 is MOE_ERR_UNSUPPORTED. x_q / x_q_scale are
 *                  NULL unless quantising. x_perm may be NULL (metadata,
 *                  and x_q if given, only).
 *   workspace      device scratch of moe_permute_workspace_size() bytes.
 * topk_ids outside [0, E) are counted nowhere and flag
 * MOE_DEVSTAT_BAD_EXPERT_ID in dev_status (outputs are then undefined).
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_permute_workspace_size(int32_t T, int32_t k, int32_t E, size_t* bytes);

MOE_API moe_status moe_permute(int32_t T, int32_t k, int32_t E, int32_t H,
                       const int32_t* topk_ids, const float* topk_w,
                       const void* x, moe_dtype x_dtype, const float* x_scale,
                       void* x_perm, moe_dtype perm_dtype, float* x_perm_scale,
                       void* x_q, float* x_q_scale,
                       int32_t* expert_offsets, int32_t* src_token,
                       int32_t* slot_to_row, float* row_w,
                       void* workspace, size_t workspace_bytes,
                       int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_permute_static_ws -- moe_permute without a caller-provided workspace.
 * The pages have no counterpart: this is a library convenience.
 *
 * For callers that cannot allocate device memory where they call the
 * permutation: code whose device memory all belongs to a framework allocator
 * and must not be taken around it, code that must not risk the implicit
 * device synchronisation a cudaMalloc can cause, and plugin interfaces that
 * hand in only input and output buffers. Arguments, outputs and errors are
 * those of moe_permute with perm_dtype = x_dtype and no x_q / x_q_scale,
 * minus `workspace` / `workspace_bytes`.
 *
 * The scratch is a 1 MiB array in the library's own device memory (every GPU
 * that loads the library holds it until the process exits). It fits
 * ceil(T / 64) * E <= 262144, e.g. T <= 65536 tokens with E = 256; larger
 * T, E return MOE_ERR_UNSUPPORTED before anything is launched. No memory is
 * allocated. The first call on a device looks up the array's address for
 * that device (cudaGetSymbolAddress), so make that first call before any
 * stream capture. All calls share the one array: calls whose work overlaps
 * on the GPU (other streams, other host threads) race and give wrong
 * results; serialise them. Nothing needs clearing between calls (every call
 * rewrites the part of the array it reads).
 * The looked-up address is cached per device index for the life of the
 * process: after cudaDeviceReset (or anything else that destroys and
 * recreates the device's primary context) it is stale, and the next call
 * would write through it. Do not call this entry point again in a process
 * that has reset the device.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_permute_static_ws(int32_t T, int32_t k, int32_t E, int32_t H,
                       const int32_t* topk_ids, const float* topk_w,
                       const void* x, moe_dtype x_dtype, const float* x_scale,
                       void* x_perm, float* x_perm_scale,
                       int32_t* expert_offsets, int32_t* src_token,
                       int32_t* slot_to_row, float* row_w,
                       int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_grouped_swiglu -- SwiGLU experts over contiguous row segments.
 * [MoE-walk] §3.3.1 (w13 = [w1; w3], gate = first I outputs, up = last I,
 * h = SiLU(gate) * up, out = h @ w2^T) and the grouped GEMM of the same
 * section (one launch for all experts, segmented by expert offsets);
 * §3.3.2 / §2.3 shared experts (merged into one FFN: call with offsets = NULL).
 *
 *   rows      number of activation rows (T*k routed, T shared).
 *   H         hidden size (K of the first GEMM, N of the second).
 *   w         weights: w13 [groups, 2I, H], w2 [groups, H, I] (out-major,
 *             i.e. K contiguous), or, bf16 with w->tiled = 1, the same
 *             values in the tiled layout moe_tile_ffn_weights writes.
 *             MOE_E4M3 weights carry fp32 block scales
 *             w13_scale [groups, 2I/128, H/128], w2_scale [groups, H/128,
 *             I/128] (moe_quantize_blocks).
 *   a         [rows, H] activations: bf16, or e4m3 codes with a_scale
 *             [rows, H/128] when w->dtype == MOE_E4M3.
 *   offsets   [groups+1] device int32 segment starts (from moe_permute), or
 *             NULL: one group covering all rows (groups must be 1).
 *   row_w     [rows] fp32 per-row output weight fused into the epilogue of
 *             the second GEMM, or NULL (= 1).
 *   h_ws      [rows, I] intermediate: bf16, or e4m3 codes with h_scale_ws
 *             [rows, I/128] for MOE_E4M3 (re-quantised per 1x128 tile).
 *   out       [rows, H] bf16 = row_w * (SiLU(a w1^T) * (a w3^T)) w2^T.
 * Limits: I % 128 == 0, H % 256 == 0, rows >= 1. E4M3 also needs H % 128
 * and I % 128. Accumulation is fp32 on the tensor cores; h is rounded to
 * bf16 (or quantised to e4m3) before the second GEMM.
 * ------------------------------------------------------------------------ */
typedef struct {
    const void* w13;
    const void* w2;
    const float* w13_scale;   /* E4M3 only, else NULL */
    const float* w2_scale;    /* E4M3 only, else NULL */
    moe_dtype dtype;          /* MOE_BF16 or MOE_E4M3 */
    int32_t groups;
    int32_t I;
    int32_t tiled;            /* bf16 only: 1 = w13 / w2 in the tiled layout, 0 = row-major */
} moe_ffn_weights;

MOE_API moe_status moe_grouped_swiglu(int32_t rows, int32_t H, const moe_ffn_weights* w,
                              const void* a, const float* a_scale,
                              const int32_t* offsets, const float* row_w,
                              void* h_ws, float* h_scale_ws, void* out,
                              int32_t* dev_status, void* stream);

/* The two halves of moe_grouped_swiglu, for callers that schedule or time
 * them separately (same arguments and limits as above):
 *   moe_gate_up_swiglu: h_ws = SiLU(a w1^T) * (a w3^T)        (w13 only)
 *   moe_down_proj:      out  = row_w * (h w2^T), h given as  (w2 only)
 *                       h [rows, I] (+ h_scale [rows, I/128] for E4M3). */
MOE_API moe_status moe_gate_up_swiglu(int32_t rows, int32_t H, const moe_ffn_weights* w,
                              const void* a, const float* a_scale,
                              const int32_t* offsets, void* h_ws, float* h_scale_ws,
                              int32_t* dev_status, void* stream);
MOE_API moe_status moe_down_proj(int32_t rows, int32_t H, const moe_ffn_weights* w,
                         const void* h, const float* h_scale, const int32_t* offsets,
                         const float* row_w, void* out, int32_t* dev_status, void* stream);

/* The routed experts and the shared expert in one launch per GEMM ([MoE-walk]
 * §3.3: the routed experts as one grouped GEMM, the merged shared expert as
 * one more group of all T rows), so the shared expert's tiles and the routed
 * experts' ragged tiles share the persistent CTAs instead of each launch
 * ending on its own partly idle last wave:
 *   moe_gate_up_swiglu_with_shared: h_ws = SwiGLU of (a, w13) per segment
 *       of offsets, and sh_h_ws = SwiGLU of (sh_a, sw13);
 *   moe_down_proj_with_shared: out = row_w * (h w2^T) per segment, and
 *       sh_out = sh_h sw2^T (weight 1).
 * w: routed weights (groups = E), sw: shared weights (groups must be 1, same
 * dtype; its I may differ from w's). rows / sh_rows: T*k / T. Other
 * arguments, limits and errors as moe_gate_up_swiglu / moe_down_proj; E4M3
 * scales as there (sh_a_scale / sh_h_scale for the shared rows). bf16 layers
 * run as one launch; E4M3 layers as two launches of the same calls in this
 * order. */
MOE_API moe_status moe_gate_up_swiglu_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w,
                              const void* a, const float* a_scale, const int32_t* offsets,
                              void* h_ws, float* h_scale_ws,
                              int32_t sh_rows, const moe_ffn_weights* sw,
                              const void* sh_a, const float* sh_a_scale,
                              void* sh_h_ws, float* sh_h_scale_ws,
                              int32_t* dev_status, void* stream);
MOE_API moe_status moe_down_proj_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w,
                              const void* h, const float* h_scale, const int32_t* offsets,
                              const float* row_w, void* out,
                              int32_t sh_rows, const moe_ffn_weights* sw,
                              const void* sh_h, const float* sh_h_scale, void* sh_out,
                              int32_t* dev_status, void* stream);

/* moe_swiglu_ffn_with_shared -- both GEMMs of the routed experts and of the
 * shared expert in ONE persistent launch ([MoE-walk] §3.3: SwiGLU experts as
 * one grouped GEMM, the merged shared expert as one more group):
 *   h_ws    = SiLU(a w1^T) * (a w3^T) per segment of offsets,
 *   out     = row_w * (h_ws w2^T),
 *   sh_h_ws = SwiGLU of (sh_a, sw13),  sh_out = sh_h_ws sw2^T,
 * the same values, bit for bit, as moe_gate_up_swiglu_with_shared followed by
 * moe_down_proj_with_shared. The CTAs take the tiles of both GEMMs from one
 * counter, in order, and a token block's down tiles start as soon as its h
 * rows are stored (a counter per token block in sync_ws, bounded waits), so
 * no SM idles while the last gate/up tiles end.
 *   sync_ws        device scratch of at least moe_swiglu_ffn_sync_size()
 *                  bytes, 16-byte aligned; zeroed by the call (stream order),
 *                  so it may not be shared by calls in flight at once.
 * bf16 only (MOE_ERR_UNSUPPORTED otherwise); other arguments, limits and
 * errors as the two calls it replaces. A wait that runs out flags
 * MOE_DEVSTAT_TIMEOUT in dev_status. */
MOE_API moe_status moe_swiglu_ffn_sync_size(int32_t rows, int32_t groups, int32_t sh_rows, size_t* bytes);
MOE_API moe_status moe_swiglu_ffn_with_shared(int32_t rows, int32_t H, const moe_ffn_weights* w,
                              const void* a, const int32_t* offsets, const float* row_w,
                              void* h_ws, void* out,
                              int32_t sh_rows, const moe_ffn_weights* sw, const void* sh_a,
                              void* sh_h_ws, void* sh_out,
                              void* sync_ws, size_t sync_ws_bytes,
                              int32_t* dev_status, void* stream);

/* moe_down_proj_combine -- the second GEMM with the combine fused into its
 * epilogue ([MoE-walk] §3.3.1 + §3.4): every routed row's weighted output
 * row_w[r] * (h[r] w2[e]^T) is added in fp32 straight into the row of its token
 * src_token[r] of acc_ws, the shared expert's output (sw, sh_h: optional) into
 * its own token's row, and y = bf16(acc_ws) at the end; no [rows, H]
 * intermediate and no separate combine.
 *   rows = T*k; h [rows, I] bf16; offsets, row_w, src_token from moe_permute;
 *   sw / sh_h: shared expert (groups 1) and its h [T, I_s], or NULL / NULL;
 *   acc_ws [T, H] fp32 device scratch (zeroed by the call); y [T, H] bf16.
 * bf16 only. The adds are atomic, so their order, and the last bits of y,
 * can differ from run to run; y agrees with moe_down_proj + moe_combine to
 * the rounding of o to bf16 that it skips. */
MOE_API moe_status moe_down_proj_combine(int32_t rows, int32_t T, int32_t H, const moe_ffn_weights* w,
                                 const void* h, const int32_t* offsets, const float* row_w,
                                 const int32_t* src_token, const moe_ffn_weights* sw,
                                 const void* sh_h, float* acc_ws, void* y,
                                 int32_t* dev_status, void* stream);

/* moe_gate_up_swiglu_gather -- the routed experts' first GEMM with the
 * permutation fused into its operand fetch ([MoE-walk] §3.2 + §3.3.1): row p
 * of the expert segments is read directly from x[src_token[p]], so
 * moe_permute can run with x_perm = NULL (no [T*k, H] copy is written).
 *   rows      T*k; x [T, H] bf16; src_token [rows] (from moe_permute, each in
 *             [0, T): indices outside are flagged MOE_DEVSTAT_BAD_EXPERT_ID in
 *             dev_status and not read); offsets [groups+1] (required);
 *   h_ws      [rows, I] bf16 = SiLU(x_p w1^T) * (x_p w3^T).
 * bf16 weights only (MOE_ERR_UNSUPPORTED otherwise); limits as above.
 * The rows are fetched with 16-byte cp.async by two extra warps; at the V3
 * shape on B200 this is slower than moe_permute + moe_gate_up_swiglu, whose
 * token rows arrive as TMA boxes, so use it where memory for x_perm is short. */
MOE_API moe_status moe_gate_up_swiglu_gather(int32_t rows, int32_t H, const moe_ffn_weights* w,
                                     const void* x, int32_t T, const int32_t* src_token,
                                     const int32_t* offsets, void* h_ws,
                                     int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_combine -- unpermute and weighted combine, [MoE-walk] §3.4:
 *   y[t] = shared_out[t] + sum_j topk_w[t][j] * expert_out[slot_to_row[t*k+j]]
 * summed in fp32 in slot order j = 0..k-1, then rounded once to bf16.
 * expert_out [T*k, H] bf16; slot_to_row [T*k]; topk_w [T, k] fp32 or NULL
 * (weights already applied, e.g. via row_w in moe_grouped_swiglu);
 * shared_out [T, H] bf16 or NULL; y [T, H] bf16 out. H % 8 == 0.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_combine(int32_t T, int32_t k, int32_t H, const void* expert_out,
                       const int32_t* slot_to_row, const float* topk_w,
                       const void* shared_out, void* y, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_bias_update -- aux-loss-free load balancing step, [V3-digest] §2.2:
 * overloaded experts' selection bias goes down, underloaded ones' up:
 *   bias[e] = bias[e] - gamma * sign(expert_counts[e] * E - T * k)
 * The sign is taken on exact integers (load vs the mean T*k/E); the update
 * is one fp32 subtraction. load_cv (optional, [1] fp32 out) receives the
 * coefficient of variation of the counts, sample std (E-1) / mean
 * ([V3-teardown] §4 load statistic). E <= 1024.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_bias_update(int32_t E, int32_t T, int32_t k, const int32_t* expert_counts,
                           float* bias, float gamma, float* load_cv, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_aux_loss -- sequence-level auxiliary balance loss, forward value only,
 * [MoE-walk] §6.2 (seq_aux, aux_loss_alpha = 0.001 for V2-Lite):
 *   the T tokens form T / seq_len sequences of seq_len consecutive tokens;
 *   per sequence   E * sum_e f_e * P_e   with
 *     f_e = #{(t, j) in the sequence : topk_ids[t][j] == e} / (seq_len * k)
 *     P_e = mean over the sequence's tokens of the token's score for e,
 *           normalised over all E experts (softmax probability, or the
 *           sigmoid divided by the sum of the E sigmoids);
 *   aux_out[0] = alpha * (mean over the sequences), fp32.
 * The value is 1 * alpha when loads and scores are uniform.
 *   logits    [T, E] fp32 (e.g. as written by moe_route); topk_ids [T, k]
 *   scoring   MOE_SOFTMAX or MOE_SIGMOID
 *   seq_len   divides T (seq_len = T: the batch is one sequence)
 *   workspace device scratch of moe_aux_loss_workspace_size() bytes, 8-byte
 *             aligned. E <= 256.
 * Scores are evaluated and summed in fp64; partial sums are combined in a
 * fixed order, so the result does not vary from run to run. topk_ids outside
 * [0, E) are not counted and flag MOE_DEVSTAT_BAD_EXPERT_ID in dev_status.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_aux_loss_workspace_size(int32_t T, int32_t E, int32_t seq_len, size_t* bytes);
MOE_API moe_status moe_aux_loss(int32_t T, int32_t E, int32_t k, int32_t seq_len, int32_t scoring,
                        const float* logits, const int32_t* topk_ids, float alpha, float* aux_out,
                        void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------ *
 * moe_tile_ffn_weights -- the bf16 expert weights in the layout the grouped
 * GEMMs stream fastest: the 256 weight rows x 64 K a GEMM tile loads in one
 * step (w13: 128 gate rows and the same features' 128 up rows; w2: 256 rows)
 * are one contiguous 32 KB block, the blocks of a tile in K order:
 *   w13_t[((g*(I/128) + f)*(H/64) + kb)*256 + r][c] = w13[g][f*128 + r][kb*64 + c]        (r < 128)
 *   w13_t[((g*(I/128) + f)*(H/64) + kb)*256 + r][c] = w13[g][I + f*128 + r-128][kb*64 + c] (r >= 128)
 *   w2_t [((g*(H/256) + b)*(I/64) + kb)*256 + r][c] = w2 [g][b*256 + r][kb*64 + c]
 * (c < 64). The values are unchanged, so results are bit-identical to the
 * row-major weights; pass the tiled copies with w->tiled = 1. The pages
 * state the weights only as [E, 2I, H] / [E, H, I] matrices; the tiling is
 * a layout of this library.
 *   src   row-major weights (src->tiled must be 0, dtype MOE_BF16).
 *   w13_t / w2_t  device outputs of the same sizes as src->w13 / src->w2 (either
 *         may be NULL to skip it); an output overlapping an input or the other
 *         output is refused (MOE_ERR_INVALID_ARG).
 * Limits: those of moe_grouped_swiglu (I % 128 == 0, H % 256 == 0).
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_tile_ffn_weights(int32_t H, const moe_ffn_weights* src, void* w13_t, void* w2_t,
                                        void* stream);

/* ------------------------------------------------------------------------ *
 * FP8 E4M3 quantisers ([V3-teardown] §3 infer.toml: weight_block_size
 * [128, 128], activation_scheme dynamic; [FP8-infer] 1x128 / 128x128 tiles).
 *   scale = amax / 448 in fp32 (1.0 for an all-zero tile);
 *   code  = e4m3 round-to-nearest-even, saturating, of v / scale (fp32 div).
 * moe_quantize_blocks: w [batch, N, K] bf16 -> q [batch, N, K] codes,
 *   scale [batch, N/128, K/128]. N % 128 == 0, K % 128 == 0.
 * moe_quantize_rows:   a [M, K] bf16 -> q [M, K] codes, scale [M, K/128].
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_quantize_blocks(int32_t batch, int32_t N, int32_t K, const void* w,
                               void* q, float* scale, void* stream);
MOE_API moe_status moe_quantize_rows(int32_t M, int32_t K, const void* a, void* q,
                             float* scale, void* stream);

/* ------------------------------------------------------------------------ *
 * Status helpers.
 * moe_read_device_status: copies *dev_status to *out after the work queued
 *   on `stream` finishes (synchronises that stream) and maps it to a status:
 *   0 -> MOE_OK, MOE_DEVSTAT_TIMEOUT -> MOE_ERR_DEVICE_TIMEOUT, any other
 *   nonzero -> MOE_ERR_DEVICE_CHECK.
 * moe_last_cuda_error: the cudaError_t behind the last MOE_ERR_CUDA on this
 *   thread (0 if none).
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_read_device_status(const int32_t* dev_status, int32_t* out, void* stream);
MOE_API int32_t moe_last_cuda_error(void);

/* ------------------------------------------------------------------------ *
 * Bounded device waits (debugging). The pages have no counterpart.
 * Every kernel that waits on an mbarrier (the grouped GEMMs, the gate GEMM)
 * gives up a wait after a limit of wall time, sets MOE_DEVSTAT_TIMEOUT in
 * its dev_status, lets its in-flight copies and MMAs finish, frees its
 * tensor memory and returns; its outputs are then incomplete.
 * moe_set_wait_limit_ns: the limit for launches issued after the call, in
 *   nanoseconds, process-wide; 0 restores the default (2 s). A limit far
 *   below a kernel's normal waits (a few ns) makes it time out on purpose,
 *   which is how the timeout path is tested. Always MOE_OK.
 * moe_wait_limit_ns: the current limit.
 * ------------------------------------------------------------------------ */
MOE_API moe_status moe_set_wait_limit_ns(uint64_t ns);
MOE_API uint64_t moe_wait_limit_ns(void);
MOE_API const char* moe_status_string(moe_status s);
MOE_API int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
