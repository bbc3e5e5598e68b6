/*
 * moefp8.h -- C ABI of libmoefp8.so: the forward of one fused routed-expert FP8 MoE layer on
 * NVIDIA B200 (sm_100a): the whole layer on one GPU (moe_forward), the gate in front of its
 * router (moe_gate), and the device steps of expert parallelism over the GPUs of a node
 * (moe_ep_dispatch, moe_forward_rows, moe_combine_rows), around an all-to-all the caller runs.
 *
 * The layer (sources are web pages, cited by title and section):
 *   "MindIE-SD Fused MoE" -- function signature and parameter table (hidden_states,
 *       router_logits, num_experts, top_k, w13 [E, hidden, 2*inter], w2 [E, inter, hidden],
 *       biases, weight scales, k_group / group_count / group_select_mode, routing_method,
 *       renormalize, routed_scaling_factor, custom_routing_function); execution flow
 *       (select_experts -> dispatch -> mlp -> combine); routing selection; MXFP8 example.
 *   "MATE Mega MoE" -- Typical Flow (a caller-owned runtime workspace, a one-time weight
 *       transform, then the fused expert compute), Current Limits, API (swiglu).
 *   "metrale_model_layers fp8_grouped_tc_w8a8.rs" -- the W8A8 step: activations quantized to
 *       E4M3 per (row, 128 group), FP8 weights in E4M3 tensor-core MMAs, SiLU products
 *       requantized, then the down projection; nothing launches unless the shapes fit.
 *   "DeepGEMM PR #371: Add W8A8 (FP8xFP8) Mega MoE support" -- UE8M0 scale factors per 32
 *       elements, 4 packed per 32-bit word; hidden / intermediate sizes that are not multiples
 *       of 512 (e.g. 768 and 1152).
 *   "mlx_native ops/moe_gate.rs" -- top-K + softmax + per_expert_scale; output expert ids and
 *       fp32 weights [T, k]; argument validation with an error message.
 *
 * Conventions for every entry point:
 *   - All tensors are row-major and contiguous; "device" pointers are CUDA device memory of the
 *     current device, "host" pointers are ordinary host memory.
 *   - The caller owns every buffer.  The library allocates no device memory and never
 *     synchronizes the stream, except where an entry point says so.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); all work is enqueued on it
 *     and runs asynchronously.
 *   - Return value: MOE_OK, or a negative MOE_ERR_* code.  On an error, nothing is launched and
 *     moe_last_error() (per host thread) describes the first problem found.
 *   - Faults found on the device (a bounded wait that ran out, an index out of range) do not
 *     trap; they are written to the workspace status word, readable with moe_read_status().
 */
#ifndef MOEFP8_H
#define MOEFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)   /* a dimension <= 0, top_k outside [1, E], NULL pointer, small buffer */
#define MOE_ERR_UNSUPPORTED (-2)   /* a valid problem outside what this library implements */
#define MOE_ERR_CUDA (-3)          /* a CUDA runtime call failed */
#define MOE_ERR_TIMEOUT (-4)       /* device status: a bounded wait inside a kernel ran out */
#define MOE_ERR_BOUNDS (-5)        /* device status: an index read from memory was out of range */

#define MOE_MAX_EXPERTS 256

/* One problem.  All fields are validated on every call; the library keeps no global state.
 *   routing            0 = softmax, 1 = sigmoid  ("MindIE-SD Fused MoE", routing_method)
 *   renormalize        softmax only: divide the selected weights by their sum; sigmoid
 *                      weights are always normalized over the selected experts
 *   group_count        experts form this many contiguous groups (1 = no grouped routing)
 *   k_group            groups kept per token, in [1, group_count]
 *   group_select_mode  group score: 0 = max score in the group, 1 = sum of its two largest
 *   routed_scaling_factor  multiplies every routing weight (applied last)
 *   recipe             0 = E4M3 with an fp32 scale per (row, 128-element block) for
 *                          activations and per (output column, 128-deep K block) for weights
 *                      1 = MXFP8: E4M3 with a UE8M0 power-of-two scale per 32 elements
 *                      2 = W4A8: weights E2M1 (FP4) with a UE8M0 scale per 32 K-elements,
 *                          activations MXFP8 as recipe 1 ("DeepGEMM PR #371", Changes: the W4A8
 *                          (FP8 x FP4) path, e2m1 weights with the same 4-packed UE8M0 scale
 *                          factors; "MATE Mega MoE": the W4A8 mixed-dtype GEMM path).  Weight
 *                          codes are packed two per byte along the last (N) dimension, the
 *                          even column in the low nibble: w13 [E, H, I] and w2 [E, I, H/2] bytes.
 *   shared_experts     0, or 1: one more expert, index num_experts, that every token uses with
 *                      weight 1 after its top_k routed experts ("metrale_model_layers
 *                      fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8: the shared expert's
 *                      gate/up and down run in the same grouped steps).  The weight and bias
 *                      tensors then hold num_experts + 1 experts, the shared one last; the
 *                      router still selects among num_experts.
 * Limits (MOE_ERR_UNSUPPORTED): hidden % 128, inter % 128, num_experts <= 256,
 * num_experts % group_count, k_group in [1, group_count], top_k <= k_group * experts per
 * group, group_select_mode 1 needs >= 2 experts per group.  ("MATE Mega MoE", Current Limits
 * asks hidden % 128 and inter % 256; inter % 128 is accepted here, as the DeepGEMM PR's
 * unaligned sizes such as inter = 1152 require.) */
typedef struct {
    int32_t num_tokens, hidden, inter, num_experts, top_k;
    int32_t routing;
    int32_t renormalize;
    int32_t group_count, k_group, group_select_mode;
    float routed_scaling_factor;
    int32_t recipe;
    int32_t shared_experts;
} moe_config_t;

/* Byte offsets of the regions inside a forward workspace (for tests and diagnostics).
 * S = shared_experts, k' = top_k + S expert slots per token (slot top_k is the shared
 * expert), E' = num_experts + S, A = num_tokens * k' rows.  Scales are stored K-block-major: one 4-byte word per
 * (128-column block, row) with a row stride of scale_rows words; the word is the fp32 scale
 * (recipe 0) or the four UE8M0 bytes of the block's four 32-column groups, lowest group in the
 * lowest byte (recipes 1 and 2).  All offsets are multiples of 1024. */
typedef struct {
    size_t status;       /* int32 status word (MOE_OK or a device MOE_ERR_*)             */
    size_t topk_idx;     /* int32 [T, k]   routing computed by moe_forward               */
    size_t topk_weights; /* fp32  [T, k]                                                 */
    size_t counts;       /* int32 [E']     rows per expert                               */
    size_t offsets;      /* int32 [E' + 1] first permuted row of each expert             */
    size_t tile_start;   /* int32 [E' + 1] first 128-row M tile of each expert           */
    size_t row_src;      /* int32 [A]      permuted row r came from slot row t*k' + j    */
    size_t row_of;       /* int32 [T, k']  permuted row of slot (t, j)                   */
    size_t hist;         /* int32 [chunks, E] per-chunk expert histograms                */
    size_t xq;           /* E4M3  [A, H]   quantized activations in permuted order       */
    size_t xs;           /* word  [H/128, scale_rows]                                    */
    size_t act_q;        /* E4M3  [A, I]   requantized SwiGLU products                   */
    size_t act_s;        /* word  [I/128, scale_rows]                                    */
    size_t o;            /* fp32  [A, H]   down-projection output per permuted row       */
    size_t scale_rows;   /* row stride (in words) of xs and act_s; >= A                  */
    size_t total;        /* bytes the workspace needs                                    */
} moe_workspace_layout_t;

/* Opaque per-stage timer (CUDA events) for moe_forward_profiled. */
typedef struct moe_profile moe_profile_t;

#define MOE_NUM_STAGES 6   /* route, permute, quantize, gemm1+swiglu+requant, gemm2, combine */

/* Message for the last error returned on this host thread ("" if none). */
const char *moe_last_error(void);

/* Validate a configuration without launching anything.  Returns MOE_OK or the error code the
 * other entry points would return for it. */
int moe_check_config(const moe_config_t *cfg);

/* Sizes, in bytes, of the four transformed-weight buffers that moe_transform_weights fills
 * (host call, no CUDA work). */
int moe_transformed_weights_size(const moe_config_t *cfg, size_t *w13_bytes, size_t *w13s_bytes,
                                 size_t *w2_bytes, size_t *w2s_bytes);

/* Re-lay the grouped FP8 expert weights for the forward ("MATE Mega MoE", Typical Flow step 2
 * and transform_weights_for_mega_moe).  Runs once, offline; deterministic and re-runnable.
 * (E below is num_experts + shared_experts: the shared expert's tensors come last.)
 *   w13        device, E4M3 codes [E, H, 2I] (K rows x N columns; columns 0:I gate, I:2I up);
 *              recipe 2: E2M1 codes two per byte along N, [E, H, I] bytes
 *   w13_scale  device, recipe 0: fp32 [E, H/128, 2I]; recipes 1, 2: UE8M0 bytes [E, H/32, 2I]
 *   w2         device, E4M3 codes [E, I, H]; recipe 2: [E, I, H/2] bytes of E2M1 pairs
 *   w2_scale   device, recipe 0: fp32 [E, I/128, H];  recipes 1, 2: UE8M0 bytes [E, I/32, H]
 * (scales are K-block-major, the orientation of the "MindIE-SD Fused MoE" MXFP8 example.)
 * Outputs (device, sizes from moe_transformed_weights_size; opaque to the caller): K-major
 * codes (recipe 2: still two per byte, now along K) with gate/up columns interleaved in blocks,
 * and the scales re-laid to match.  The code outputs must be 32-byte aligned, the scale outputs
 * 16-byte aligned.  Inputs and outputs must not overlap. */
int moe_transform_weights(const moe_config_t *cfg, const void *w13, const void *w13_scale,
                          const void *w2, const void *w2_scale, void *w13_t, void *w13s_t,
                          void *w2_t, void *w2s_t, void *stream);

/* Workspace bytes moe_forward needs for cfg->num_tokens tokens (host call).  A workspace sized
 * for T tokens serves every call with num_tokens <= T and the other fields equal.  Like
 * get_symm_buffer_for_mega_moe ("MATE Mega MoE", API), but on one GPU. */
int moe_workspace_size(const moe_config_t *cfg, size_t *bytes);

/* Region offsets of that workspace (host call). */
int moe_workspace_layout(const moe_config_t *cfg, moe_workspace_layout_t *layout);

/* Router top-k alone ("MindIE-SD Fused MoE", select_experts and routing selection;
 * "mlx_native ops/moe_gate.rs", output ids and weights).
 *   router_logits     device fp32 [T, E]
 *   per_expert_scale  device fp32 [E] or NULL (multiplies each selected expert's weight)
 *   topk_idx          device int32 [T, k]  out: expert ids, best first; ties -> lower index
 *   topk_weights      device fp32  [T, k]  out: routing weights                          */
int moe_route(const moe_config_t *cfg, const float *router_logits, const float *per_expert_scale,
              int32_t *topk_idx, float *topk_weights, void *stream);

/* The gate in front of the router ("mlx_native ops/moe_gate.rs": RMS-Norm of the hidden state,
 * the router matmul, then top-K + softmax + per-expert scale):
 *   logits[t, e] = sum_h ( x[t,h] / sqrt(mean_h x[t,h]^2 + rms_eps) * norm_weight[h] ) * router_weight[e, h]
 * in fp32, computed as r_t * sum_h x[t,h] * w'[e,h] with w'[e,h] = fl32(norm_weight[h] * router_weight[e,h])
 * and r_t = 1 / sqrt(mean_h x[t,h]^2 + rms_eps), then the router of moe_route on those logits with
 * cfg's routing fields.
 *
 * moe_transform_gate_weights writes w' once per set of weights, as three bf16 parts
 * hi = rn(w'), mid = rn(w' - hi), lo = rn(w' - hi - mid), each [E, H] row-major, back to back
 * (moe_gate_weights_size writes 3 * E * H * 2 to *bytes):
 *   norm_weight       device fp32 [H], 16-byte aligned
 *   router_weight     device fp32 [E, H] row-major, 16-byte aligned (E = cfg->num_experts)
 *   gate_weights      device, moe_gate_weights_size bytes, 16-byte aligned; out
 *
 * moe_gate: the sums run on the tensor core (bf16 x times each bf16 part, all accumulated in one
 * fp32 accumulator, so every product is exact), the H range split in eight fixed shares whose
 * partial sums are added in share order: a token's logits depend on its own row and on H only,
 * not on T or on the other tokens.
 *   hidden_states     device bf16 [T, H], 16-byte aligned
 *   gate_weights      device, from moe_transform_gate_weights, 16-byte aligned
 *   per_expert_scale  device fp32 [E] or NULL
 *   logits            device fp32 [T, E]  out
 *   topk_idx          device int32 [T, k] out;  topk_weights device fp32 [T, k] out
 * Two launches (the router matmul, then the router, which also applies r_t).  A wait that runs
 * out inside the matmul leaves NaN logits for the tiles it covers.  Feed topk_idx/topk_weights
 * to moe_forward to run the layer on them. */
int moe_gate_weights_size(const moe_config_t *cfg, size_t *bytes);
int moe_transform_gate_weights(const moe_config_t *cfg, const float *norm_weight, const float *router_weight,
                               void *gate_weights, void *stream);
int moe_gate(const moe_config_t *cfg, const void *hidden_states, const void *gate_weights, float rms_eps,
             const float *per_expert_scale, float *logits, int32_t *topk_idx, float *topk_weights, void *stream);

/* The fused layer forward ("MindIE-SD Fused MoE", fused_moe; "MATE Mega MoE",
 * fp8_fp8_mega_moe): route -> permute -> quantize -> gate+up GEMM with SwiGLU and
 * requantization -> down GEMM -> weighted combine.
 *   hidden_states     device bf16 [T, H]
 *   router_logits     device fp32 [T, E], or NULL when topk_idx/topk_weights are given
 *   per_expert_scale  device fp32 [E] or NULL (used only with router_logits)
 *   topk_idx          device int32 [T, k] or NULL: routing supplied by the caller (the
 *   topk_weights      device fp32  [T, k]  custom routing function path); exactly one of
 *                                           router_logits and topk_idx must be non-NULL.
 *                                           The k ids of a token must be distinct, in [0, E).
 *   w13_t .. w2s_t    device, from moe_transform_weights with the same cfg fields (codes
 *                     32-byte aligned, scales 16-byte aligned)
 *   w13_bias          device bf16 [E', 2I] or NULL (16-byte aligned; E' = num_experts + shared_experts)
 *   w2_bias           device bf16 [E', H] or NULL (16-byte aligned)
 *   y                 device bf16 [T, H], contiguous; out
 *   expert_counts     device int32 [E'] or NULL; out: rows routed to each expert (the shared
 *                     expert's count is num_tokens)
 *   workspace         device, >= moe_workspace_size bytes, 256-byte aligned; scratch owned by
 *                     the caller; must not be shared by calls in flight at the same time
 * A row's output bits do not depend on the other rows of the batch. */
int moe_forward(const moe_config_t *cfg, const void *hidden_states, const float *router_logits,
                const float *per_expert_scale, const int32_t *topk_idx, const float *topk_weights,
                const void *w13_t, const void *w13s_t, const void *w2_t, const void *w2s_t,
                const void *w13_bias, const void *w2_bias, void *y, int32_t *expert_counts,
                void *workspace, size_t workspace_bytes, void *stream);

/* moe_forward without a caller workspace, for callers that cannot allocate device memory: code
 * running inside a host framework that owns all device memory (a serving engine's pre-reserved
 * pool, a plugin interface that gives its kernels no scratch), where cudaMalloc is not allowed
 * because it can synchronize the device and can fail under memory pressure mid-serving.
 * The pages have no counterpart of this entry point.
 *   Arguments as moe_forward, minus workspace / workspace_bytes.  The caller still owns and
 *   passes every input and output; the scratch is a fixed 16 MiB array in the library's device
 *   image (each GPU that loads the library holds it until the process exits).  A problem whose
 *   moe_workspace_size exceeds 16 MiB (16777216 bytes) is rejected with MOE_ERR_UNSUPPORTED
 *   and nothing is launched; e.g. the 64-token decode problem (H 2816, I 768, E 128, top-8)
 *   needs about 7.7 MB.
 *   The first call on a device looks the array's address up (cudaGetSymbolAddress) with that
 *   device current; make that first call before any stream capture.  The array is shared by
 *   every call on the device and keeps the last call's contents (the forward clears its status
 *   word itself); calls that overlap on the GPU race on it.  Allocates nothing: no cudaMalloc,
 *   no cudaFree, no allocating library routine.  The return code reports what the host checks
 *   find and launch failures; faults the kernels find on the device (a bounded wait that ran
 *   out, an index out of range) land in the array's status word, read with
 *   moe_static_workspace_status. */
int moe_forward_static_workspace(const moe_config_t *cfg, const void *hidden_states,
                                 const float *router_logits, const float *per_expert_scale,
                                 const int32_t *topk_idx, const float *topk_weights,
                                 const void *w13_t, const void *w13s_t, const void *w2_t,
                                 const void *w2s_t, const void *w13_bias, const void *w2_bias,
                                 void *y, int32_t *expert_counts, void *stream);

/* Test hook, the gate+up step taken apart ("DeepGEMM PR #371", Testing: overlapped and
 * non-overlapped runs give bitwise-identical outputs).  Runs the forward's permutation and
 * quantization from the given routing, then the forward's gate+up GEMM kernel with its
 * down-projection epilogue, storing the promoted fp32 gate/up sums without bias into h, then a
 * separate SwiGLU + requantization kernel that writes the act codes and scales into the
 * workspace (moe_workspace_layout: act_q, act_s), where moe_forward's fused epilogue writes them.
 *   topk_idx          device int32 [T, k], ids in [0, E)
 *   w13_t, w13s_t     as for moe_forward;  w13_bias device bf16 [E', 2I] or NULL
 *   h                 device fp32 [T*(k + shared_experts), 2I], 32-byte aligned; out, columns in
 *                     the transformed order of w13_t
 *   workspace         as for moe_forward
 * The codes and scales must equal moe_forward's bit for bit on the same inputs. */
int moe_debug_unfused_gate_up(const moe_config_t *cfg, const void *hidden_states, const int32_t *topk_idx,
                              const void *w13_t, const void *w13s_t, const void *w13_bias, float *h,
                              void *workspace, size_t workspace_bytes, void *stream);

/* The status word of the last moe_forward_static_workspace call on the current device
 * (MOE_OK, or MOE_ERR_TIMEOUT / MOE_ERR_BOUNDS set by a kernel), like moe_read_status: it
 * synchronizes `stream`, then copies the word into *status (host).  The pages have no
 * counterpart of this entry point. */
int moe_static_workspace_status(int32_t *status, void *stream);

/* moe_forward, recording a CUDA event before each of the MOE_NUM_STAGES stages and after the
 * last one into `prof` (which accumulates per-stage device time until reset).  prof may be
 * NULL, which makes this identical to moe_forward. */
int moe_forward_profiled(const moe_config_t *cfg, const void *hidden_states,
                         const float *router_logits, const float *per_expert_scale,
                         const int32_t *topk_idx, const float *topk_weights, const void *w13_t,
                         const void *w13s_t, const void *w2_t, const void *w2s_t,
                         const void *w13_bias, const void *w2_bias, void *y,
                         int32_t *expert_counts, void *workspace, size_t workspace_bytes,
                         moe_profile_t *prof, void *stream);

/* Expert parallelism over `ranks` ranks of one node ("MindIE-SD Fused MoE", execution flow:
 * dispatch, mlp, combine, and the dynamic dispatcher's all-to-all; "MATE Mega MoE", Typical
 * Flow: up to 8 intranode ranks).  Rank r owns experts r*E/R .. (r+1)*E/R - 1 (E % R == 0, no
 * shared expert); each rank routes its own T tokens with moe_route, then:
 *
 * moe_ep_dispatch orders this rank's A = T*k routed slots (slot = t*k + j) by destination rank,
 * stable in slot order, and gathers what each destination needs.  cfg: this rank's tokens, the
 * global expert count.
 *   hidden_states   device bf16 [T, H], 16-byte aligned
 *   topk_idx        device int32 [T, k]: global expert ids
 *   send_counts     device int32 [ranks]   out: slots going to each rank
 *   send_x          device bf16 [A, H]     out: each slot's token row, in send order (16-byte aligned)
 *   send_expert     device int32 [A]       out: each slot's expert id local to its destination
 *   slot_pos        device int32 [T, k]    out: each slot's position in send order
 *   workspace       as for moe_forward with the same cfg (scratch for the ordering)
 *   A memset and four launches.  An expert id outside [0, E) is reported as MOE_ERR_BOUNDS in
 *   the workspace's status word (moe_read_status); its slot is not sent (not counted in
 *   send_counts) and its slot_pos is -1.
 *
 * The caller then exchanges send_x and send_expert (all-to-all with the counts: NCCL, or peer
 * copies), and every rank runs moe_forward_rows on the N rows it received:
 *
 * moe_forward_rows: each row through one local expert with weight 1.  cfg: num_tokens = N,
 * top_k = 1, num_experts = E/R, no shared expert; weights from moe_transform_weights on this
 * rank's experts.
 *   rows            device bf16 [N, H], 16-byte aligned
 *   expert_of_row   device int32 [N]: local expert ids
 *   o_rows          device fp32 [N, H] out, 16-byte aligned: each row's GEMM2 output (+ b2), in row
 *                   order, bit-identical to the same row's output inside moe_forward (a row's
 *                   result depends only on its own codes and its expert's weights)
 *   The forward's launches, the last one copying the rows out in row order.
 *
 * The caller returns the rows (the reverse all-to-all), so that o_home[i] belongs to send
 * position i, and combines them on the home rank:
 *
 * moe_combine_rows: y[t] = bf16_rn( sum_j topk_weights[t,j] * o_home[slot_pos[t,j]] ), fp32, in
 * slot order: the combine of moe_forward, so y is bit-identical to the single-GPU forward.
 *   o_rows          device fp32 [num_rows, H], 16-byte aligned (may be NULL when num_rows is 0)
 *   num_rows        rows of o_rows: the sum of the send counts, in [0, T*k]
 *   slot_pos        device int32 [T, k] from moe_ep_dispatch
 *   y               device bf16 [T, H], 16-byte aligned; out
 *   status          device int32 or NULL: a slot whose position lies outside [0, num_rows) adds
 *                   nothing to its token's sum and sets it to MOE_ERR_BOUNDS (if it held MOE_OK)
 *   One launch. */
int moe_ep_dispatch(const moe_config_t *cfg, int ranks, const void *hidden_states, const int32_t *topk_idx,
                    int32_t *send_counts, void *send_x, int32_t *send_expert, int32_t *slot_pos,
                    void *workspace, size_t workspace_bytes, void *stream);
int moe_forward_rows(const moe_config_t *cfg, const void *rows, const int32_t *expert_of_row,
                     const void *w13_t, const void *w13s_t, const void *w2_t, const void *w2s_t,
                     const void *w13_bias, const void *w2_bias, float *o_rows, void *workspace,
                     size_t workspace_bytes, void *stream);
int moe_combine_rows(const moe_config_t *cfg, const float *o_rows, int32_t num_rows, const int32_t *slot_pos,
                     const float *topk_weights, void *y, int32_t *status, void *stream);

/* Create / destroy a stage profiler (creates CUDA events on the current device). */
int moe_profile_create(moe_profile_t **prof);
int moe_profile_destroy(moe_profile_t *prof);
/* Synchronize on the recorded events, add their elapsed times into the totals and return the
 * totals: stage_ms[MOE_NUM_STAGES] (milliseconds summed over calls) and *calls. */
int moe_profile_read(moe_profile_t *prof, float *stage_ms, int32_t *calls);
int moe_profile_reset(moe_profile_t *prof);

/* Read the workspace status word (blocking copy after synchronizing `stream`): MOE_OK, or
 * MOE_ERR_TIMEOUT / MOE_ERR_BOUNDS set by a kernel.  moe_forward clears it when it starts. */
int moe_read_status(const void *workspace, int32_t *status, void *stream);

/* Failure-detection self test: launch one kernel that waits on a barrier nothing will ever
 * complete, with a limit of `timeout_us` microseconds, after which it writes MOE_ERR_TIMEOUT to
 * the device int32 *status and returns.  The context stays usable. */
int moe_selftest_bounded_wait(int32_t *status, uint32_t timeout_us, void *stream);

/* Fault injection for failure-detection tests (no counterpart on the pages).  Only the debug
 * library, libmoefp8_debug.so (built with MOE_FAULT_INJECTION), acts on it; the release library
 * returns MOE_ERR_UNSUPPORTED.  MOE_FAULT_SKIP_STAGE arms one fault for the next moe_forward on
 * this host thread: the gate+up GEMM's producer in CTA 0 skips its first K stage (no copies, no
 * arrival), so the MMA role's bounded wait runs out (about 2 s), every role of that CTA leaves
 * cleanly and the status word reads MOE_ERR_TIMEOUT.  Nothing faults or hangs; the context stays
 * usable.  MOE_FAULT_NONE disarms it. */
#define MOE_FAULT_NONE 0
#define MOE_FAULT_SKIP_STAGE 1
int moe_debug_inject_fault(int fault);

#ifdef __cplusplus
}
#endif

#endif /* MOEFP8_H */
