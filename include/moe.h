/*
 * moe.h -- C ABI of the B200 (sm_100a) fine-grained Mixture-of-Experts layer:
 * forward, and (for training) forward with saved activations and backward.
 *
 * The layer (per token x of length d) is the one described on the FusionLLM
 * page "FusionLLM：融合 MLA、GDN 与 MoE 的高效混合架构大模型训练框架", section
 * "混合专家（MoE）" (fine-grained DeepSeekMoE layer, group-limited routing,
 * bias-free sigmoid gating) with the sizes of its section "模型配置与规模"
 * (64 routed experts, 6 active, 4 shared, moe_inter_dim 1536, dim 2048):
 *
 *   s_e  = sigmoid(W_router[e] . x)                       gate scores
 *   keep the topk_group of n_group expert groups with the largest max score,
 *   idx  = the k largest s_e inside the kept groups (descending, ties to the
 *          lower index), w_j = s_idx[j] / sum_j s_idx[j]
 *   y    = sum_j w_j * SwiGLU_{idx[j]}(x) + sum_s SwiGLU_shared_s(x)
 *   SwiGLU_e(x) = W_down[e] (silu(W_gate[e] x) * (W_up[e] x))
 *
 * (router g(x) = W_g x and fixed-k top-k: "大模型工程（一）：Transformer 到
 * MoE", section "MoE 数学：路由、容量与平衡详解"; weighted sum over the chosen
 * experts: its MoEBlock listing, section "混合专家：更多参数，相同 FLOPs", and
 * the moe_layer pseudocode of "开源混合架构大模型技术解析", section 四.)
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must point to memory of the current
 *     CUDA device; the library reads or writes them only from kernels queued
 *     on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 *     stream).  Calls are asynchronous unless stated otherwise: they return
 *     after queueing work and never synchronise the stream.
 *   - The caller owns every buffer.  The library allocates no device memory;
 *     it keeps only per-process caches (kernel attributes) and one fixed
 *     256 KiB device array that only moe_expert_counts_noalloc uses.
 *   - All matrices are row-major and contiguous.  Device pointers must be
 *     16-byte aligned; `workspace` must be 256-byte aligned.
 *   - Errors: invalid arguments are reported synchronously, before anything
 *     is queued, as a negative moe_status.  A failed launch returns
 *     MOE_ERR_CUDA.  Faults found on the device (a wait that ran out of time,
 *     a bounds check) do not trap: the kernel records a code in the status
 *     word at the start of the workspace, returns early, and the host reads
 *     it with moe_get_device_status().
 *   - T = 0 is valid and queues nothing (moe_forward_ex with an expert_load
 *     buffer queues the zeroing of that buffer).
 *   - moe_forward can be captured in a CUDA graph: every replay resets the
 *     status word and its internal counters itself.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
#define MOE_EXTERN extern "C"
#else
#define MOE_EXTERN extern
#endif
#define MOE_API MOE_EXTERN __attribute__((visibility("default")))

/* Gates (routing weights).  MOE_GATE_SIGMOID is the FusionLLM gate
 * ("FusionLLM：融合 MLA、GDN 与 MoE 的高效混合架构大模型训练框架", section
 * "混合专家（MoE）"): sigmoid scores, weights = scores of the chosen experts
 * normalised to sum 1.  MOE_GATE_SOFTMAX_TOPK is the Mixtral-style gate of
 * "大模型工程（一）：Transformer 到 MoE", section "MoE 数学：路由、容量与平衡详解":
 * the k largest logits, weights = softmax of those k logits. */
typedef enum { MOE_GATE_SIGMOID = 0, MOE_GATE_SOFTMAX_TOPK = 1 } moe_gate;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* a size, pointer or alignment check failed          */
    MOE_ERR_UNSUPPORTED = -2, /* valid, but outside what the kernels implement      */
    MOE_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed        */
    MOE_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than moe_workspace_bytes */
    MOE_ERR_TIMEOUT = -5,     /* device: a bounded wait gave up                     */
    MOE_ERR_DEVICE = -6       /* device: a bounds check failed                      */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/*
 * Shape limits checked by every entry point (else MOE_ERR_INVALID_ARG or
 * MOE_ERR_UNSUPPORTED):
 *   T >= 0, T * k < 2^31;  1 <= E <= 256;  1 <= n_group <= 32;
 *   E % n_group == 0;  1 <= topk_group <= n_group;  1 <= k <= 8;
 *   k <= topk_group * (E / n_group);
 *   d % 64 == 0;  inter % 128 == 0;  0 <= n_shared;
 *   bf16 path (moe_forward): d % 256 == 0 (output tiles of 256 columns).
 */

/*
 * moe_workspace_bytes -- bytes of device workspace moe_forward needs for
 * these sizes.  Host only, no CUDA calls.  Returns 0 for invalid sizes.
 */
MOE_API size_t moe_workspace_bytes(int T, int d, int E, int k, int inter, int n_shared,
                                   int in_dt);

/* Regions of the workspace (byte offsets from its start). */
enum {
    MOE_WS_STATUS = 0,       /* int32[64]: [0] status code, [1] where, [2..3] info     */
    MOE_WS_COUNTS = 1,       /* int32[E]   tokens routed to each expert                */
    MOE_WS_OFFSETS = 2,      /* int32[E+1] first row of each expert in the permuted
                                layout (bf16: unpadded; f32: padded to 128 rows)     */
    MOE_WS_BLOCK_COUNTS = 3, /* int32[max(ceil(T/256), ceil(T/32)) * E] per-block
                                histogram (the permutation's token blocks)          */
    MOE_WS_TOPK_IDX = 4,     /* int32[T*k] chosen experts (used when no output given)  */
    MOE_WS_TOPK_W = 5,       /* f32[T*k]   gate weights                               */
    MOE_WS_ROW_SRC = 6,      /* int32[rows_cap] permuted row -> t*k + j, or -1 (pad)    */
    MOE_WS_X_PERM = 7,       /* in_dt[rows_cap, d] x rows in expert-contiguous order    */
    MOE_WS_H = 8,            /* in_dt[rows_cap, inter] silu(gate) * up, routed rows    */
    MOE_WS_H_SHARED = 9,     /* in_dt[T, n_shared*inter] the same for shared experts   */
    MOE_WS_SLOTS = 10,       /* in_dt[T*k, d] w_j * expert output, token order          */
    MOE_WS_Y_SHARED = 11,    /* bf16 with shared experts: f32[T, d] shared output        */
    MOE_WS_TOTAL = 12        /* total size                                            */
};
/* rows_cap = T*k + 128*E (the padded permuted layout never needs more). */

/*
 * moe_workspace_layout -- fill offsets[0..n-1] (n <= MOE_WS_TOTAL + 1) with
 * the byte offsets of the regions above, offsets[MOE_WS_TOTAL] with the
 * total.  Host only.  Returns MOE_OK or MOE_ERR_INVALID_ARG.
 */
MOE_API int moe_workspace_layout(int T, int d, int E, int k, int inter, int n_shared,
                                 int in_dt, size_t *offsets, int n);

/*
 * moe_route -- routing only: router GEMM, sigmoid, group limit, top-k,
 * normalisation.
 *   x         device, in_dt[T, d]
 *   W_router  device, in_dt[E, d]
 *   topk_idx  device, int32[T, k] out: chosen experts, descending score,
 *             ties to the lower index
 *   topk_w    device, f32[T, k]   out: normalised gate weights (sum to 1)
 * Logits accumulate in fp32; selection compares fp32 logits (sigmoid is
 * monotone, so this is the same choice as comparing scores), weights are
 * fp32 sigmoid values normalised over the chosen k.
 */
MOE_API int moe_route(const void *x, const void *W_router, int T, int d, int E, int k,
                      int n_group, int topk_group, int in_dt, int32_t *topk_idx,
                      float *topk_w, void *stream);

/*
 * moe_forward -- the whole layer.
 *   x          device, in_dt[T, d]
 *   W_router   device, in_dt[E, d]
 *   W_gate_up  device, in_dt[E, 2*inter, d]: rows [0, inter) gate, [inter, 2*inter) up
 *   W_down     device, in_dt[E, d, inter]
 *   W_shared   device, in_dt: gate_up [2*S*inter, d] (the S gate blocks, then
 *              the S up blocks) followed by down [d, S*inter]; NULL iff
 *              n_shared == 0
 *   y          device, out_dt[T, d] out
 *   topk_idx_out, topk_w_out  device, optional (NULL = keep in workspace)
 *   workspace  device, >= moe_workspace_bytes(...) bytes, 256-byte aligned;
 *              its contents need no initialisation and are overwritten
 * Arithmetic: in_dt inputs, fp32 accumulation in every GEMM; the SwiGLU
 * hidden h is stored as in_dt between the two expert GEMMs; each routed
 * expert's output row is scaled by its gate weight in fp32 and stored once as
 * in_dt (a "slot"); the final sum is y = shared + slot_0 + ... + slot_{k-1}
 * in fp32, in that fixed order, so y is bitwise reproducible from run to run.
 * bf16 uses tcgen05 tensor cores; f32 uses CUDA cores.
 */
MOE_API int moe_forward(const void *x, const void *W_router, const void *W_gate_up,
                        const void *W_down, const void *W_shared, int T, int d, int E, int k,
                        int n_group, int topk_group, int inter, int n_shared, int in_dt,
                        int out_dt, void *y, int32_t *topk_idx_out, float *topk_w_out,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_route_ex / moe_forward_ex -- moe_route / moe_forward with the gating
 * variants of "大模型工程（一）：Transformer 到 MoE", section "MoE 数学：路由、容量
 * 与平衡详解" (moe_route and moe_forward are these with MOE_GATE_SIGMOID, no
 * bias and no load output):
 *   gate         MOE_GATE_SIGMOID or MOE_GATE_SOFTMAX_TOPK (see moe_gate)
 *   expert_bias  device f32[E] or NULL: selection-only bias (the aux-loss-free
 *                load balancing of DeepSeek-V3 described there): the group
 *                limit and the top-k compare gate score + expert_bias[e]
 *                (gate score = sigmoid(logit) for MOE_GATE_SIGMOID, the logit
 *                for MOE_GATE_SOFTMAX_TOPK); the weights use the unbiased
 *                scores.  The caller updates the bias between steps from the
 *                expert loads.
 *   expert_load  (moe_forward_ex) device int32[E] or NULL, out: tokens routed
 *                to each expert in this call (sum = T * k), the load figure
 *                that such a bias update reads.
 * Other arguments, layouts, ownership and errors as moe_route / moe_forward;
 * an unknown gate or a host pointer for expert_bias / expert_load returns
 * MOE_ERR_INVALID_ARG before any launch.
 */
MOE_API int moe_route_ex(const void *x, const void *W_router, int T, int d, int E, int k,
                         int n_group, int topk_group, int in_dt, int gate,
                         const float *expert_bias, int32_t *topk_idx, float *topk_w,
                         void *stream);
MOE_API int moe_forward_ex(const void *x, const void *W_router, const void *W_gate_up,
                           const void *W_down, const void *W_shared, int T, int d, int E, int k,
                           int n_group, int topk_group, int inter, int n_shared, int in_dt,
                           int out_dt, int gate, const float *expert_bias, void *y,
                           int32_t *topk_idx_out, float *topk_w_out, int32_t *expert_load,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_get_device_status -- synchronise `stream`, then copy the status word
 * of `workspace` to *status (MOE_OK or a negative code) and, if `where` is
 * not NULL, the code of the kernel site that set it.  Returns MOE_OK or
 * MOE_ERR_CUDA.
 */
MOE_API int moe_get_device_status(const void *workspace, int *status, int *where,
                                  void *stream);

/* moe_clear_device_status -- queue a reset of the status word to MOE_OK. */
MOE_API int moe_clear_device_status(void *workspace, void *stream);

/*
 * moe_selftest_timeout -- queue one kernel that waits on a barrier nothing
 * will ever signal, with a limit of `limit_us` microseconds (1..1000000); when
 * the limit runs out the kernel writes MOE_ERR_TIMEOUT into the status word of
 * `workspace` and returns.  Exercises the bounded-wait path of the GEMM
 * kernels without hanging the GPU.
 */
MOE_API int moe_selftest_timeout(void *workspace, int limit_us, void *stream);

/*
 * moe_set_stage_events -- optional instrumentation for benchmarks.  With
 * events != NULL (n == MOE_N_STAGE_EVENTS handles of type cudaEvent_t, created
 * by the caller), every following moe_forward in this process records
 * events[i] on its stream: [0] start, [1] after routing, [2] after the
 * permutation, [3] after the gate/up GEMM (shared and routed experts, one
 * launch), [4] after the down GEMM (shared and routed experts, one launch),
 * [5] at the end (after the final sum y = shared + slots).  A NULL entry is
 * not recorded (an event record between two kernels keeps the second from
 * starting early, so a timing run records only the boundaries it needs).
 * events == NULL turns it off.  Process-wide setting, not thread-safe.
 * Returns MOE_OK or MOE_ERR_INVALID_ARG.
 */
#define MOE_N_STAGE_EVENTS 6
MOE_API int moe_set_stage_events(void *const *events, int n);

/*
 * moe_expert_counts_noalloc -- per-expert token counts and segment offsets
 * of a routing result, for callers that must not allocate device memory or
 * pass a workspace on the call path (e.g. a serving step whose device memory
 * is planned once up front).  The pages have no counterpart of this entry
 * point; it computes the histogram and scan of the permutation stage on its
 * own, with its scratch in a fixed device array of the library.
 *   topk_idx  device, int32[T, k]: expert ids; every occurrence counts (a
 *             row that repeats an id adds it as often as it appears); ids
 *             outside [0, E) are skipped without an error
 *   counts    device, int32[E]   out: occurrences of each expert id
 *   offsets   device, int32[E+1] out: exclusive prefix sum of counts
 *             (unpadded segments; offsets[E] = number of counted ids)
 * Limits: 1 <= k <= 8, k <= E <= 256, ceil(T/256) * E <= 65536 (the fixed
 * scratch: 256 KiB; e.g. T <= 262144 at E = 64).  Larger sizes return
 * MOE_ERR_WORKSPACE before any launch; bad arguments MOE_ERR_INVALID_ARG.
 * Allocates nothing.  The first call on a device (with it current) looks up
 * the scratch array's device address; make that first call before any stream
 * capture.  All calls share the one array: calls that overlap in time (two
 * streams, two host threads) race and must be serialised by the caller.
 * Nothing in the array needs to start at zero.  Queues work on `stream` and
 * returns without synchronising.
 */
MOE_API int moe_expert_counts_noalloc(const int32_t *topk_idx, int T, int k, int E,
                                      int32_t *counts, int32_t *offsets, void *stream);

/*
 * ---- Training: forward with saved activations, and the layer backward -----
 *
 * The layer is trained with the rest of the model (the FusionLLM page is a
 * pretraining framework: section "训练优化技术", whose fused kernels include a
 * grouped GEMM for the MoE layer; pretraining on 8 GPUs per its section
 * "模型配置与规模"); its backward is the chain rule through the forward above,
 * for an upstream gradient dy = dL/dy:
 *   a_j  = dy . SwiGLU_{idx[j]}(x)   (dL/dw_j),   abar = sum_j w_j a_j
 *   MOE_GATE_SIGMOID:      dL/dlogit_j = (a_j - abar) / sum_i s_i * s_j (1 - s_j)
 *   MOE_GATE_SOFTMAX_TOPK: dL/dlogit_j = w_j (a_j - abar)
 *   (only the chosen experts' logits get a gradient; the selection, the group
 *    limit and a selection bias pass none)
 *   dW_router[e] = sum_t dL/dlogit_{t,e} x_t,  dx += sum_j dL/dlogit_j W_router[idx[j]]
 *   per chosen expert (weight w_j; shared experts weight 1): dh = w_j W_down^T dy,
 *   dg = dh * up * silu'(gate), du = dh * silu(gate), dW_down += w_j dy h^T,
 *   dW_gate += dg x^T, dW_up += du x^T, dx += W_gate^T dg + W_up^T du.
 *
 * moe_saved_bytes -- bytes of the `saved` buffer of moe_forward_train (bf16
 * layers): the gate / up pre-activations, bf16, in blocks of 16 features.
 * Routed part: [inter/16][T*k][16 gate | 16 up], rows in expert-contiguous
 * order (expert 0's tokens in token order, then expert 1's, ...); then the
 * shared part [n_shared*inter/16][T][16 gate | 16 up] (feature f of block b is
 * shared feature 16 b + f, counting all shared experts' features in order).
 * The layout lets each warp of the GEMMs write and read 32 rows x 64 B in one
 * piece.  0 for invalid sizes.
 */
MOE_API size_t moe_saved_bytes(int T, int k, int inter, int n_shared);

/*
 * moe_forward_train -- moe_forward_ex that also writes the pre-activations
 * the backward needs into `saved` (device, moe_saved_bytes bytes, 16-byte
 * aligned, owned by the caller until the matching moe_backward has run).  y,
 * topk_idx_out and topk_w_out as moe_forward_ex; the backward needs the
 * routing, so topk_idx_out and topk_w_out are required here.  bf16 layers only
 * (MOE_ERR_UNSUPPORTED otherwise); other arguments and errors as
 * moe_forward_ex.
 */
MOE_API int moe_forward_train(const void *x, const void *W_router, const void *W_gate_up,
                              const void *W_down, const void *W_shared, int T, int d, int E,
                              int k, int n_group, int topk_group, int inter, int n_shared,
                              int in_dt, int out_dt, int gate, const float *expert_bias,
                              void *y, int32_t *topk_idx_out, float *topk_w_out,
                              int32_t *expert_load, void *saved, size_t saved_bytes,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_backward_workspace_bytes -- scratch bytes of moe_backward for these
 * sizes (bf16 layers; 0 for invalid or unsupported sizes).  Regions: status
 * words and tile counters, expert counts and padded offsets, the permutation
 * (segments padded to 128 rows) and its inverse, x and dy rows in that order,
 * the SwiGLU backward rows dg|du and w*h, the per-row parts of dL/dw,
 * dL/dlogit, the chosen experts' dx rows, the shared experts' rows and their
 * fp32 dx, and row-slice sums of dW_router.
 */
MOE_API size_t moe_backward_workspace_bytes(int T, int d, int E, int k, int inter,
                                            int n_shared);

/*
 * moe_backward -- gradients of the layer for the forward that
 * moe_forward_train ran with the same x, weights, gate and `saved`:
 *   x, W_router, W_gate_up, W_down, W_shared  the forward's inputs (bf16)
 *   dy          device, bf16 [T, d]: dL/dy
 *   topk_idx    device, int32 [T, k]: the forward's topk_idx_out
 *   topk_w      device, f32 [T, k]: the forward's topk_w_out
 *   saved       device: the forward's saved pre-activations
 *   gate        the forward's gate
 * Outputs (device, fp32, overwritten; same layouts as the forward tensors):
 *   dx [T, d], dW_router [E, d], dW_gate_up [E, 2*inter, d], dW_down
 *   [E, d, inter], dW_shared [2*SI*d + d*SI] (SI = n_shared*inter; NULL iff
 *   n_shared == 0).  Experts no token chose get zero gradients.
 * Every sum runs in a fixed order: results are bitwise reproducible.
 * Requirements: in_dt == MOE_BF16, d and inter multiples of 256 (else
 * MOE_ERR_UNSUPPORTED); workspace of moe_backward_workspace_bytes bytes (else
 * MOE_ERR_WORKSPACE), 256-byte aligned.  Device faults as for the forward
 * (status word of `workspace`).  T = 0 queues the zeroing of the weight
 * gradients only.  Queues work on `stream`; no synchronisation, no
 * allocation; capturable in a CUDA graph.
 */
MOE_API int moe_backward(const void *x, const void *W_router, const void *W_gate_up,
                         const void *W_down, const void *W_shared, const void *dy,
                         const int32_t *topk_idx, const float *topk_w, const void *saved,
                         int T, int d, int E, int k, int inter, int n_shared, int in_dt,
                         int gate, float *dx, float *dW_router, float *dW_gate_up,
                         float *dW_down, float *dW_shared, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * moe_set_backward_stage_events -- the instrumentation of moe_set_stage_events
 * for moe_backward: with n == MOE_N_BWD_STAGE_EVENTS cudaEvent_t handles,
 * every following moe_backward records events[i]: [0] start, [1] after the
 * permutation and row gather, [2] after dh = W_down^T dy with the SwiGLU
 * backward, [3] after dL/dlogit, [4] after the dx parts W_gate_up^T [dg|du],
 * [5] after the dx sum, [6] after dW_down, [7] after dW_gate_up, [8] at the end
 * (after dW_router).  NULL entries are skipped; events == NULL turns it off.
 * Process-wide, not thread-safe.  Returns MOE_OK or MOE_ERR_INVALID_ARG.
 */
#define MOE_N_BWD_STAGE_EVENTS 9
MOE_API int moe_set_backward_stage_events(void *const *events, int n);

/*
 * ---- Expert parallelism ---------------------------------------------------
 *
 * The layer spread over n_ranks GPUs, rank r holding the routed experts
 * [r E_l, (r+1) E_l) (E_l = E / n_ranks) and a copy of the router and shared
 * experts: each rank routes its own tokens, sends each chosen (token, expert)
 * row to the rank that owns the expert, the owners run their experts on what
 * they received, and the weighted results come back to be summed
 * ("大模型工程（一）：Transformer 到 MoE", section "混合专家：更多参数，相同 FLOPs":
 * experts on different GPUs, token exchange by all-to-all over NVLink; its
 * Mixtral / Qwen3-MoE / DeepSeek-V3 comparison: expert groups per GPU).  The
 * two exchanges are the caller's (NCCL all-to-all); these calls are the
 * compute around them.  bf16 layers only (else MOE_ERR_UNSUPPORTED); d a
 * multiple of 256 and inter of 128.  Results equal moe_forward's: the same
 * routing, the same fp32-accumulated expert GEMMs, each routed row scaled by
 * its gate weight and rounded once to bf16, and the same fixed-order sum.
 *
 * moe_dispatch_workspace_bytes -- scratch bytes of moe_dispatch (0 if invalid).
 */
MOE_API size_t moe_dispatch_workspace_bytes(int T, int E, int k);

/*
 * moe_dispatch -- routing (as moe_route_ex) and the permutation of this
 * rank's T tokens into expert-contiguous rows.
 *   topk_idx, topk_w  device int32 / f32 [T, k] out: the routing
 *   counts     device int32 [E] out: rows for each expert (destination rank
 *              of expert e: e / E_l, so rank q's rows are the contiguous
 *              block of experts [q E_l, (q+1) E_l))
 *   x_perm     device bf16 [T*k, d] out: row r is x of the token of slot
 *              t*k + j, rows ordered by expert, inside an expert by token
 *   w_perm     device f32 [T*k] out: the gate weight w_j of row r
 *   slot_row   device int32 [T*k] out: slot t*k + j -> its row r
 *   workspace  device, moe_dispatch_workspace_bytes, 256-byte aligned
 * Other arguments and errors as moe_route_ex.  T = 0 zeroes counts.
 */
MOE_API int moe_dispatch(const void *x, const void *W_router, int T, int d, int E, int k,
                         int n_group, int topk_group, int in_dt, int gate,
                         const float *expert_bias, int32_t *topk_idx, float *topk_w,
                         int32_t *counts, void *x_perm, float *w_perm, int32_t *slot_row,
                         void *workspace, size_t workspace_bytes, void *stream);

/* moe_experts_workspace_bytes -- scratch bytes of moe_experts_forward for R
 * received rows (0 if invalid). */
MOE_API size_t moe_experts_workspace_bytes(int R, int d, int E_local, int inter);

/*
 * moe_experts_forward -- the local experts on the rows this rank received.
 *   x_rows       device bf16 [R, d]: the received rows, grouped by source
 *                rank (0, 1, ...), inside a source by local expert, in the
 *                source's order (the concatenation of the sources' x_perm
 *                blocks for this rank)
 *   w_rows       device f32 [R]: the gate weight of each received row
 *   recv_counts  device int32 [n_src, E_local]: rows from each source for
 *                each local expert (sum = R; a sum above R computes nothing
 *                and sets MOE_ERR_DEVICE in the status word)
 *   W_gate_up    device bf16 [E_local, 2*inter, d], W_down [E_local, d, inter]:
 *                this rank's experts
 *   y_rows       device bf16 [R, d] out: row i = w_rows[i] * SwiGLU expert
 *                of row i (fp32 accumulation, rounded once), in the receive
 *                order, ready to be sent back
 *   workspace    moe_experts_workspace_bytes(R, ...), 256-byte aligned; its
 *                first 256 bytes are the status word (moe_get_device_status)
 * Limits: n_src * E_local <= 2048.  R = 0 queues nothing.
 */
MOE_API int moe_experts_forward(const void *x_rows, const float *w_rows,
                                const int32_t *recv_counts, int n_src, int R,
                                const void *W_gate_up, const void *W_down, int d, int E_local,
                                int inter, int in_dt, void *y_rows, void *workspace,
                                size_t workspace_bytes, void *stream);

/* moe_shared_workspace_bytes -- scratch bytes of moe_shared_forward. */
MOE_API size_t moe_shared_workspace_bytes(int T, int d, int inter, int n_shared);

/*
 * moe_shared_forward -- the n_shared >= 1 shared experts on T tokens:
 * y_shared = sum_s SwiGLU_shared_s(x), device f32 [T, d] out (W_shared laid
 * out as for moe_forward).  Independent of the exchange: it can run on
 * another stream while the rows are in flight.
 */
MOE_API int moe_shared_forward(const void *x, const void *W_shared, int T, int d, int inter,
                               int n_shared, int in_dt, float *y_shared, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * moe_combine -- y[t] = shared[t] + rows[slot_row[t*k + 0]] + ... +
 * rows[slot_row[t*k + k-1]] in fp32, in that order (bitwise reproducible).
 *   rows      device bf16 [n_rows, d]: the rows sent back, in x_perm order
 *   slot_row  device int32 [T*k]: moe_dispatch's slot_row
 *   shared    device f32 [T, d] or NULL (no shared experts)
 *   y         device out_dt [T, d] out
 *   status_ws device workspace whose status word receives MOE_ERR_DEVICE
 *             for a slot_row entry outside [0, n_rows), or NULL
 */
MOE_API int moe_combine(const void *rows, int n_rows, const int32_t *slot_row,
                        const float *shared, int T, int d, int k, int out_dt, void *y,
                        void *status_ws, void *stream);

/* moe_status_string -- static text for a status code. */
MOE_API const char *moe_status_string(int status);

/* moe_version -- ABI version of this header (1). */
MOE_API int moe_version(void);

#endif /* MOE_B200_H */
