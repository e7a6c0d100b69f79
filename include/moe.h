/*
 * moe.h -- C ABI of libmoe, the forward pass of a Mixture-of-Experts FFN
 * layer on one NVIDIA B200 (sm_100a).
 *
 * The layer (sources are named by page title and section):
 *   router      h = x W_r (+ per-expert logit offset), fp32 scores:
 *               softmax over the E experts ("Mixture-of-Experts", Vector
 *               Institute post, router section; "Fine-tuning and serving MoE
 *               models", How an MoE layer actually works: fp32 router softmax),
 *               or sigmoid with a selection-only bias ("Fine-Tuning Mixture of
 *               Experts (MoE) Models: Router Optimization Techniques", How It
 *               Works 2, auxiliary-loss-free routing).
 *   top-k       the k experts with the largest score (+ selection bias), gates
 *               from the full softmax (Eq. moe-output) or renormalised over
 *               the selected experts; sigmoid gates s_i / sum_selected s.
 *   capacity    an expert keeps at most floor(c * k * T / E) assignments, the
 *               earliest tokens first; the rest are dropped (contribute zero)
 *               (Vector Institute post, expert-capacity paragraph; "Mixture of
 *               Experts" tutorial, The capacity factor formula).
 *   experts     GELU: W2 GELU(W1 x + b1) + b2 (Linear-GELU-Linear with biases);
 *               SwiGLU: W_down (SiLU(W_gate x) * (W_up x)) (Router Optimization
 *               page, What Is It?); optional always-on shared expert (weight 1).
 *   combine     y_t = sum_s gate[t,s] * E_{idx[t,s]}(x_t) (+ shared(x_t)).
 *   balance     f_e = counts_e / (T k), P_e = mean_t score_e(t),
 *               L = E * sum_e f_e P_e (Eq. balance; Router Optimization page,
 *               How It Works 1).
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers owned by the caller, except the
 *     moe_config pointer and the out-pointers of moe_get_device_status, which
 *     are host pointers.  The library never allocates or frees device memory;
 *     scratch comes from the caller's workspace `ws` of `ws_bytes` bytes
 *     (moe_workspace_size() bytes suffice for every entry point), aligned to
 *     256 bytes.  The first 256 bytes of ws hold a device status word; zero
 *     them once with moe_workspace_init() before first use.
 *   - Calls are asynchronous on `stream` and never synchronise the device
 *     (moe_get_device_status and moe_workspace_init excepted, see there).
 *   - Arguments are checked on the host before any launch; a bad argument
 *     returns MOE_ERR_INVALID_ARG (or MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE)
 *     and launches nothing.  A failed launch returns MOE_ERR_CUDA.  Problems
 *     only the device can see (an expert id out of range, a row index out of
 *     range, a pipeline wait that ran past its time limit) are recorded in the
 *     workspace status word and read back by moe_get_device_status.
 *   - Layouts are row-major.  x, y and expert weights are in cfg->dtype
 *     (bf16 or fp32); router weights, biases, gates, logits and statistics are
 *     fp32; the loss is fp64.  Expert weights use the nn.Linear [out, in]
 *     layout stacked over experts.
 *   - bf16 layers run the expert GEMMs on tcgen05 tensor cores with fp32
 *     accumulation; the hidden activation H and the gate-scaled expert
 *     outputs are rounded to bf16, the combine accumulates in fp32 and rounds
 *     once.  fp32 layers run everything in fp32.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, k > E, ...   */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but not built: E > 256, d % 8 != 0, ... */
    MOE_ERR_WORKSPACE = 3,     /* ws_bytes below moe_workspace_size() or ws misaligned */
    MOE_ERR_CUDA = 4,          /* a CUDA call failed (launch, tensor map, copy)  */
    MOE_ERR_TIMEOUT = 5,       /* device: a pipeline wait ran past its limit     */
    MOE_ERR_DEVICE_BOUNDS = 6  /* device: an expert id or row index out of range */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_ACT_GELU_BIAS = 0, MOE_ACT_SWIGLU = 1 } moe_act;
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score;

typedef struct {
    int32_t T;                 /* tokens, >= 0                                    */
    int32_t d_model;           /* >= 8 and a multiple of 8                        */
    int32_t E;                 /* routed experts, 1..256                          */
    int32_t d_ff;              /* routed expert hidden width, >= 8, multiple of 8 */
    int32_t top_k;             /* 1..E                                             */
    int32_t dtype;             /* moe_dtype of x, y and expert weights            */
    int32_t act;               /* moe_act                                          */
    int32_t score;             /* moe_score                                        */
    int32_t renorm;            /* softmax: 1 renormalise gates over the top-k,
                                  0 keep the full-softmax probabilities           */
    float capacity_factor;     /* <= 0: no capacity limit                          */
    int32_t d_ff_shared;       /* shared expert hidden width; 0: none; else a
                                  multiple of 8 (same activation as the routed
                                  experts, no biases)                              */
} moe_config;

/* Bytes of workspace every entry point below can run in (0 on a bad config). */
MOE_API size_t moe_workspace_size(const moe_config *cfg);

/* Per-expert capacity floor(capacity_factor * top_k * T / E) computed in
 * double, or -1 when capacity_factor <= 0 (or cfg is invalid).              */
MOE_API int32_t moe_capacity(const moe_config *cfg);

/* Rows of the per-block partial score sums written by moe_router_topk
 * (the `psum` array is [moe_router_blocks(cfg), E] fp32).                   */
MOE_API int32_t moe_router_blocks(const moe_config *cfg);

/* Rows of y_perm: T*top_k routed rows, plus T shared-expert rows when
 * d_ff_shared > 0 (routed row r of expert e lies in [offsets[e], offsets[e+1]),
 * shared row of token t is T*top_k + t).                                     */
MOE_API int64_t moe_perm_rows(const moe_config *cfg);

/* Zero the workspace status header (an async 256-byte memset on `stream`). */
MOE_API moe_status moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Frozen router (inference with fixed router weights).  For bf16 layers the
 * router splits W_r into three bf16 terms inside the workspace on every call
 * (an exact split, one small launch).  moe_router_freeze does that split now
 * and marks the workspace: later moe_router_topk / moe_forward /
 * moe_forward_fp8 calls on the same workspace with the same W_r pointer (and
 * the same d_model and E) skip it.  The mark is kept on the host, per
 * workspace address; a call with other router weights re-splits and clears
 * it, and so does moe_workspace_init.  After changing the values at W_r in
 * place, call moe_router_freeze again (or moe_workspace_init).  fp32 layers:
 * nothing to prepare, returns MOE_OK.  Wr [d_model, E] fp32 device pointer;
 * stream-ordered like the other calls.                                      */
MOE_API moe_status moe_router_freeze(const moe_config *cfg, const float *Wr, void *ws, size_t ws_bytes,
                                     moe_stream_t stream);

/* Router + score + top-k + gates (see the header comment for the sources).
 *   x          [T, d_model]  cfg->dtype
 *   Wr         [d_model, E]  fp32
 *   logit_bias [E] fp32 or NULL: added to every logit (enters scores and
 *              selection, i.e. a router Linear with bias)
 *   sel_bias   [E] fp32 or NULL: added to the score for the selection only
 *              (softmax: to the logit; sigmoid: to sigmoid(logit)); gates and
 *              statistics never see it
 *   idx        [T, top_k] int32 out: chosen experts, best first; equal keys
 *              go to the lower expert id
 *   gate       [T, top_k] fp32 out
 *   logits_out [T, E] fp32 out or NULL: h (with logit_bias)
 *   psum       [moe_router_blocks(cfg), E] fp32 out: per-block sums over the
 *              block's tokens of the score whose token-mean is P_e (softmax
 *              probability, or sigmoid normalised over all E experts)        */
MOE_API moe_status moe_router_topk(const moe_config *cfg, const void *x, const float *Wr,
                           const float *logit_bias, const float *sel_bias,
                           int32_t *idx, float *gate, float *logits_out, float *psum,
                           void *ws, size_t ws_bytes, moe_stream_t stream);

/* Counting, capacity and permutation into expert-contiguous order, stable by
 * token id within each expert (rows in (expert, token) order).
 *   x          [T, d_model] cfg->dtype;  idx [T, top_k] int32;  gate [T, top_k] fp32
 *   counts     [E] int32 out: assignments per expert before capacity
 *   kept       [E] int32 out: min(counts, capacity)
 *   offsets    [E+1] int32 out: exclusive prefix sum of kept
 *   row_of     [T, top_k] int32 out: row of each assignment, -1 when dropped
 *   row_token  [T*top_k] int32 out: token of each row (first offsets[E] valid)
 *   row_gate   [T*top_k] fp32 out: gate of each row
 *   x_perm     [T*top_k, d_model] cfg->dtype out: x rows in row order, or NULL
 *              to write the row tables only
 *   n_dropped  device int32 out (may be NULL): assignments dropped by capacity
 * An expert id outside [0, E) is recorded as MOE_ERR_DEVICE_BOUNDS and the
 * assignment is treated as dropped.                                          */
MOE_API moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *idx,
                       const float *gate, int32_t *counts, int32_t *kept, int32_t *offsets,
                       int32_t *row_of, int32_t *row_token, float *row_gate, void *x_perm,
                       int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream);

/* All experts as one grouped GEMM pair.  For every expert e and every row r
 * in [offsets[e], offsets[e+1]):
 *   GELU:   y_perm[r] = row_gate[r] * (W2[e] GELU(W1[e] x_perm[r] + b1[e]) + b2[e])
 *   SwiGLU: y_perm[r] = row_gate[r] * (W2[e] (SiLU(W1[e] x_perm[r]) * (Wu[e] x_perm[r])))
 * and, with a shared expert, for every token t:
 *   y_perm[T*top_k + t] = Wsh_d (act(Wsh_g x[t]) [* (Wsh_u x[t])])
 *   W1  [E, d_ff, d_model] (GELU W1 or SwiGLU W_gate);  Wu [E, d_ff, d_model]
 *       (SwiGLU W_up; NULL for GELU);  W2 [E, d_model, d_ff] (W2 / W_down)
 *   b1  [E, d_ff] fp32, b2 [E, d_model] fp32 (GELU; either may be NULL)
 *   x, Wsh_g [d_ff_shared, d_model], Wsh_u (SwiGLU), Wsh_d [d_model, d_ff_shared]:
 *       shared expert (NULL when d_ff_shared == 0)
 *   y_perm [moe_perm_rows(cfg), d_model] cfg->dtype out; rows past offsets[E]
 *       and before the shared rows are left untouched.                      */
MOE_API moe_status moe_grouped_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                           const float *row_gate, const void *W1, const float *b1,
                           const void *Wu, const void *W2, const float *b2,
                           const void *x, const void *Wsh_g, const void *Wsh_u,
                           const void *Wsh_d, void *y_perm,
                           void *ws, size_t ws_bytes, moe_stream_t stream);

/* y[t] = sum over s with row_of[t,s] >= 0 of y_perm[row_of[t,s]]  (+ the
 * shared row T*top_k + t), accumulated in fp32 in slot order and rounded once.
 *   y_perm [moe_perm_rows(cfg), d_model], row_of [T, top_k], y [T, d_model].
 * A row index >= T*top_k is recorded as MOE_ERR_DEVICE_BOUNDS and skipped. */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *row_of,
                       void *y, void *ws, size_t ws_bytes, moe_stream_t stream);

/* f_e = counts_e / (T*top_k), P_e = (sum_b psum[b,e]) / T (fp64 sums),
 * loss = E * sum_e f_e P_e (fp64).  f, P [E] fp32 out; loss device fp64 out. */
MOE_API moe_status moe_balance_stats(const moe_config *cfg, const int32_t *counts, const float *psum,
                             float *f, float *P, double *loss, moe_stream_t stream);

/* The whole layer on one stream: router, permute, grouped FFN, combine,
 * balance statistics.  Inputs as above; outputs:
 *   y [T, d_model] cfg->dtype; idx, gate [T, top_k]; counts [E] int32;
 *   f, P [E] fp32; loss device fp64; logits_out [T, E] fp32 or NULL;
 *   n_dropped device int32 or NULL.
 * Everything else lives in ws (moe_workspace_size(cfg) bytes).             */
MOE_API moe_status moe_forward(const moe_config *cfg, const void *x, const float *Wr,
                       const float *logit_bias, const float *sel_bias,
                       const void *W1, const float *b1, const void *Wu, const void *W2,
                       const float *b2, const void *Wsh_g, const void *Wsh_u, const void *Wsh_d,
                       void *y, int32_t *idx, float *gate, int32_t *counts, float *f, float *P,
                       double *loss, float *logits_out, int32_t *n_dropped,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Where moe_forward / moe_forward_fp8 leave their intermediate results inside
 * a workspace: the dispatch tables (rows in (expert, token) order, see
 * moe_permute), the packed input rows, the hidden activation and the gated
 * expert outputs.  They are valid after the forward pass on the workspace's
 * stream has completed and until the next call that uses the workspace.  A
 * host-only call: it computes addresses (device pointers into ws) and launches
 * nothing.  Returns MOE_ERR_INVALID_ARG on a bad config or NULL out,
 * MOE_ERR_WORKSPACE when ws is NULL, misaligned or smaller than
 * moe_workspace_size(cfg).                                                  */
typedef struct {
    int32_t *kept;        /* [E]            min(counts, capacity)                     */
    int32_t *offsets;     /* [E+1]          exclusive prefix sum of kept              */
    int32_t *row_of;      /* [T, top_k]     row of each assignment, -1 when dropped   */
    int32_t *row_token;   /* [T*top_k]      token of each row (first offsets[E] valid) */
    float *row_gate;      /* [T*top_k]      gate of each row                          */
    void *x_perm;         /* [T*top_k, d_model] packed x rows (e4m3 codes with FP8 experts) */
    void *H;              /* [moe_perm_rows(cfg), hF] hidden activation, hF = h_stride */
    void *y_perm;         /* [moe_perm_rows(cfg), d_model] gate-scaled expert outputs */
    int64_t h_stride;     /* row stride of H in elements: max(d_ff, d_ff_shared)      */
} moe_ws_view;
MOE_API moe_status moe_workspace_view(const moe_config *cfg, void *ws, size_t ws_bytes, moe_ws_view *out);

/* ---- Backward pass ------------------------------------------------------
 * The layer is trained ("Fine-Tuning Mixture of Experts (MoE) Models: Router
 * Optimization Techniques", The Fine-Tuning Router Challenge and How It Works
 * 1: the router and the experts learn from the task loss plus the balance
 * loss).  moe_backward gives the gradient of
 *     ell = sum_t <dy_t, y_t> + alpha * L_aux
 * (dy: the gradient of the task loss with respect to the layer output y;
 * L_aux = E sum_e f_e P_e) with respect to x, W_r, the logit offset and every
 * expert's weights and biases, shared expert included.  The expert choice,
 * the capacity ranks and the counts f_e are piecewise constant in the inputs
 * and carry no gradient; the selection bias gets none.
 *   - Run it after moe_forward on the same stream with the same cfg, inputs
 *     and workspace `fwd_ws` (its dispatch tables, packed rows and hidden
 *     activation are read from there; the expert pre-activations are
 *     recomputed, unless the forward pass was moe_forward_train with this
 *     backward workspace), passing the forward's outputs idx, gate, counts
 *     and its router logits (moe_forward's logits_out, required here).
 *   - bf16 layers with d_model, d_ff and d_ff_shared multiples of 64 (else
 *     MOE_ERR_UNSUPPORTED).  dy and dx [T, d_model] bf16; every other
 *     gradient fp32 in the layout of its parameter: dWr [d_model, E],
 *     dlogit_bias [E] (may be NULL), dW1 / dWu [E, d_ff, d_model], db1 [E,
 *     d_ff] and db2 [E, d_model] (GELU; may be NULL), dW2 [E, d_model, d_ff],
 *     dWsh_g / dWsh_u [d_ff_shared, d_model], dWsh_d [d_model, d_ff_shared].
 *     Gradients are written, not accumulated.
 *   - Contractions run on the tensor cores with bf16 operands (dy scaled by
 *     the gates, the recomputed pre-activations, their gradients, dh) and
 *     fp32 accumulation; the rest in fp32.
 *   - ws: moe_backward_workspace_size(cfg) bytes of scratch, 256-byte aligned
 *     (0 on a bad or unsupported config).  Device errors land in fwd_ws's
 *     status word.                                                          */
MOE_API size_t moe_backward_workspace_size(const moe_config *cfg);
MOE_API moe_status moe_backward(const moe_config *cfg, const void *x, const float *Wr, const void *W1,
                                const float *b1, const void *Wu, const void *W2, const float *b2,
                                const void *Wsh_g, const void *Wsh_u, const void *Wsh_d,
                                const int32_t *idx, const float *gate, const float *logits, const int32_t *counts,
                                const void *dy, float alpha, void *dx, float *dWr, float *dlogit_bias,
                                float *dW1, float *db1, float *dWu, float *dW2, float *db2,
                                float *dWsh_g, float *dWsh_u, float *dWsh_d,
                                void *fwd_ws, size_t fwd_ws_bytes, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Training forward pass: moe_forward (same arguments, same results) that
 * also leaves the expert pre-activations -- G and U of the SwiGLU experts,
 * W_1 x + b_1 of the GELU experts, shared expert included, in bf16 as the
 * first GEMM computed them -- inside `bwd_ws`, the workspace the following
 * moe_backward will use, so that call skips their recomputation (two grouped
 * GEMMs, about a sixth of its time on a Qwen3-shaped layer).
 *   - bwd_ws: moe_backward_workspace_size(cfg) bytes, 256-byte aligned; the
 *     layer must be one moe_backward supports (else MOE_ERR_UNSUPPORTED).
 *   - The hand-over is recorded on the host: the next moe_backward with
 *     workspace bwd_ws, forward workspace ws and an identical cfg uses the
 *     saved values; any call that rewrites ws's packed rows or hidden
 *     activation (moe_forward*, moe_grouped_ffn*, moe_permute) or
 *     reinitialises ws or bwd_ws (moe_workspace_init) cancels the record, and
 *     moe_backward recomputes.  Calls are taken in host order, as the
 *     stream runs them.                                                     */
MOE_API moe_status moe_forward_train(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                                     const float *sel_bias, const void *W1, const float *b1, const void *Wu,
                                     const void *W2, const float *b2, const void *Wsh_g, const void *Wsh_u,
                                     const void *Wsh_d, void *y, int32_t *idx, float *gate, int32_t *counts, float *f,
                                     float *P, double *loss, float *logits_out, int32_t *n_dropped, void *ws,
                                     size_t ws_bytes, void *bwd_ws, size_t bwd_ws_bytes, moe_stream_t stream);

/* ---- Expert parallelism -------------------------------------------------
 * The experts sharded over R ranks, each rank holding E / R of them ("Fine-
 * Tuning Mixture of Experts (MoE) Models: Router Optimization Techniques",
 * Why It Matters 2, token dispatch and gather, and Architecture & Distributed
 * Execution; "Mixture-of-Experts", Vector Institute post, expert-parallelism
 * paragraph): every rank routes and permutes its own tokens (moe_router_topk,
 * moe_permute), so the rows bound for rank j are the contiguous range of j's
 * experts; the rows travel to their experts' rank (an all-to-all of
 * variable-size blocks), run through that rank's experts, travel back and are
 * combined where they came from (moe_combine).  The entry point below is the
 * middle step: the grouped FFN over the rows a rank received.
 *
 * moe_ep_grouped_ffn: cfg describes the local experts: E = experts held by
 * this rank, d_model, d_ff, dtype, act (T, top_k, score, renorm, capacity and
 * d_ff_shared are not used; run a shared expert with moe_grouped_ffn).  The
 * received rows come as n_src blocks (one per source rank), each holding the
 * source's rows for local expert 0, 1, ..., E-1 in turn, so there are
 * n_src * E row groups (at most 256): group g = src * E + e holds rows
 * group_offsets[g] .. group_offsets[g+1] and uses local expert e:
 *   y_rows[r] = row_gate[r] * expert_e(x_rows[r])   (bf16 or fp32 as in
 *   moe_grouped_ffn: GELU with b1 / b2, or SwiGLU)
 *   group_offsets [n_src*E + 1] int32 device, non-decreasing, from 0 to at
 *       most max_rows;  x_rows, y_rows [max_rows, d_model];  row_gate [max_rows]
 *   W1, Wu [E, d_ff, d_model]; W2 [E, d_model, d_ff]; b1 [E, d_ff], b2
 *       [E, d_model] (GELU, may be NULL): the local experts' slices.
 * Rows past group_offsets[n_src*E] are left untouched.  The workspace (its
 * first 256 bytes a status word, as for the other entry points) holds the
 * hidden activation: moe_ep_workspace_size(cfg, n_src, max_rows) bytes (0 on
 * a bad argument).                                                         */
MOE_API size_t moe_ep_workspace_size(const moe_config *cfg, int32_t n_src, int64_t max_rows);
MOE_API moe_status moe_ep_grouped_ffn(const moe_config *cfg, int32_t n_src, const int32_t *group_offsets,
                                      int64_t max_rows, const void *x_rows, const float *row_gate,
                                      const void *W1, const float *b1, const void *Wu, const void *W2,
                                      const float *b2, void *y_rows, void *ws, size_t ws_bytes,
                                      moe_stream_t stream);

/* ---- FP8 (e4m3) experts -----------------------------------------------
 * Quantized experts for serving ("Fine-tuning and serving MoE models",
 * Serving: throughput does not scale the way you expect, consequences for
 * capacity planning: quantize the experts to FP8 since memory binds).  The
 * expert GEMMs run on the tensor cores with e4m3 x e4m3 products and fp32
 * accumulation (W8A8):
 *   e4m3: OCP 8-bit float E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa
 *     bits, no infinities, largest finite 448), one byte per element.
 *   weights: e4m3 codes in the nn.Linear [out, in] layout stacked over
 *     experts, one fp32 scale per output channel: W[e][n][j] = code * scale[e][n].
 *   activations: x and each expert's hidden activation H are quantized per
 *     row on the device (moe_quantize_rows_e4m3: scale = max|v| / 448, code =
 *     e4m3(v * 448 / max|v|), round to nearest even, saturating); H is formed
 *     in bf16 first, as in the bf16 layer.
 *   Everything else (router, dispatch, gates, combine, statistics) is the
 *   bf16 layer's.  Only bf16 layers (cfg->dtype == MOE_BF16) with d_model,
 *   d_ff and d_ff_shared multiples of 16 (else MOE_ERR_UNSUPPORTED).
 * All pointers in the struct are device pointers (codes 16-byte aligned,
 * scales 4-byte aligned); the struct itself is a host object read during
 * the call.                                                                 */
typedef struct {
    const uint8_t *W1;    const float *W1_scale;     /* [E, d_ff, d_model], [E, d_ff]   */
    const uint8_t *Wu;    const float *Wu_scale;     /* SwiGLU W_up (same shapes), else NULL */
    const uint8_t *W2;    const float *W2_scale;     /* [E, d_model, d_ff], [E, d_model] */
    const uint8_t *Wsh_g; const float *Wsh_g_scale;  /* shared expert [d_ff_shared, d_model],
                                                        [d_ff_shared], or NULL          */
    const uint8_t *Wsh_u; const float *Wsh_u_scale;  /* SwiGLU shared W_up, or NULL      */
    const uint8_t *Wsh_d; const float *Wsh_d_scale;  /* [d_model, d_ff_shared], [d_model] */
} moe_fp8_experts;

/* Per-row e4m3 quantization of a bf16 matrix: for each of `rows` rows of
 * `cols` values (row stride ld_in elements), amax = max |v| (fp32),
 * codes[r, j] = e4m3(v_j * (448 / amax)) (0 for a zero row; correctly rounded
 * fp32 quotient and product, nearest-even conversion, saturating at 448),
 * scale[r] = amax / 448.  codes: row stride ld_out bytes.  cols, ld_in and
 * ld_out multiples of 8; `in` 16-byte aligned, `codes` 8-byte aligned.     */
MOE_API moe_status moe_quantize_rows_e4m3(const void *in, int64_t rows, int32_t cols, int64_t ld_in,
                                          uint8_t *codes, int64_t ld_out, float *scale, moe_stream_t stream);

/* moe_grouped_ffn with FP8 experts.  x8_perm [T*top_k, d_model] e4m3 codes of
 * the packed rows with their row scales x8_perm_scale [T*top_k]; x8 / x8_scale
 * the codes and scales of x [T, d_model] (the shared expert's input, NULL
 * without one); b1, b2 fp32 as in moe_grouped_ffn.  Output y_perm as in
 * moe_grouped_ffn (bf16).  H, its codes and scales live in ws.             */
MOE_API moe_status moe_grouped_ffn_fp8(const moe_config *cfg, const uint8_t *x8_perm, const float *x8_perm_scale,
                                       const int32_t *offsets, const float *row_gate, const moe_fp8_experts *w,
                                       const float *b1, const float *b2, const uint8_t *x8, const float *x8_scale,
                                       void *y_perm, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward with FP8 experts: router on the bf16 x, then x quantized per
 * row, the permute of its codes, the e4m3 grouped FFN, combine, statistics.
 * Arguments and outputs as in moe_forward, the expert weights in *w.       */
MOE_API moe_status moe_forward_fp8(const moe_config *cfg, const void *x, const float *Wr,
                                   const float *logit_bias, const float *sel_bias, const moe_fp8_experts *w,
                                   const float *b1, const float *b2, void *y, int32_t *idx, float *gate,
                                   int32_t *counts, float *f, float *P, double *loss, float *logits_out,
                                   int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream);

/* ---- Block-scaled (MX) FP8 experts --------------------------------------
 * The block-scaled form of quantized experts ("Fine-tuning and serving MoE
 * models", Serving: quantize the experts since memory binds), laid out as OCP
 * microscaling (MX) FP8: along the contraction dimension of every matrix,
 * each run of 32 values shares one power-of-two scale 2^X stored as the byte
 * X + 127 (E8M0), each value one e4m3 code.  The expert GEMMs run as
 * tcgen05.mma.kind::mxf8f6f4.block_scale (the hardware applies both
 * operands' block scales; fp32 accumulation).
 *   quantization (moe_quantize_rows_mx, and H on the device): per block of
 *     32 values, amax = max |v|, X = floor(log2 amax) - 8 clamped to
 *     [-127, 127] (-127 for a zero or subnormal amax), code = e4m3(v * 2^-X),
 *     round to nearest even, saturating at 448 (values in (448, 512) * 2^X
 *     saturate).
 *   weights: codes in the nn.Linear [out, in] layout stacked over experts,
 *     scale bytes [.., out, in / 32] with rows of sld bytes.
 *   activations: x per token row along d_model; H (formed in bf16 first, as
 *     in the bf16 layer) per row along d_ff.
 * Every scale array (x, weights) has rows of sld bytes: sld a multiple of 16
 * and at least d_model / 32, d_ff / 32 and d_ff_shared / 32.  Only bf16
 * layers with d_model, d_ff and d_ff_shared multiples of 128 and E <= 256
 * (else MOE_ERR_UNSUPPORTED).  All pointers in the struct are device
 * pointers, codes and scale arrays 16-byte aligned; the struct is read
 * during the call.                                                          */
typedef struct {
    const uint8_t *W1;    const uint8_t *W1_scale;      /* [E, d_ff, d_model], [E, d_ff, sld]     */
    const uint8_t *Wu;    const uint8_t *Wu_scale;      /* SwiGLU W_up (same shapes), else NULL   */
    const uint8_t *W2;    const uint8_t *W2_scale;      /* [E, d_model, d_ff], [E, d_model, sld]  */
    const uint8_t *Wsh_g; const uint8_t *Wsh_g_scale;   /* shared expert [d_ff_shared, d_model],
                                                           [d_ff_shared, sld], or NULL            */
    const uint8_t *Wsh_u; const uint8_t *Wsh_u_scale;   /* SwiGLU shared W_up, or NULL            */
    const uint8_t *Wsh_d; const uint8_t *Wsh_d_scale;   /* [d_model, d_ff_shared], [d_model, sld] */
    int32_t sld;                                        /* scale row stride in bytes             */
} moe_mx_experts;

/* MX quantization of a bf16 matrix: `rows` rows of `cols` values (row stride
 * ld_in elements, cols a multiple of 32) -> codes [rows, ld_out bytes] and
 * one scale byte per 32 values, scales [rows, ld_scale bytes] (ld_scale >=
 * cols / 32).  ld_in, ld_out multiples of 8; in 16-byte, codes 8-byte
 * aligned.  The codes are a function of the bf16 values alone (the scaling
 * by 2^-X is exact).                                                        */
MOE_API moe_status moe_quantize_rows_mx(const void *in, int64_t rows, int32_t cols, int64_t ld_in,
                                        uint8_t *codes, int64_t ld_out, uint8_t *scales, int64_t ld_scale,
                                        moe_stream_t stream);

/* moe_grouped_ffn with MX experts (moe_forward_mx below runs the whole layer):
 * x8_perm [T*top_k, d_model] codes of the
 * packed rows with their scales xs_perm [T*top_k, sld]; x8 / xs the codes and
 * scales of x [T, d_model] (the shared expert's input; NULL without one); b1,
 * b2 fp32 as in moe_grouped_ffn.  Output y_perm [moe_perm_rows(cfg), d_model]
 * bf16 as in moe_grouped_ffn (routed rows past offsets[E] untouched, the
 * shared expert's rows from T*top_k on).  The workspace (its first 256 bytes
 * a status word) holds H in bf16, its MX codes and scales:
 * moe_grouped_ffn_mx_workspace_size(cfg, sld) bytes, 256-byte aligned (0 on
 * a bad or unsupported configuration).                                      */
MOE_API size_t moe_grouped_ffn_mx_workspace_size(const moe_config *cfg, int32_t sld);
/* moe_forward with MX experts: router on the bf16 x, x quantized to MX codes
 * per token (the codes permuted with the rows, the scale rows gathered after
 * them), the MX grouped FFN, combine, statistics.  Arguments and outputs as
 * in moe_forward, the expert weights in *w; ws is the layer's workspace
 * (moe_workspace_size) and mx_ws a second one of
 * moe_grouped_ffn_mx_workspace_size(cfg, w->sld) bytes, 256-byte aligned,
 * for x's and H's codes and scale rows.  Device status goes to ws.          */
MOE_API moe_status moe_forward_mx(const moe_config *cfg, const void *x, const float *Wr,
                                  const float *logit_bias, const float *sel_bias, const moe_mx_experts *w,
                                  const float *b1, const float *b2, void *y, int32_t *idx, float *gate,
                                  int32_t *counts, float *f, float *P, double *loss, float *logits_out,
                                  int32_t *n_dropped, void *ws, size_t ws_bytes, void *mx_ws, size_t mx_ws_bytes,
                                  moe_stream_t stream);
MOE_API moe_status moe_grouped_ffn_mx(const moe_config *cfg, const uint8_t *x8_perm, const uint8_t *xs_perm,
                                      const int32_t *offsets, const float *row_gate, const moe_mx_experts *w,
                                      const float *b1, const float *b2, const uint8_t *x8, const uint8_t *xs,
                                      void *y_perm, void *ws, size_t ws_bytes, moe_stream_t stream);

/* ---- INT4 weight-only experts --------------------------------------------
 * Weight-only INT4 experts ("Fine-tuning and serving MoE models", Serving:
 * weight-only INT4 / FP8 experts, torchao's INT4 weight-only path, once
 * memory binds): every expert weight matrix [out, in] holds signed 4-bit
 * integers q in [-8, 7], two per byte (the low nibble the even input; a
 * nibble stores q + 8), with one bf16 scale per output row and group of 128
 * consecutive inputs; a weight's value is bf16(q * s) (nearest, ties to
 * even).  Activations stay bf16 (the bf16 layer's x and H); the tensor cores
 * run bf16 x bf16 products with fp32 accumulation on weights decoded into
 * shared memory stage by stage.
 * Scale arrays have rows of sld bytes: sld a multiple of 16 and at least
 * 2 * d_model / 128, 2 * d_ff / 128 and 2 * d_ff_shared / 128.  Only bf16
 * layers with d_model, d_ff and d_ff_shared multiples of 128 and E <= 256
 * (else MOE_ERR_UNSUPPORTED).  All pointers in the struct are device
 * pointers, 16-byte aligned; the struct is read during the call.            */
typedef struct {
    const uint8_t *W1;    const uint8_t *W1_scale;      /* [E, d_ff, d_model / 2], [E, d_ff, sld] */
    const uint8_t *Wu;    const uint8_t *Wu_scale;      /* SwiGLU W_up (same shapes), else NULL   */
    const uint8_t *W2;    const uint8_t *W2_scale;      /* [E, d_model, d_ff / 2], [E, d_model, sld] */
    const uint8_t *Wsh_g; const uint8_t *Wsh_g_scale;   /* shared expert, same layouts, or NULL   */
    const uint8_t *Wsh_u; const uint8_t *Wsh_u_scale;
    const uint8_t *Wsh_d; const uint8_t *Wsh_d_scale;
    int32_t sld;                                        /* scale row stride in bytes             */
} moe_w4_experts;

/* moe_grouped_ffn with INT4 weight-only experts: arguments and output as in
 * moe_grouped_ffn (x_perm, x bf16), the experts in *w; ws is the layer's
 * workspace (moe_workspace_size: its hidden-activation region holds H).      */
MOE_API moe_status moe_grouped_ffn_w4(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                                      const float *row_gate, const moe_w4_experts *w, const float *b1,
                                      const float *b2, const void *x, void *y_perm, void *ws, size_t ws_bytes,
                                      moe_stream_t stream);
/* moe_forward with INT4 weight-only experts: the bf16 layer (router,
 * permute, combine, statistics) around the INT4 grouped FFN.  Arguments and
 * outputs as in moe_forward, the expert weights in *w.                      */
MOE_API moe_status moe_forward_w4(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                                  const float *sel_bias, const moe_w4_experts *w, const float *b1, const float *b2,
                                  void *y, int32_t *idx, float *gate, int32_t *counts, float *f, float *P,
                                  double *loss, float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes,
                                  moe_stream_t stream);

/* Auxiliary-loss-free bias update, to run after a training step on the
 * counts that step's routing produced ("Fine-Tuning Mixture of Experts (MoE)
 * Models: Router Optimization Techniques", How It Works 2, and its router
 * module): with L_target = T * top_k / E,
 *   sel_bias[e] <- sel_bias[e] - gamma * sign(counts[e] - L_target)
 * computed in double and stored as fp32 (sign(0) = 0).  counts [E] int32,
 * sel_bias [E] fp32 in/out (the selection bias moe_router_topk takes).     */
MOE_API moe_status moe_bias_update(const moe_config *cfg, const int32_t *counts, float *sel_bias,
                                   float gamma, moe_stream_t stream);

/* Routing health: out[0] = -sum_e P_e log P_e, the Shannon entropy of the
 * mean routing distribution (Router Optimization page, Best Practices 6);
 * out[1] = max_e counts / min_e counts (+inf when an expert got nothing) and
 * out[2] = max_e counts / (T * top_k) ("Fine-tuning and serving MoE models",
 * Utilization is a first-class metric).  counts [E] int32, P [E] fp32 (from
 * moe_balance_stats), out [3] fp64, all device pointers.                    */
MOE_API moe_status moe_routing_health(const moe_config *cfg, const int32_t *counts, const float *P,
                                      double *out, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory.  The paper has
 * no counterpart: this entry point exists for integration only.
 * Same computation, arguments and outputs as moe_permute (x_perm may be NULL
 * for the row tables alone), but no workspace:
 * its scratch (per-chunk expert counts and their prefix sums) lives in a
 * static device array inside libmoe (2 MiB + 256 bytes on every GPU that
 * loads the library, held until the process exits).  It serves callers that
 * cannot call cudaMalloc (a plug-in in a host framework that owns the whole
 * device-memory budget, a latency-critical caller that cannot take
 * cudaMalloc's implicit device synchronisation).
 *   - Limit: E * ceil(T / 64) <= 262144 (E = 256 allows T <= 65536); beyond it
 *     the call returns MOE_ERR_UNSUPPORTED and launches nothing.
 *   - The first call on a device looks up the array's address with that
 *     device current and keeps it; make that first call before any stream
 *     capture.  The address is that of the device's current context: after
 *     cudaDeviceReset, reload the library before calling again.
 *   - All calls share the array: calls that overlap on the GPU race.
 *   - A bad expert id is dropped (row -1) as in moe_permute but, with no
 *     workspace status word, not reported.
 * Never calls cudaMalloc, cudaFree or any allocating routine.               */
MOE_API moe_status moe_permute_noalloc(const moe_config *cfg, const void *x, const int32_t *idx,
                                       const float *gate, int32_t *counts, int32_t *kept,
                                       int32_t *offsets, int32_t *row_of, int32_t *row_token,
                                       float *row_gate, void *x_perm, int32_t *n_dropped,
                                       moe_stream_t stream);

/* Synchronise `stream`, read the workspace status word into *status_out
 * (a moe_status) and clear it.  Returns MOE_ERR_CUDA if the read fails.   */
MOE_API moe_status moe_get_device_status(void *ws, moe_stream_t stream, int32_t *status_out);

/* Self-check of the bounded waits that every tensor-core kernel of the
 * library uses on its pipeline barriers (failure detection without a GPU
 * fault): one CTA initialises a shared-memory barrier that nothing ever
 * arrives on and waits on it with the library's bounded wait; after limit_ns
 * nanoseconds (1 us .. 10 s) the wait gives up, MOE_ERR_TIMEOUT is recorded in
 * the status word of `ws` (an initialised workspace of at least 256 bytes)
 * and the kernel returns normally, leaving the context usable.  Read the
 * outcome with moe_get_device_status.  The paper has no counterpart.        */
MOE_API moe_status moe_check_wait_timeout(void *ws, uint64_t limit_ns, moe_stream_t stream);

/* Static text for a status code. */
MOE_API const char *moe_status_string(moe_status s);

/* Text describing the last host-side failure on the calling thread (which
 * check failed, or the CUDA error string); "" if none.  Owned by the library. */
MOE_API const char *moe_last_error_detail(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
