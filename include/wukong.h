/*
 * wukong.h -- C ABI of the B200 (sm_100a) Wukong interaction-stack forward.
 *
 * The method is the Wukong layer of "Wukong: Towards a Scaling Law for
 * Large-Scale Recommendation" as summarised on the xdnf.cn repost of the Zhihu
 * article (section 2.2 "Wukong", section 2.3 "Scale"), and the Wukong module of
 * WHALE (gist.science summary of arXiv 2607.17017, section 2.1, item 1). Per
 * example, layer i maps the embedding matrix X_i (n x d) to
 *
 *     X_{i+1} = LN_rows( concat_rows( FMB(X_i), LCB(X_i) ) + X_i )
 *     FMB(X)  = reshape_{n_F x d}( MLP( LN( flatten( X (X^T Y) ) ) ) )
 *     LCB(X)  = W_L X
 *
 * with Y (n x k) the learnable projection that compresses the features to k
 * before the crossing (section 2.2, FMB paragraph), W_L (n_L x n) the linear
 * compression (section 2.2, LCB paragraph) and n_F + n_L = n so that the
 * residual needs no projection. The page's formulas were lost in extraction;
 * the equations above are the reading the surviving sentences support.
 *
 * Conventions shared by every entry point
 *   - Pointers named *_host are host memory; every other data pointer is device
 *     memory on the current CUDA device. All device pointers must be 16-byte
 *     aligned. Tensors are dense and row-major (last index fastest).
 *   - dtype WK_BF16 / WK_F16: X, out, Y, W_j, W_L are 16-bit; biases and
 *     LayerNorm parameters are fp32; all products accumulate in fp32 and
 *     LayerNorm statistics are fp32. The tensor-core operands and every
 *     intermediate buffer of a stack use the 16-bit `operand_dtype` (fp16 by
 *     default: its 10-bit mantissa keeps the 8-layer drift of the intermediate
 *     roundings ~6x below bf16's, at the same tensor-core rate); bf16 weights are
 *     converted to it once, at create. Intermediate values must stay within the
 *     fp16 range (|v| < 65504) when the operand type is fp16; they are
 *     LayerNorm outputs and Linear layers of them. dtype WK_F32: everything is
 *     fp32 on CUDA cores.
 *   - Calls that take a stream are asynchronous and stream-ordered: they only
 *     validate their arguments on the host and enqueue kernels. They never
 *     synchronise and never copy between host and device, except
 *     wk_stack_forward_host, which is synchronous by design, and
 *     wk_stack_forward_host_async / wk_stack_host_wait, whose copies are waited
 *     for by the second.
 *   - Every call returns a wk_status and never aborts the process. A kernel
 *     that detects a problem on the device (a pipeline wait that ran past its
 *     limit) records it in a device status word and returns early; read it with
 *     wk_stack_sync_status or wk_device_status.
 *   - The stream argument is a cudaStream_t (NULL = legacy default stream).
 */
#ifndef WUKONG_H
#define WUKONG_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define WK_API __attribute__((visibility("default")))
#else
#define WK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* wk_stream_t; /* same type as cudaStream_t */

typedef enum {
  WK_OK = 0,
  WK_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, batch out of range, overlapping X and out */
  WK_ERR_UNSUPPORTED = 2,  /* a shape or dtype this build does not implement (e.g. n_F + n_L != n) */
  WK_ERR_OOM = 3,          /* workspace allocation failed */
  WK_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch error, no device, ...) */
  WK_ERR_TIMEOUT = 5,      /* a kernel gave up on a pipeline wait; its output is not valid */
  WK_ERR_DEVICE = 6,       /* the device status word holds another error flag */
  WK_ERR_NONFINITE = 7     /* a LayerNorm met a non-finite row: a value left the range of its
                              16-bit storage (fp16: |v| > 65504) or an input held inf / NaN;
                              the output is not valid */
} wk_status;

typedef enum { WK_F32 = 0, WK_BF16 = 1, WK_F16 = 2 } wk_dtype;

/* Shape of the stack; every layer has the same shape (n is the same for every
 * layer because n_F + n_L = n). Scaling knobs of section 2.3: num_layers = l,
 * n_f = n_F, n_l = n_L, k, and the FMB MLP (mlp_num_linear Linear layers,
 * h_0 = n*k -> mlp_hidden[0] -> ... -> h_m = n_f*d, ReLU after every Linear but
 * the last). */
typedef struct {
  int32_t num_layers;          /* l >= 1 */
  int32_t n, d, k, n_f, n_l;   /* n_f + n_l == n; d % 8 == 0 (bf16) or d % 4 == 0 (fp32) */
  int32_t mlp_num_linear;      /* m >= 1 */
  const int32_t* mlp_hidden;   /* m-1 widths (may be NULL when m == 1); copied at create */
  wk_dtype dtype;              /* storage type of X, out, Y, W_j and W_L */
  float ln_eps;                /* LayerNorm epsilon; 0 selects 1e-5 */
  int64_t max_batch;           /* largest batch a forward will be given; sizes the workspace */
  wk_dtype operand_dtype;      /* 16-bit stacks: WK_F16 or WK_BF16 tensor-core operands and
                                  intermediates; WK_F32 (0) selects the default, WK_F16.
                                  Ignored when dtype is WK_F32. */
} wk_stack_config;

/* One layer's parameters. All DEVICE pointers, BORROWED: the caller keeps them
 * alive and unchanged until wk_stack_destroy. Layouts:
 *   Y            [n, k]               dtype
 *   W[j]         [h_{j+1}, h_j]       dtype  (row-major, the torch Linear layout)
 *   b[j]         [h_{j+1}]            fp32   (b or b[j] may be NULL: zero bias)
 *   fmb_ln_gamma, fmb_ln_beta [n*k]   fp32   (LayerNorm of the flattened FM output)
 *   W_L          [n_l, n]             dtype
 *   out_ln_gamma, out_ln_beta [d]     fp32   (LayerNorm of each output embedding row) */
typedef struct {
  const void* Y;
  const void* const* W;
  const float* const* b;
  const float* fmb_ln_gamma;
  const float* fmb_ln_beta;
  const void* W_L;
  const float* out_ln_gamma;
  const float* out_ln_beta;
} wk_layer_weights;

typedef struct wk_stack wk_stack;

/* Validates cfg, records the weight pointers of cfg->num_layers layers
 * (weights[0 .. num_layers-1]), converts the weights to the operand type when it
 * differs from dtype (a device copy the handle owns; the originals are then no
 * longer read), folds the FMB LayerNorm's gamma / beta into the first MLP Linear
 * of 16-bit stacks (a handle-owned copy W0 diag(gamma) and bias b0 + W0 beta: the
 * same function, without per-example reads of gamma and beta), builds the TMA
 * descriptors of the weights and allocates the
 * workspace for cfg->max_batch examples on the current device, in the operand
 * type: A0 [max_batch, n*k], two MLP activation buffers [max_batch, max hidden],
 * the concat buffer [max_batch, n, d] and two layer buffers [max_batch, n, d].
 * Synchronises the device. The handle owns the workspace; *out is set only on WK_OK.
 * Errors: WK_ERR_INVALID_ARG (NULL, misaligned, max_batch < 1),
 * WK_ERR_UNSUPPORTED (n_f + n_l != n, unsupported d / dtype / widths),
 * WK_ERR_OOM, WK_ERR_CUDA. */
WK_API wk_status wk_stack_create(const wk_stack_config* cfg, const wk_layer_weights* weights, wk_stack** out);

/* out[b] = stack(X[b]) for b < batch. X and out are [batch, n, d] device
 * tensors of cfg->dtype; they must not overlap. batch == 0 is a no-op (WK_OK).
 * Asynchronous on `stream`. One handle is not re-entrant: two forwards on one
 * handle must be ordered (same stream, or synchronised), because they share the
 * workspace. Errors: WK_ERR_INVALID_ARG (NULL handle or pointer, misaligned,
 * batch < 0 or > max_batch, X/out overlap), WK_ERR_CUDA (launch failure). */
WK_API wk_status wk_stack_forward(wk_stack* h, const void* X, void* out, int64_t batch, wk_stream_t stream);

/* Same result as wk_stack_forward with HOST input and output buffers
 * ([batch, n, d], cfg->dtype). Splits the batch into chunks and overlaps the
 * host-to-device copy of chunk c+1 and the device-to-host copy of chunk c-1
 * with the forward of chunk c on internal streams ordered after `stream`.
 * Returns when out_host holds the result. Page-locked (pinned) host buffers give
 * the full copy bandwidth; pageable ones work but copy slower. Chunks use the
 * handle's workspace and two staging buffers allocated on first use. */
WK_API wk_status wk_stack_forward_host(wk_stack* h, const void* X_host, void* out_host, int64_t batch, wk_stream_t stream);

/* The host-buffer forward for a stream of batches, as a serving loop issues them. The
 * Wukong paper has no counterpart: it specifies the layer, not how batches reach the GPU.
 * Enqueues the copy of X_host into one of two device input slots, one wk_stack_forward
 * of the whole batch on `stream`, and the copy of its result into out_host, then returns
 * without waiting. Successive calls alternate the slots, so the input copy of call i+1
 * and the output copy of call i-1 run on internal copy streams while the forward of
 * call i computes; each forward keeps the full batch (no chunking of the GEMMs).
 * *ticket (may be NULL) receives the call's sequence number for wk_stack_host_wait.
 * Ownership: the caller keeps X_host unchanged and does not touch out_host until
 * wk_stack_host_wait has returned for this ticket or a later one; both must be
 * page-locked for the copies to overlap (pageable buffers give the same result with
 * copies that block the host). Successive calls on one handle use one stream (they
 * share the workspace). The slots, 4 * max_batch * n * d elements of cfg->dtype, are
 * allocated on the first call. batch == 0 is a no-op (*ticket = the last ticket, -1 if
 * none). Errors: as wk_stack_forward, WK_ERR_OOM, WK_ERR_CUDA; on an error nothing of
 * the call is left to wait for. */
WK_API wk_status wk_stack_forward_host_async(wk_stack* h, const void* X_host, void* out_host, int64_t batch,
                                             wk_stream_t stream, int64_t* ticket);

/* Blocks the host until the output copy of wk_stack_forward_host_async call `ticket` has
 * landed in its out_host, and with it the copies of every earlier call (ticket < 0: of
 * every call made so far). A ticket more than two calls old may also wait for a later
 * call's copy. WK_OK, WK_ERR_INVALID_ARG (NULL handle, a ticket not issued yet),
 * WK_ERR_CUDA (a copy or a kernel it waited for failed). Device-side errors of the
 * forwards are read with wk_stack_sync_status. */
WK_API wk_status wk_stack_host_wait(wk_stack* h, int64_t ticket);

/* Waits for `stream`, then reads and clears the device status word.
 * WK_OK, WK_ERR_TIMEOUT, WK_ERR_NONFINITE, WK_ERR_DEVICE or WK_ERR_CUDA.
 * WK_ERR_NONFINITE: a 16-bit stack stores its intermediates in fp16 by default (see
 * wk_stack_config.operand_dtype); every LayerNorm of the forward (the FMB LayerNorm, each
 * layer's output LayerNorm) checks its row statistics, so a value that overflowed fp16
 * anywhere upstream is reported here instead of leaving inf / NaN silently in `out`. */
WK_API wk_status wk_stack_sync_status(wk_stack* h, wk_stream_t stream);

/* Frees the workspace and the handle (synchronises the device first). NULL is a no-op. */
WK_API void wk_stack_destroy(wk_stack* h);

/* Static string for a status code. */
WK_API const char* wk_status_string(wk_status s);

/* ---- CUDA graphs of a forward (for launch-bound batches) ----
 *
 * Captures one forward on FIXED device buffers X and out into a CUDA graph that
 * wk_graph_launch replays with one launch: every kernel of the stack (or MoE stack)
 * in order, with none of the host work of a forward call (argument checks, TMA
 * descriptor encoding, launch overhead per kernel). The caller refills X between
 * launches; the graph reads X and writes out at replay time. The handle must outlive
 * the graph and must not be used by another forward while a replay runs (same
 * workspace). Capture happens on a private stream; profiling records are not taken
 * inside graphs. Errors: WK_ERR_INVALID_ARG (as for the forward), WK_ERR_CUDA. */
typedef struct wk_graph wk_graph;
WK_API wk_status wk_stack_graph_create(wk_stack* h, const void* X, void* out, int64_t batch, wk_graph** g);
WK_API wk_status wk_graph_launch(wk_graph* g, wk_stream_t stream);
WK_API void wk_graph_destroy(wk_graph* g);

/* ---- per-kernel timing of a handle's forwards (CUDA events on the launch stream) ---- */

typedef enum { WK_KERNEL_FM_LN = 0, WK_KERNEL_MLP_GEMM = 1, WK_KERNEL_LCB = 2, WK_KERNEL_RES_LN = 3,
               WK_KERNEL_CONVERT = 4, WK_KERNEL_MOE_GATE = 5, WK_KERNEL_MOE_COMBINE = 6,
               WK_KERNEL_HEAD = 7, WK_KERNEL_WHALE_ATTN = 8, WK_KERNEL_WHALE_FFN = 9,
               WK_KERNEL_BW_CONTRACT = 10, WK_KERNEL_BW_ROWS = 11, WK_KERNEL_FRONT = 12,
               WK_KERNEL_COUNT = 13 } wk_kernel_kind;

/* enable != 0: every later forward records a start/stop event pair around each
 * kernel launch on its stream (adds no synchronisation). */
WK_API wk_status wk_stack_set_profiling(wk_stack* h, int enable);

/* Waits for the recorded events, then reports, per kernel kind, the summed
 * device time in ms and the number of launches since the last call, and clears
 * the record. total_ms and launches are arrays of WK_KERNEL_COUNT entries. */
WK_API wk_status wk_stack_kernel_times(wk_stack* h, double* total_ms, int64_t* launches);

/* ---- the steps of one layer as stand-alone calls (no handle, no workspace) ---- */

/* FMB front: A0[b] = LN( flatten( X_b (X_b^T Y) ) ) * gamma + beta, b < batch.
 * X [batch, n, d], Y [n, k] (dtype), gamma/beta [n*k] fp32, A0 [batch, n*k] dtype.
 * gamma and beta may both be NULL: A0 then holds the normalised values (a stack
 * passes NULL, having folded gamma and beta into its first MLP Linear).
 * The FM runs per example on the tensor cores (bf16) with fp32 accumulation;
 * X_b^T Y is rounded to bf16 before the second product (bf16 path only). */
WK_API wk_status wk_fm_ln(const void* X, const void* Y, const float* gamma, const float* beta, void* A0, int64_t batch,
                   int32_t n, int32_t d, int32_t k, wk_dtype dtype, float eps, wk_stream_t stream);

/* One Linear of the FMB MLP over the batch: C[r, c] = act( sum_q A[r, q] W[c, q] + bias[c] ),
 * r < M, c < N; act = ReLU if relu != 0. A [M, K] (row stride K), W [N, K],
 * bias [N] fp32 or NULL, C [M, N] with row stride ldc elements (ldc >= N; the
 * last Linear writes straight into the concat buffer with ldc = n*d).
 * K % 8 == 0, N % 8 == 0, ldc % 8 == 0 (bf16). */
WK_API wk_status wk_mlp_linear(const void* A, const void* W, const float* bias, void* C, int64_t M, int32_t K, int32_t N,
                        int64_t ldc, int relu, wk_dtype dtype, wk_stream_t stream);

/* LCB: concat[b, n_f + r, :] = sum_i W_L[r, i] X[b, i, :] for r < n_l, b < batch.
 * W_L [n_l, n], X [batch, n, d], concat [batch, n_f + n_l, d] (dtype); rows
 * 0..n_f-1 of concat are not touched. */
WK_API wk_status wk_lcb(const void* W_L, const void* X, void* concat, int64_t batch, int32_t n, int32_t d, int32_t n_f,
                 int32_t n_l, wk_dtype dtype, wk_stream_t stream);

/* Concat + residual + LayerNorm: out[r, :] = LN( concat[r, :] + X[r, :] ) * gamma + beta
 * over each of `rows` embedding rows of d values. concat, X, out [rows, d] (dtype),
 * gamma/beta [d] fp32. out may alias concat. */
WK_API wk_status wk_res_ln(const void* concat, const void* X, const float* gamma, const float* beta, void* out, int64_t rows,
                    int32_t d, wk_dtype dtype, float eps, wk_stream_t stream);

/* Waits for `stream`, then reads and clears the device status word of the
 * stand-alone calls above (handles have their own). */
WK_API wk_status wk_device_status(wk_stream_t stream);

/* ---- prediction head ----
 *
 * Wukong page, section 2.2, first paragraph: the model crosses features with the
 * stacked Wukong layers and then produces the prediction with an MLP. The page gives
 * the head no sizes; the reading implemented: the last layer's output X_L is
 * flattened row-major (n*d values per example), q Linear layers follow with ReLU
 * after all but the last, the last has one output (the logit), and the prediction
 * is its logistic sigmoid:
 *
 *     z_0 = vec(X_L),  z_{j+1} = ReLU(T_j z_j + c_j) (j < q-1),
 *     logit = T_{q-1} z_{q-1} + c_{q-1},  prob = 1 / (1 + exp(-logit)). */
typedef struct {
  int32_t num_linear;       /* q >= 1 */
  const int32_t* hidden;    /* q-1 hidden widths, multiples of 8 (copied); NULL when q == 1 */
  const void* const* T;     /* q weights [out_j, in_j] in the stack's dtype, row-major; in_0 = n*d,
                               out_{q-1} = 1. Device pointers, BORROWED like the layer weights
                               (copied at this call when dtype differs from the operand type) */
  const float* const* c;    /* q biases [out_j] fp32; c or c[j] may be NULL (zero) */
} wk_head;

/* Attaches (or replaces) the prediction head of a 16-bit stack: converts its weights
 * to the operand type when needed, allocates two activation buffers [max_batch,
 * widest hidden] and builds the head's GEMM descriptors. Synchronises the device.
 * Errors: WK_ERR_INVALID_ARG (NULL, misaligned), WK_ERR_UNSUPPORTED (fp32 stack,
 * widths not multiples of 8), WK_ERR_OOM, WK_ERR_CUDA. */
WK_API wk_status wk_stack_set_head(wk_stack* h, const wk_head* head);

/* The stack forward on X [batch, n, d] followed by the head: logit [batch] fp32 and,
 * when prob is not NULL, prob [batch] fp32. The last layer's output stays on the
 * device in the operand type; the head's hidden Linears run on the tensor-core GEMM,
 * its one-output Linear and the sigmoid in head_out_kernel. Asynchronous on
 * `stream`; not re-entrant. WK_ERR_INVALID_ARG without a head. */
WK_API wk_status wk_stack_predict(wk_stack* h, const void* X, float* logit, float* prob, int64_t batch,
                                  wk_stream_t stream);

/* ---- Wukong mixture of experts ----
 *
 * The Kunlun page (gist.science summary of arXiv 2602.10016, section 2.3, "Wukong
 * Mixture of Experts") describes a global interaction module in which several
 * Wukong modules run in parallel as the experts of one layer, spreading the layer's
 * computation over them. The page gives no formula; the reading implemented is the
 * dense mixture of experts: expert e of MoE layer l is a whole Wukong layer (its own
 * FMB, LCB, residual and output LayerNorm), and a softmax gate computed per example
 * from the flattened layer input weights the experts' outputs:
 *
 *     g(X)    = softmax( W_g vec(X) + b_g ),    W_g [E, n*d], vec row-major
 *     MoE(X)  = sum_e g_e(X) * WukongLayer_e(X)
 *
 * Every expert runs on every example (the page names no routing). A stack of
 * num_layers MoE layers maps X_0 to X_L. 16-bit dtypes only. */

typedef struct {
  const void* W_g;   /* [num_experts, n*d] dtype, row e scores expert e; BORROWED like the
                        layer weights (copied at create when dtype differs from the operand type) */
  const float* b_g;  /* [num_experts] fp32, or NULL for zero */
} wk_moe_gate;

typedef struct wk_moe wk_moe;

#define WK_MOE_MAX_EXPERTS 8

/* cfg: the shape of every expert layer and of the MoE stack (cfg->num_layers MoE
 * layers; dtype WK_BF16 or WK_F16; operand_dtype, ln_eps and max_batch as for
 * wk_stack_create). experts: num_layers * num_experts layer weights, layer-major
 * (experts[l * num_experts + e] is expert e of layer l), device pointers BORROWED
 * as for wk_stack_create. gates: num_layers gate parameters. 1 <= num_experts <=
 * WK_MOE_MAX_EXPERTS. Allocates, per expert, the workspace of one layer's front
 * (A0, MLP activations, concat buffer), plus the gate weights [max_batch,
 * num_experts] fp32 and two layer buffers [max_batch, n, d] in the operand type.
 * Synchronises the device. Errors as wk_stack_create; WK_ERR_UNSUPPORTED for fp32. */
WK_API wk_status wk_moe_create(const wk_stack_config* cfg, int32_t num_experts, const wk_layer_weights* experts,
                               const wk_moe_gate* gates, wk_moe** out);

/* out[b] = MoE stack(X[b]) for b < batch; X and out [batch, n, d] of cfg->dtype, not
 * overlapping. Per MoE layer on `stream`: the gate (moe_gate_kernel), each expert's
 * FM + LayerNorm, MLP and LCB into its own concat buffer, then one kernel that
 * applies every expert's residual + LayerNorm and mixes them with the gate
 * (moe_combine_kernel). Asynchronous; not re-entrant (as wk_stack_forward). */
WK_API wk_status wk_moe_forward(wk_moe* h, const void* X, void* out, int64_t batch, wk_stream_t stream);

/* Waits for `stream`, then reads and clears the experts' device status words. */
WK_API wk_status wk_moe_sync_status(wk_moe* h, wk_stream_t stream);

/* Per-kernel event timing of a handle's forwards, as wk_stack_set_profiling /
 * wk_stack_kernel_times (the experts' kernels summed per kind, plus
 * WK_KERNEL_MOE_GATE and WK_KERNEL_MOE_COMBINE). */
WK_API wk_status wk_moe_set_profiling(wk_moe* h, int enable);
WK_API wk_status wk_moe_kernel_times(wk_moe* h, double* total_ms, int64_t* launches);

/* Frees the handle, its experts and workspace (synchronises the device). NULL is a no-op. */
WK_API void wk_moe_destroy(wk_moe* h);

/* A CUDA graph of one MoE forward on fixed X and out (as wk_stack_graph_create);
 * replay with wk_graph_launch, free with wk_graph_destroy. */
WK_API wk_status wk_moe_graph_create(wk_moe* h, const void* X, void* out, int64_t batch, wk_graph** g);

/* Stand-alone gate: g[b, e] = softmax_e( sum_j W_g[e, j] X[b, j] + b_g[e] ), X [batch, nd]
 * and W_g [num_experts, nd] of dtype (16-bit, nd % 8 == 0), b_g [num_experts] fp32 or
 * NULL, g [batch, num_experts] fp32. Dot products accumulate in fp32. */
WK_API wk_status wk_moe_gate_softmax(const void* X, const void* W_g, const float* b_g, float* g, int64_t batch,
                                     int64_t nd, int32_t num_experts, wk_dtype dtype, wk_stream_t stream);

/* Stand-alone mixture of the experts' residual + LayerNorm outputs:
 *   out[b, i, :] = sum_e g[b, e] * ( LN( concat_e[b, i, :] + X[b, i, :] ) * gamma_e + beta_e )
 * concats: num_experts pointers to [batch, n, d]; X, out [batch, n, d] (dtype, 16-bit);
 * g [batch, num_experts] fp32; gammas, betas: num_experts pointers to [d] fp32. */
WK_API wk_status wk_moe_combine(const void* const* concats, const void* X, const float* g, const float* const* gammas,
                                const float* const* betas, void* out, int64_t batch, int32_t n, int32_t d,
                                int32_t num_experts, wk_dtype dtype, float eps, wk_stream_t stream);

/* ---- backward pass of the stack (training) ----
 *
 * The pages train Wukong (Wukong page, section 3.2.1: Adam for the dense parameters)
 * but give no backward; this is the forward of wk_stack_forward differentiated by the
 * chain rule. Given the stack's input X and dOut = dL/d(output), it computes dX =
 * dL/dX and, per layer, the gradients of every parameter of wk_layer_weights (the
 * caller's W0, b0, gamma1, beta1 as given at create, though the forward runs a folded
 * first Linear), summed over the batch. */
typedef struct {           /* fp32 DEVICE buffers the backward overwrites, one set per layer */
  float* Y;                /* [n, k] */
  float* const* W;         /* m entries, [h_{j+1}, h_j] (16-byte aligned) */
  float* const* b;         /* m entries, [h_{j+1}] */
  float* fmb_ln_gamma, *fmb_ln_beta;   /* [n*k] */
  float* W_L;              /* [n_l, n] */
  float* out_ln_gamma, *out_ln_beta;   /* [d] */
} wk_layer_grads;

/* X [batch, n, d] in the stack's dtype (the input of the forward whose gradient is
 * wanted); dOut and dX [batch, n, d] fp32; grads: num_layers gradient sets. The forward
 * is run once with every layer's input and activations saved (the FMB LayerNorm output,
 * the hidden ReLU outputs, the concat buffer), then each layer is differentiated, last
 * layer first: the output LayerNorm and the residual per row; the FMB MLP's input,
 * weight and bias gradients on the tensor-core GEMM (16-bit operands read MN-major where
 * the contraction needs their transposes, fp32 weight gradients); the FMB LayerNorm per
 * example; the FM's and the LCB's products on the tf32 tensor cores (fp32 accumulation).
 * Supported: 16-bit stacks with fp16 operands (the default), at most 3 MLP Linears,
 * batch % 8 == 0, d % 32 == 0 and d <= 256; otherwise WK_ERR_UNSUPPORTED. The first call
 * (or a larger batch) allocates the backward workspace (all layer inputs and
 * activations, fp32 gradients of the layer stream, the MLP gradients, fp32 copies of X,
 * W_L and Y; transposed copies only when batch or a hidden width is at most 128).
 * Asynchronous on `stream` apart from that allocation; not re-entrant (shares the
 * forward's workspace). */
WK_API wk_status wk_stack_backward(wk_stack* h, const void* X, const float* dOut, float* dX,
                                   const wk_layer_grads* grads, int64_t batch, wk_stream_t stream);

/* The same, recording layer_done[l] (a cudaEvent_t created by the caller, or NULL to skip
 * it; the array itself may be NULL) on `stream` as soon as layer l's parameter gradients
 * are written. Layers finish last first, so a data-parallel caller can start reducing
 * layer l's gradients across ranks (on another stream, after that event) while the
 * layers below it are still being differentiated. Errors as wk_stack_backward. */
WK_API wk_status wk_stack_backward_events(wk_stack* h, const void* X, const float* dOut, float* dX,
                                          const wk_layer_grads* grads, int64_t batch, wk_stream_t stream,
                                          void* const* layer_done);

/* ---- WHALE attention-based fusion ----
 *
 * The WHALE pages (gist.science summaries of arXiv 2607.17017, Korean and French),
 * section 2.1 item 3: the Wukong interaction representation H_w is the query and the
 * HSTU behaviour representation H_s both key and value of an attention; its output is
 * concatenated with H_w, projected by a fusion MLP and passed through a pre-norm
 * SwiGLU FFN, giving the fused representation H_f. Section 2.2: K = V (one tensor
 * for both) and the gate and up projections of the SwiGLU share one matrix
 * (W_gate = W_up). The pages give no formulas; the reading implemented (one head, no
 * Q/K/V projections, a one-Linear fusion MLP, no FFN biases), per example:
 *
 *     A   = softmax_rows( H_w H_s^T / sqrt(d) ) H_s          H_w [n, d], H_s [L, d]
 *     Z   = [H_w | A] W_F^T + b_F                            W_F [d, 2d]
 *     U   = LN(Z) W_up^T                                     W_up [h, d], LN over d
 *     H_f = Z + ( SiLU(U) * U ) W_down^T                     W_down [d, h]
 *
 * 16-bit storage (bf16 or fp16) for H_w, H_s, H_f, A and the weight matrices; fp32
 * accumulation, softmax and LayerNorm statistics; the softmax weights and the gated
 * activations are rounded to the 16-bit type as tensor-core operands. */

typedef struct {
  int32_t n;          /* query rows per example (rows of H_w and H_f), >= 1 */
  int32_t d;          /* embedding width: 32, 64, 128 or 160 */
  int32_t L;          /* key / value rows per example (rows of H_s), >= 1 */
  int32_t h;          /* FFN width, a positive multiple of 64 */
  wk_dtype dtype;     /* WK_BF16 or WK_F16 */
  float ln_eps;       /* LayerNorm epsilon; 0 selects 1e-5 */
  int64_t max_batch;  /* examples per forward, sizes the workspace */
} wk_whale_config;

typedef struct {      /* DEVICE pointers, BORROWED: the caller keeps them alive until destroy */
  const void* W_F;    /* [d, 2d] dtype, row-major (PyTorch Linear layout) */
  const float* b_F;   /* [d] fp32, or NULL for zero */
  const float* ln_gamma, *ln_beta;  /* [d] fp32 */
  const void* W_up;   /* [h, d] dtype */
  const void* W_down; /* [d, h] dtype */
} wk_whale_weights;

typedef struct wk_whale wk_whale;

/* Validates the shape (WK_ERR_UNSUPPORTED for a d, h or dtype the kernels do not
 * handle; WK_ERR_INVALID_ARG for NULL or misaligned pointers, n, L or max_batch < 1),
 * allocates the attention output A [max_batch, n, d] and a status word. Synchronises
 * the device. */
WK_API wk_status wk_whale_create(const wk_whale_config* cfg, const wk_whale_weights* w, wk_whale** out);

/* Hf[b] = fusion(Hw[b], Hs[b]) for b < batch: Hw, Hf [batch, n, d], Hs [batch, L, d],
 * all dtype, 16-byte aligned; Hf must not overlap Hw or Hs. Two kernels on `stream`:
 * whale_attn_kernel (A) and whale_ffn_kernel (Z, LayerNorm, SwiGLU, residual).
 * batch == 0 is a no-op; batch > max_batch is WK_ERR_INVALID_ARG. Asynchronous; not
 * re-entrant (the handle's A buffer is shared). */
WK_API wk_status wk_whale_forward(wk_whale* h, const void* Hw, const void* Hs, void* Hf, int64_t batch,
                                  wk_stream_t stream);

/* Waits for `stream`, then reads and clears the handle's device status word. */
WK_API wk_status wk_whale_sync_status(wk_whale* h, wk_stream_t stream);

/* Per-kernel event timing of the handle's forwards (kinds WK_KERNEL_WHALE_ATTN and
 * WK_KERNEL_WHALE_FFN), as wk_stack_set_profiling / wk_stack_kernel_times. */
WK_API wk_status wk_whale_set_profiling(wk_whale* h, int enable);
WK_API wk_status wk_whale_kernel_times(wk_whale* h, double* total_ms, int64_t* launches);

/* Frees the handle and its workspace (synchronises the device). NULL is a no-op. */
WK_API void wk_whale_destroy(wk_whale* h);

/* Stand-alone attention with shared keys and values:
 *   A[b] = softmax_rows( Hw[b] Hs[b]^T / sqrt(d) ) Hs[b]
 * Hw, A [batch, n, d], Hs [batch, L, d] (dtype, 16-bit); d in {32, 64, 128, 160}. */
WK_API wk_status wk_whale_attention(const void* Hw, const void* Hs, void* A, int64_t batch, int32_t n, int32_t L,
                                    int32_t d, wk_dtype dtype, wk_stream_t stream);

/* Stand-alone fusion Linear + pre-norm shared-gate SwiGLU FFN over `rows` rows:
 *   Z = [Hw | A] W_F^T + b_F,  Hf = Z + ( SiLU(U) * U ) W_down^T,  U = LN(Z) W_up^T
 * Hw, A, Hf [rows, d] (dtype); weights as wk_whale_weights; eps 0 selects 1e-5. */
WK_API wk_status wk_whale_fusion_ffn(const void* Hw, const void* A, const wk_whale_weights* w, void* Hf,
                                     int64_t rows, int32_t d, int32_t h, wk_dtype dtype, float eps,
                                     wk_stream_t stream);

/* ---- one layer without allocating: for callers that cannot call cudaMalloc ----
 *
 * The paper has no counterpart to this entry point; it exists for callers that
 * must not have the library allocate device memory: a serving process that has
 * handed all device memory to its own pool allocator, or a latency-critical loop
 * where cudaMalloc / cudaFree (which synchronise the device) are not allowed.
 * wk_stack_create allocates a workspace, so such callers use this instead.
 *
 * Runs ONE Wukong layer, out = LN_rows(concat(FMB(X), LCB(X)) + X), with the
 * weights `w` used as given (operands in cfg->dtype; cfg->operand_dtype must be 0
 * or equal to cfg->dtype, since converting weights would need memory). X and out
 * are caller-owned device tensors [batch, n, d] of cfg->dtype that must not
 * overlap; cfg->num_layers and cfg->max_batch are ignored. Every pointer (X, out,
 * and each weight, bias and LayerNorm vector in `w`) must be 16-byte aligned, as
 * for wk_stack_create; a misaligned one returns WK_ERR_INVALID_ARG before
 * anything is launched. The FMB LayerNorm affine is applied in the FM's
 * epilogue here (nothing is folded into a weight copy).
 *
 * Intermediates live in one fixed device array of WK_NOALLOC_SCRATCH_BYTES that
 * is part of the library image: every GPU that loads the library reserves it
 * until the process exits. A batch needs, in bytes (each term rounded up to 256):
 *   es * batch * (n*k + n*d + [m >= 2] * h + [m >= 3] * h),
 * es = 2 (16-bit) or 4 (fp32), h = the widest hidden layer; a batch that needs
 * more returns WK_ERR_INVALID_ARG before anything is launched. Nothing in the
 * array has to start at zero: every call writes each region before reading it.
 *
 * No call allocates: no cudaMalloc, cudaFree or allocating library routine. The
 * first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * which may load the library's device code on that device); make that first call
 * before any stream capture. Every call shares the one array, so calls whose
 * kernels can overlap on the GPU (different streams without ordering, or several
 * host threads) race and corrupt each other's results; order them on one stream.
 * Asynchronous on `stream`; device-side errors go to the status word that
 * wk_device_status reads. */
#define WK_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
WK_API wk_status wk_layer_forward_noalloc(const wk_stack_config* cfg, const wk_layer_weights* w, const void* X,
                                          void* out, int64_t batch, wk_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WUKONG_H */
