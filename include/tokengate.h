/*
 * tokengate.h -- C ABI of libtokengate, a B200 (sm_100a) implementation of
 * the data-parallel hot path of TokenGate's gated prefill.
 *
 * Sources (web pages about the TokenGate paper), cited below by tag:
 *   [TC] Tencent Cloud developer article "TokenGate：端到端可训练的 Token 剪枝机制，
 *        让大模型 Prefill 提速 11.3 倍"
 *   [FW] farwalk.ai item "Researchers from Stanford and Berkeley propose
 *        TokenGate, using learnable pruning to speed up long-context Prefill
 *        by up to about 11x", section "论文的方法"
 *   [AI] ai.866data.com article "让大模型学会"略读"：TokenGate如何破解长上下文推理
 *        的效率困局", section "可学习剪枝的机制设计"
 *
 * Conventions shared by every call
 * --------------------------------
 *  - The caller owns all memory. Tensor arguments are DEVICE pointers unless
 *    a comment says otherwise; the library allocates nothing. Scratch space
 *    is passed as (ws, ws_bytes); tg_workspace_size() gives the size.
 *  - Layouts are row-major and token-major. Weight matrices are stored
 *    [out_features, in_features] (the nn.Linear layout).
 *  - Activations and weight matrices use the call's tg_dtype (bf16 or fp32).
 *    One-dimensional parameters (norm weights, scorer bias/w2, gain, tau) and
 *    scores are always fp32. Indices and positions are int32.
 *  - Calls are asynchronous on the given stream and never synchronise with
 *    the host. Arguments are validated on the host before any launch; a bad
 *    argument returns an error and launches nothing.
 *  - Results are deterministic: the same inputs give the same bits.
 *  - Device code never traps. Every wait inside a kernel is bounded; a wait
 *    that runs out sets a sticky device error word, read by
 *    tg_device_error().
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* tg_stream;

typedef enum {
  TG_OK = 0,
  TG_ERR_INVALID_ARG = 1, /* null pointer, bad size or unaligned pointer */
  TG_ERR_UNSUPPORTED = 2, /* dtype / head_dim / width not built for     */
  TG_ERR_BUDGET = 3,      /* k < 1 or k > n                              */
  TG_ERR_WORKSPACE = 4,   /* ws_bytes smaller than tg_workspace_size()   */
  TG_ERR_CUDA = 5         /* a CUDA call failed; see tg_last_cuda_error  */
} tg_status;

typedef enum { TG_F32 = 0, TG_BF16 = 1 } tg_dtype;

typedef enum {
  TG_OP_SCORE = 0,
  TG_OP_TOPK_SELECT = 1,
  TG_OP_COMPACT = 2,
  TG_OP_GATED_ATTN = 3,
  TG_OP_PREFILL = 4,
  TG_OP_DECODE = 5,  /* shape: d_model, heads, head_dim, d_ffn, k = kept prompt tokens, dtype */
  TG_OP_GATED_ATTN_BWD = 6  /* shape: k = rows, heads, head_dim */
} tg_op;

/* Sizes used to size a workspace; fields an op does not use are ignored. */
typedef struct {
  int64_t n;        /* tokens entering the gate                        */
  int64_t k;        /* tokens kept (rows of the gated attention)        */
  int32_t d_model;
  int32_t n_heads_q;
  int32_t n_heads_kv;
  int32_t head_dim;
  int32_t d_score;  /* scorer hidden width F                           */
  int32_t d_ffn;    /* SwiGLU intermediate width I (0: no FFN)          */
  int32_t n_layers;
  int32_t gate_layer;
  tg_dtype dtype;
} tg_shape;

/* Bytes of scratch the op needs for these sizes (0 if none). */
size_t tg_workspace_size(tg_op op, const tg_shape* shape);

/*
 * tg_score -- importance score of every token.
 *   s_t = w2 . SiLU(W1 . RMSNorm(x_t; norm_w, eps) + b1) + b2
 * A small MLP reads each token's post-attention residual at the gate layer
 * and emits one scalar ([TC] "TokenGate 提前筛选 Token"; [AI]). The pages do
 * not fix the MLP's inner form; this library uses RMSNorm -> Linear(d->f) ->
 * SiLU -> Linear(f->1).
 *   x       [n, d] dtype       norm_w [d] fp32     w1 [f, d] dtype
 *   b1      [f] fp32 or NULL   w2 [f] fp32         b2 [1] fp32 or NULL
 *   scores  [n] fp32 (out)
 * bf16 needs f % 16 == 0, f <= 256, d % 8 == 0; fp32 any f <= 1024.
 */
tg_status tg_score(const void* x, int64_t n, int32_t d, int32_t f, const float* norm_w, float eps,
                   const void* w1, const float* b1, const float* w2, const float* b2, tg_dtype dtype,
                   float* scores, void* ws, size_t ws_bytes, tg_stream stream);

/*
 * tg_topk_select -- the kept set.
 * Keeps exactly k tokens: every protected token (protect[i] != 0) plus the
 * k - P best unprotected tokens ranked by (score descending, index
 * ascending); -0.0 ranks equal to +0.0 and NaN below -inf. kept_idx is
 * written ascending. The top-K selector and the un-prunable question span
 * are from [TC] "TokenGate 提前筛选 Token" and [AI]; the tie order is this
 * library's choice (deterministic).
 *   scores  [n] fp32           protect [n] uint8 or NULL (none protected)
 *   kept_idx [k] int32 (out)
 * If more than k tokens are protected (known only on the device), kept_idx
 * is filled with -1 and the workspace's first int32 is set to TG_ERR_BUDGET
 * (it is TG_OK otherwise).
 */
tg_status tg_topk_select(const float* scores, const uint8_t* protect, int64_t n, int64_t k,
                         int32_t* kept_idx, void* ws, size_t ws_bytes, tg_stream stream);

/*
 * tg_topk_select_noalloc -- tg_topk_select without a workspace argument.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot hand the library scratch device memory: code that only receives
 * input and output buffers from a host application which keeps the GPU's
 * memory in its own pool, or a latency-critical loop that must not call
 * cudaMalloc/cudaFree because those calls can synchronise the device.
 * The selection is the same as tg_topk_select (same kernels, same result).
 * Its scratch (about 24 KB) is a static array in device memory that every
 * GPU loading the library holds until the process exits.
 *  - n must not exceed TG_SELECT_NOALLOC_MAX_N; larger n returns
 *    TG_ERR_UNSUPPORTED before any launch (use tg_topk_select instead).
 *  - The first call in a CUDA context looks up the array's device address
 *    (one runtime call, with the caller's device current) and caches it
 *    under the context's unique id; make that first call before any stream
 *    capture. After cudaDeviceReset, or in another context made current
 *    through the driver API, the next call looks the address up again.
 *  - Every call on a device shares the one array, and each call clears what
 *    it needs. Calls whose kernels overlap on the GPU (e.g. on two streams)
 *    race on it: keep them ordered on one stream.
 *  - If more than k tokens are protected, kept_idx is filled with -1.
 * The call itself allocates nothing.
 */
#define TG_SELECT_NOALLOC_MAX_N 1048576
tg_status tg_topk_select_noalloc(const float* scores, const uint8_t* protect, int64_t n,
                                 int64_t k, int32_t* kept_idx, tg_stream stream);

/*
 * tg_compact -- gather of the kept rows.
 *   x_out[r] = x[kept_idx[r]], pos_out[r] = pos_in[kept_idx[r]] (or
 *   kept_idx[r] when pos_in is NULL), scores_out[r] = scores[kept_idx[r]].
 * Only the kept tokens continue into the layers above the gate, carrying
 * their original positions ([TC] "TokenGate 提前筛选 Token"; [FW]).
 *   x [n, d] dtype, pos_in [n] int32 or NULL, scores [n] fp32 or NULL,
 *   kept_idx [k] int32 with every entry in [0, n) (checked on the device:
 *   an entry out of range writes a zero row and sets the device error word).
 *   x_out [k, d], pos_out [k], scores_out [k] or NULL.
 * x and x_out rows must be 16-byte aligned (d * elem % 16 == 0).
 */
tg_status tg_compact(const void* x, const int32_t* pos_in, const float* scores,
                     const int32_t* kept_idx, int64_t n, int64_t k, int32_t d, tg_dtype dtype,
                     void* x_out, int32_t* pos_out, float* scores_out, tg_stream stream);

/*
 * tg_gated_attn_prefill -- token-gated causal GQA attention over the kept rows.
 *   l_ij = (q_i . k_j) / (sqrt(dh) * tau_h) + gain_h * logsigmoid(s_j),
 *   for pos_j <= pos_i; o_i = sum_j softmax_j(l_ij) v_j.
 * The kept tokens' scores enter the attention logits of the layers above the
 * gate as a bias, with a learnable per-head gain and temperature ([TC]
 * "门控机制为评分网络建立梯度路径"; [AI]). The pages state the bias only in
 * words; the formula above is this library's reading. q and kk are rotated
 * here by RoPE (rotate-half, theta_i = rope_base^(-2i/dh)) at the original
 * positions pos. Query head h reads KV head h / (hq / hkv).
 *   q [k, hq, dh], kk [k, hkv, dh], v [k, hkv, dh] dtype (un-rotated)
 *   pos [k] int32 strictly ascending; s [k] fp32 or NULL (no bias)
 *   gain [hq] fp32 or NULL (0); tau [hq] fp32 > 0 or NULL (1)
 *   out [k, hq, dh] dtype
 * bf16 needs dh == 128; fp32 needs dh in {64, 128}. hq % hkv == 0.
 */
tg_status tg_gated_attn_prefill(const void* q, const void* kk, const void* v, const int32_t* pos,
                                const float* s, const float* gain, const float* tau, int64_t k,
                                int32_t hq, int32_t hkv, int32_t dh, float rope_base,
                                tg_dtype dtype, void* out, void* ws, size_t ws_bytes,
                                tg_stream stream);

/*
 * tg_gated_attn_forward -- tg_gated_attn_prefill that also writes what its
 * backward takes:
 *   lse [hq, k] fp32: lse[h][i] = log sum_{j <= i} exp(l_ij), natural log.
 *   out_f32 [k, hq, dh] fp32 or NULL: the output before its rounding to
 *   bf16. The backward forms D_i = dout_i . o_i; from the bf16 output that
 *   product carries the output's rounding (2^-9 relative) into every
 *   gradient of row i, so pass this when exact-to-fp32 gradients matter.
 * bf16 (dh == 128) or fp32 (dh 64 or 128; out is then already fp32 and
 * out_f32 must be NULL); other arguments, workspace (TG_OP_GATED_ATTN) and
 * errors as tg_gated_attn_prefill. lse NULL, or out_f32 not 16-byte
 * aligned, is TG_ERR_INVALID_ARG.
 */
tg_status tg_gated_attn_forward(const void* q, const void* kk, const void* v, const int32_t* pos,
                                const float* s, const float* gain, const float* tau, int64_t k,
                                int32_t hq, int32_t hkv, int32_t dh, float rope_base,
                                tg_dtype dtype, void* out, float* lse, float* out_f32, void* ws,
                                size_t ws_bytes, tg_stream stream);

/*
 * tg_gated_attn_backward -- gradients of tg_gated_attn_forward for an
 * upstream gradient dout of its output. The top-K choice is discrete, but
 * the kept tokens' scores stay in the differentiable graph through the
 * attention bias, so the task loss reaches the scorer along loss -> upper
 * attention -> gate scores -> scorer, and the per-head gain and temperature
 * are learned with it ([TC] "门控机制为评分网络建立梯度路径"; [AI]
 * "可学习剪枝的机制设计"). The formulas are the chain rule of the forward's
 * logits (the pages give only the path):
 *   P_ij = exp(l_ij - lse_i), dl_ij = P_ij (dout_i . v_j - dout_i . o_i)
 *   dq_i = R_i^T sum_j dl_ij k'_j / (sqrt(dh) tau_h)
 *   dk_j = R_j^T sum_{h in group} sum_i dl_ij q'_i / (sqrt(dh) tau_h)
 *   dv_j = sum_{h in group} sum_i P_ij dout_i
 *   ds_j = sigmoid(-s_j) sum_h gain_h sum_i dl_ij
 *   dgain_h = sum_ij dl_ij logsigmoid(s_j),  dtau_h = -(1 / tau_h) sum_i q'_i . dq'_i
 * where q', k' are q, k rotated by RoPE R at their positions (as in the
 * forward) and dq' the gradient before the rotation back.
 *   q, kk, v, pos, s, gain, tau, k, hq, hkv, dh, rope_base: the forward's
 *   inputs, unchanged since that call.
 *   out [k, hq, dh] dtype, out_f32 [k, hq, dh] fp32 or NULL, lse [hq, k]
 *   fp32: the forward's outputs (D_i = dout_i . o_i is taken from out_f32
 *   when given, else from out).
 *   dout [k, hq, dh] dtype.
 *   dq [k, hq, dh], dk [k, hkv, dh], dv [k, hkv, dh] dtype (w.r.t. the
 *   un-rotated q and kk); ds [k] fp32 or NULL (needs s); dgain [hq] fp32 or
 *   NULL (0 when s is NULL); dtau [hq] fp32 or NULL.
 * bf16 with dh == 128 (tensor cores), or fp32 with dh 64 or 128 (CUDA
 * cores; out_f32 NULL); else TG_ERR_UNSUPPORTED. All bf16 buffers and ws
 * 16-byte aligned (else TG_ERR_INVALID_ARG). Workspace:
 * tg_workspace_size(TG_OP_GATED_ATTN_BWD) with k, heads, head_dim. The
 * result is deterministic (fixed summation orders, no atomics).
 */
tg_status tg_gated_attn_backward(const void* q, const void* kk, const void* v, const int32_t* pos,
                                 const float* s, const float* gain, const float* tau, int64_t k,
                                 int32_t hq, int32_t hkv, int32_t dh, float rope_base,
                                 tg_dtype dtype, const void* out, const float* out_f32,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                 float* ds,
                                 float* dgain, float* dtau, void* ws, size_t ws_bytes,
                                 tg_stream stream);

/*
 * tg_linear -- the backbone's projection GEMM, y = x . w^T (+ residual).
 * The dense contraction of every QKV / output / FFN projection in the layers
 * the gated stack runs ([TC] "TokenGate 提前筛选 Token": layers compute
 * attention and feed-forward per token); exposed on its own for users and
 * for measuring the kernel against a library GEMM.
 *   x [m, k], w [n, k], residual [m, n] or NULL (may equal y), y [m, n]; dtype
 * bf16: tcgen05 tensor cores, needs n % 32 == 0, k % 8 == 0, 16-byte aligned
 * pointers; fp32: CUDA-core GEMM, any sizes.
 */
tg_status tg_linear(const void* x, const void* w, const void* residual, int64_t m, int32_t n,
                    int32_t k, tg_dtype dtype, void* y, tg_stream stream);

/*
 * tg_fold_norm_weight -- W_g[j, i] = bf16(W[j, i] * g[i]): a projection
 * weight with the weight g of the RMSNorm in front of it folded in, for the
 * optional wqkv_g / w_gate_up_g / score_w1_g fields (the RMSNorm of
 * [TC] "TokenGate 提前筛选 Token"'s Qwen3 backbone and of the scorer's input
 * is y = x / sqrt(mean(x^2) + eps) * g, so y . W^T = (x . W_g^T) / rms(x)).
 * Device pointers: w and out [rows, cols] bf16 (out must not overlap w),
 * g [cols] fp32. rows, cols >= 1, else TG_ERR_INVALID_ARG, as for NULL
 * pointers. One kernel on `stream`, exact (one rounding per element).
 */
tg_status tg_fold_norm_weight(const void* w, const float* g, int64_t rows, int64_t cols, void* out,
                              tg_stream stream);

/* ---- hybrid models: the Gated DeltaNet mixer -----------------------------
 *
 * In a hybrid model most layers are Gated DeltaNet layers and only some are
 * full attention. The scorer reads hidden states, so the gate may sit at a
 * Gated DeltaNet layer. Above the gate the token-gated logit bias applies
 * only in the full-attention layers (tg_gated_attn_prefill); a Gated
 * DeltaNet layer has no logits and runs on the kept tokens as they are
 * ([TC] "门控位置影响剪枝效果", figure 5). The layer's projections are plain
 * GEMMs (tg_linear); this call is its token mixer over one sequence, the K
 * kept rows in ascending original order (the pages do not spell the layer
 * out; the mixer is the published gated delta rule of Yang, Kautz and
 * Hatamizadeh, "Gated Delta Networks", ICLR 2025, in the Qwen3-Next shape):
 *   c_t = SiLU(sum_{i<W} conv_w[:, i] * x_{t-W+1+i})  over the qkv channels
 *   q = l2norm(c_q) / sqrt(dk), k = l2norm(c_k), v = c_v  (l2norm: x / sqrt(|x|^2 + 1e-6))
 *   alpha = exp(-exp(A_log) * softplus(a_t + dt_bias)), beta = sigmoid(b_t)
 *   S_t = alpha S_{t-1} (I - beta k k^T) + beta v k^T,  o_t = S_t q  (per value head)
 *   y_t = o_t / sqrt(mean(o_t^2) + norm_eps) * norm_w * SiLU(z_t)    (per value head)
 * Value head h reads key head h / (hv / hk).
 */
typedef struct {
  int32_t n_heads_k;   /* hk                                               */
  int32_t n_heads_v;   /* hv, a multiple of hk                             */
  int32_t head_dim_k;  /* dk: 64 or 128                                    */
  int32_t head_dim_v;  /* dv: a multiple of 32, at most 256                */
  int32_t conv_width;  /* W: 1..4                                          */
  const float* conv_w; /* [C, W] with C = 2 hk dk + hv dv                  */
  const float* A_log;  /* [hv]                                             */
  const float* dt_bias;/* [hv]                                             */
  const float* norm_w; /* [dv]                                             */
  float norm_eps;
} tg_gdn_layer;

/* ---- the full stack ---------------------------------------------------- */

typedef struct {
  const float* attn_norm; /* [d]                                               */
  const void* wqkv;       /* [(hq + 2 hkv) dh, d]: rows of Wq, then Wk, then Wv */
  const float* q_norm;    /* [dh] per-head RMSNorm weight of q; NULL = off      */
  const float* k_norm;    /* [dh] same for k (both or neither)                  */
  const void* wo;         /* [d, hq dh]                                        */
  const float* ffn_norm;  /* [d]                                               */
  const void* w_gate_up;  /* [2 I, d]: rows of W_gate, then W_up; NULL = no FFN */
  const void* w_down;     /* [d, I]                                            */
  const float* gain;      /* [hq] gate-bias gain, layers above the gate; NULL=0 */
  const float* tau;       /* [hq] temperature, layers above the gate; NULL = 1  */
  /* A hybrid model's Gated DeltaNet layer: gdn != NULL makes the layer's
   * token mixer the Gated DeltaNet mixer (tg_gated_deltanet) instead of
   * attention: r = x + W_out . mixer(W_in . RMSNorm(x; attn_norm)), then the
   * same FFN sub-layer. wqkv, q_norm, k_norm, wo, gain and tau are unused. */
  const tg_gdn_layer* gdn; /* HOST pointer to the mixer's parameters, or NULL   */
  const void* w_in;       /* [C + hv dv + 2 hv, d]: rows giving qkv (C = 2 hk dk
                             + hv dv channels), then z, then a, then b          */
  const void* w_out;      /* [d, hv dv]                                         */
  /* Optional (bf16): the projections that read an RMSNorm-ed row, with that
   * norm's weight folded in, W_g[j, i] = bf16(W[j, i] g[i]) (made by
   * tg_fold_norm_weight): wqkv_g from wqkv and attn_norm, w_gate_up_g from
   * w_gate_up and ffn_norm. RMSNorm(x; g) . W^T = (x . W_g^T) / rms(x), so
   * with them a sub-layer whose input rows were just written by a residual
   * GEMM runs no RMSNorm kernel: that GEMM's epilogue leaves each row's sum
   * of squares (of the stored bf16 values) and the projection's epilogue
   * scales its accumulator row by 1 / rms(x) = 1 / sqrt(mean(x^2) + eps).
   * The rounding differs from the norm-then-project order only in where one
   * bf16 rounding falls (on W g instead of on the normed row). NULL: the
   * RMSNorm kernel and the plain weights (also used for rows that were not
   * just written by a residual GEMM: the stack's input; the compaction
   * carries the kept rows' sums of squares along, so they stay folded). */
  const void* wqkv_g;      /* [(hq + 2 hkv) dh, d] or NULL (unused with gdn)     */
  const void* w_gate_up_g; /* [2 I, d] or NULL                                   */
} tg_layer;

typedef struct {
  tg_dtype dtype;
  int32_t n_layers, d_model, n_heads_q, n_heads_kv, head_dim, d_ffn, d_score;
  float norm_eps, rope_base;
  const tg_layer* layers;   /* HOST array of n_layers entries (device pointers inside) */
  const float* final_norm;  /* [d] or NULL (no final norm)                    */
  const float* score_norm;  /* [d]                                           */
  const void* score_w1;     /* [F, d]                                        */
  const float* score_b1;    /* [F] or NULL                                   */
  const float* score_w2;    /* [F]                                           */
  const float* score_b2;    /* [1] or NULL                                   */
  const void* score_w1_g;   /* [F, d] score_w1 with score_norm folded in (as
                               tg_layer.wqkv_g), or NULL                     */
} tg_model;

/* Per-layer KV outputs (post-RoPE keys, values), each [rows, hkv, dh] dtype.
 * rows = n for layers <= gate_layer, k above it. NULL pointers skip a layer. */
typedef struct {
  void* k;
  void* v;
} tg_kv;

/*
 * tg_prefill -- the gated prefill of a decoder stack ([TC] "TokenGate 提前筛选
 * Token"; [FW]; [AI]).
 * Layers below gate_layer L run over all n tokens. Layer L runs attention
 * over all n tokens; the scorer reads its post-attention residual; the
 * selector keeps k tokens (protected ones always); layer L's FFN and every
 * layer above run over the k kept rows only, with token-gated attention at
 * the kept tokens' original positions, and make KV for those rows only.
 * Layers at and below L keep n-row KV ([TC] "TokenGate 的工程验证仍有限").
 * gate_layer = -1 puts the gate before layer 0 (the scorer reads x itself).
 * With k == n and every gain NULL/0 and tau NULL/1 the call is a dense
 * prefill.
 *   x [n, d] dtype (input hidden states, only read: layer 0 reads them in
 *     place, so x must stay valid until the stream reaches the end of the
 *     call's work); protect [n] uint8 or NULL
 *   out [k, d] dtype: final-normed hidden states of the kept rows
 *   kept_idx [k] int32 (out, ascending); scores [n] fp32 (out) or NULL
 *   kv: HOST array of n_layers tg_kv, or NULL (bf16: 16-byte aligned pointers)
 * Hybrid stacks: a layer with gdn != NULL runs the Gated DeltaNet mixer
 * over its rows in ascending original order (all n rows at and below the
 * gate, the k kept rows above it); the scorer then reads the post-mixer
 * residual when the gate sits at such a layer, and the gate bias applies
 * only to the attention layers above the gate ([TC] "门控位置影响剪枝效果",
 * figure 5). For such a layer kv[l].k receives the mixer's last W-1 conv
 * input rows [W-1, C] (dtype) and kv[l].v its final state [hv, dv, dk]
 * (fp32), which a following call continues from. bf16 only; the w_in
 * output width C + hv dv + 2 hv must be a multiple of 32.
 *   taps: HOST array of n_layers tg_layer_taps, or NULL. Each non-NULL
 *     pointer of taps[l] receives a copy of one intermediate of layer l, for
 *     inspection and per-layer checks (one device copy per requested tensor):
 *       attn_out [rows, hq dh]: the attention output before the output
 *         projection (rows = n at and below the gate, k above it); for a
 *         Gated DeltaNet layer the mixer output [rows, hv dv];
 *       resid [rows, d]: the residual stream after the attention sub-layer
 *         (x + Wo . attn_out; rows as attn_out);
 *       hidden [rows', d]: the layer's output after its FFN (rows' = n below
 *         the gate, k for the gate layer and above; kept rows ascending);
 *       mixer_in [rows, C + hv dv + 2 hv]: a Gated DeltaNet layer's input
 *         projection (qkv | z | a | b, the mixer's input); unused for
 *         attention layers.
 */
typedef struct {
  void* attn_out;
  void* resid;
  void* hidden;
  void* mixer_in;
} tg_layer_taps;

/*
 * tg_prefill_host -- tg_prefill with the input hidden states in HOST memory
 * (page-locked for the copies to be asynchronous): what a serving stack
 * calls when the prompt's hidden states come from the host. Same arguments,
 * results and workspace as tg_prefill (no taps), except that x is a host
 * pointer [n, d] dtype; protect, out, kept_idx, scores and kv stay device
 * pointers. The call copies x into its workspace; when the model runs bf16
 * paired-head attention at layer 0, the gate is at or above layer 0 and n >
 * 8192, the copy goes in 4096-row chunks on a library-owned stream, and the
 * RMSNorm, the fused QKV projection and the causal attention of each chunk's
 * rows run on `stream` as soon as the chunk has landed, so that the copy
 * overlaps layer 0 (the results are the same as tg_prefill's bit for bit).
 * Returns when the work is queued on `stream`; x must stay valid until the
 * stream reaches the end of the call's work. The chunked copy uses one
 * non-blocking stream per device (created on the first such call, kept for
 * the process) and a few CUDA events per call; no device memory is
 * allocated.
 */
tg_status tg_prefill_host(const tg_model* model, const void* x_host, const uint8_t* protect,
                          int64_t n, int64_t k, int32_t gate_layer, void* out, int32_t* kept_idx,
                          float* scores, const tg_kv* kv, void* ws, size_t ws_bytes,
                          tg_stream stream);

/* Workspace bytes of tg_prefill (and tg_prefill_multi with k = max(ks)) for
 * this model: tg_workspace_size(TG_OP_PREFILL) plus the buffers of a hybrid
 * stack's Gated DeltaNet layers (0 on invalid sizes). */
size_t tg_prefill_workspace_size(const tg_model* model, int64_t n, int64_t k);

tg_status tg_prefill(const tg_model* model, const void* x, const uint8_t* protect, int64_t n,
                     int64_t k, int32_t gate_layer, void* out, int32_t* kept_idx, float* scores,
                     const tg_kv* kv, const tg_layer_taps* taps, void* ws, size_t ws_bytes,
                     tg_stream stream);

/*
 * tg_prefill_multi -- the gated prefill at several budgets of one request
 * (the mixed-budget use the pages describe: one trained gate serves every
 * budget, and training averages the full-context loss with a random-budget
 * loss each step; [AI] "可学习剪枝的机制设计"; [TC] "门控机制为评分网络建立梯度路径").
 * The layers below the gate, the gate layer's attention and the scores do not
 * depend on the budget, so they run once; then each budget ks[b] gets its
 * own selection, compaction and upper layers, exactly as tg_prefill with that
 * k (the same kernels on the same data: the results are bit-identical).
 *   ks: HOST array of n_budgets budgets, 1 <= n_budgets <= TG_MAX_BUDGETS,
 *       each valid for tg_prefill (any order, repeats allowed)
 *   outs, kept_idx: HOST arrays of n_budgets device pointers; outs[b]
 *       [ks[b], d] dtype, kept_idx[b] [ks[b]] int32
 *   scores [n] fp32 (out) or NULL; no KV or per-layer outputs.
 * Workspace: tg_workspace_size(TG_OP_PREFILL) with k = max(ks).
 */
#define TG_MAX_BUDGETS 64
tg_status tg_prefill_multi(const tg_model* model, const void* x, const uint8_t* protect,
                           int64_t n, const int64_t* ks, int32_t n_budgets, int32_t gate_layer,
                           void* const* outs, int32_t* const* kept_idx, float* scores, void* ws,
                           size_t ws_bytes, tg_stream stream);

/*
 * tg_prefill_batch -- the gated prefill of a batch of independent requests
 * of different lengths in one call. Request b owns rows [cu_n[b], cu_n[b+1])
 * of x and keeps ks[b] of them. The projection GEMMs, the norms and the
 * scorer run over every request's rows at once (one GEMM per projection and
 * layer for the whole batch); attention, selection and compaction run per
 * request, each with its own positions 0..n_b-1, budget and protected span.
 * Each request's result is the one tg_prefill gives for it alone (the same
 * kernels on the same rows: bit-identical).
 *   cu_n: HOST array [batch + 1], cu_n[0] = 0, strictly increasing;
 *   ks: HOST array [batch], 1 <= ks[b] <= n_b; 1 <= batch <= TG_MAX_BATCH
 *   x [cu_n[batch], d] bf16; protect [cu_n[batch]] uint8 or NULL
 *   out [sum ks, d] bf16 and kept_idx [sum ks] int32: request b's rows at
 *     offset ks[0] + ... + ks[b-1]; kept indices are local to the request
 *     (0..n_b-1), ascending
 *   scores [cu_n[batch]] fp32 (out) or NULL; no KV or per-layer outputs.
 * bf16 with head_dim 128 only (TG_ERR_UNSUPPORTED otherwise). Internally
 * every request's rows start on a 128-row boundary, so the workspace covers
 * the padded counts: tg_prefill_batch_workspace_size (0 on invalid sizes).
 */
#define TG_MAX_BATCH 64
size_t tg_prefill_batch_workspace_size(const tg_model* model, const int64_t* cu_n,
                                       const int64_t* ks, int32_t batch);
tg_status tg_prefill_batch(const tg_model* model, const void* x, const uint8_t* protect,
                           const int64_t* cu_n, const int64_t* ks, int32_t batch,
                           int32_t gate_layer, void* out, int32_t* kept_idx, float* scores,
                           void* ws, size_t ws_bytes, tg_stream stream);

/* ---- decode over the pruned cache ---------------------------------------
 *
 * tg_decode_step -- one generated token through every layer after a gated
 * prefill. Generated tokens are never pruned ([TC] "TokenGate 提前筛选
 * Token"): the token runs every layer and appends its k and v to every
 * layer's cache. Layers at and below the gate hold the whole prompt's KV,
 * layers above it only the kept tokens' KV, and in decoding the gate bias
 * fixed at prefill acts as an additive mask over the cached keys ([TC]
 * "TokenGate 的工程验证仍有限"). Above the gate the logit of cache row j is
 * (q.k_j) / (sqrt(dh) tau_h) + gain_h logsigmoid(s_j) for the kept prompt
 * tokens (rows j < k_kept) and (q.k_j) / (sqrt(dh) tau_h) for generated ones.
 *   x [1, d] bf16: the token's input hidden state; pos: its position (the
 *     prompt is 0..n-1, the t-th generated token has pos n + t).
 *   kv: HOST array of n_layers caches, each k and v [cap_l, hkv, dh] bf16
 *     (keys after RoPE, as tg_prefill writes them), rows in position order.
 *   lens: HOST array of n_layers row counts before this step: n + t at or
 *     below the gate, k + t above. The token's k and v go to row lens[l];
 *     the caller sizes every cache for the rows it appends and advances lens.
 *   scores [n] fp32 and kept_idx [k_kept] int32: tg_prefill's outputs for
 *     an n-token prompt; the bias of upper-layer row j < k_kept is
 *     logsigmoid(scores[kept_idx[j]]). An index outside [0, n) gets no bias
 *     and sets bit 2 of the device error word. scores NULL: no gate bias.
 *   out [1, d] bf16: the token's final-normed hidden state.
 * bf16 and head_dim 128 only (TG_ERR_UNSUPPORTED otherwise); GQA groups of 1,
 * 2, 4 or 8 query heads; attention layers only (a Gated DeltaNet layer is
 * TG_ERR_UNSUPPORTED). Workspace: tg_workspace_size(TG_OP_DECODE) with
 * shape.k = k_kept. Asynchronous on the stream; validates on the host first.
 */
tg_status tg_decode_step(const tg_model* model, const void* x, int64_t pos, int32_t gate_layer,
                         const tg_kv* kv, const int64_t* lens, const float* scores, int64_t n,
                         const int32_t* kept_idx, int64_t k_kept, void* out, void* ws,
                         size_t ws_bytes, tg_stream stream);

/* ---- the Gated DeltaNet mixer on its own (tg_gdn_layer is above) -------- */

/* Workspace bytes of tg_gated_deltanet for T tokens (0 for a bad layer). */
size_t tg_gated_deltanet_workspace_size(const tg_gdn_layer* layer, int64_t T);

/*
 * tg_gated_deltanet -- the mixer above over T >= 0 tokens.
 *   qkv [T, C] dtype: the projections before the convolution, channels
 *     [q (hk dk) | k (hk dk) | v (hv dv)];  z [T, hv dv], a [T, hv],
 *     b [T, hv] dtype.
 *   conv_in [W-1, C] dtype or NULL (zeros): the rows before token 0;
 *   conv_out [W-1, C] dtype or NULL: the last W-1 rows of [conv_in; qkv],
 *     for a following call. Must not overlap conv_in.
 *   state_in [hv, dv, dk] fp32 or NULL (zeros); state_out [hv, dv, dk] fp32
 *     or NULL: S after the last token. state_out may equal state_in but not
 *     overlap it otherwise.
 *   y [T, hv dv] dtype.
 * Splitting a sequence across calls that carry conv_out / state_out into the
 * next call's conv_in / state_in gives the same result as one call, up to
 * rounding (the carried conv rows are stored in dtype, as the inputs are).
 * dtype bf16 or fp32; the arithmetic is fp32 throughout. ws 16-byte aligned.
 * Errors: null pointers, T < 0, bad layer sizes or overlapping state buffers
 * are TG_ERR_INVALID_ARG (dk other than 64/128 or dv outside the range is
 * TG_ERR_UNSUPPORTED); a short workspace is TG_ERR_WORKSPACE.
 */
tg_status tg_gated_deltanet(const tg_gdn_layer* layer, const void* qkv, const void* z,
                            const void* a, const void* b, int64_t T, tg_dtype dtype,
                            const void* conv_in, void* conv_out, const float* state_in,
                            float* state_out, void* y, void* ws, size_t ws_bytes,
                            tg_stream stream);

/* ---- launch tracing (optional) --------------------------------------------
 * Measurement aid with no counterpart on the pages (they report only
 * end-to-end prefill latency and memory). While tracing is on for a host
 * thread, every kernel the library launches from that thread is bracketed by
 * a pair of CUDA events on its stream, and the launch's algorithmic work
 * (FLOPs of the contraction, or bytes an ideal kernel must move) is noted.
 * Events are host-side driver objects created on first use; no device
 * memory is allocated. */

typedef enum {
  TG_K_COPY = 0,          /* device-to-device copy                          */
  TG_K_RMSNORM = 1,
  TG_K_GEMM_STORE = 2,    /* tcgen05 GEMM, plain store epilogue             */
  TG_K_GEMM_RESIDUAL = 3, /* tcgen05 GEMM, residual-add epilogue            */
  TG_K_GEMM_SWIGLU = 4,   /* tcgen05 GEMM, SiLU(gate)*up epilogue           */
  TG_K_GEMM_SCORE = 5,    /* tcgen05 GEMM, scorer-tail epilogue             */
  TG_K_ROPE_PREP = 6,     /* RoPE + qk-norm + V transpose + gate bias        */
  TG_K_ATTENTION = 7,     /* tcgen05 gated attention                        */
  TG_K_SELECT = 8,        /* the radix-select kernels of one top-K           */
  TG_K_COMPACT = 9,
  TG_K_GEMM_F32 = 10,     /* SIMT fp32 GEMM                                 */
  TG_K_ATTENTION_F32 = 11,
  TG_K_F32_HELPER = 12,   /* fp32 SwiGLU / scorer tail                      */
  TG_K_GEMM_QKV = 13,     /* tcgen05 GEMM, fused qk-norm + RoPE + V^T epilogue */
  TG_K_ROPE_TABLE = 14,   /* cos/sin table of one set of positions           */
  TG_K_DECODE_STEP = 15,  /* decode: one token through every layer (one launch) */
  TG_K_ATTN_BWD_PREP = 16,   /* backward: transposes, lse in log2 units, D = dout . o */
  TG_K_ATTN_BWD_DKDV = 17,   /* backward: dK, dV and the per-key sums of dl (tcgen05) */
  TG_K_ATTN_BWD_DQ = 18,     /* backward: dQ and q . dq (tcgen05)                   */
  TG_K_ATTN_BWD_FINAL = 19,  /* backward: ds, dgain, dtau                           */
  TG_K_GDN_PREP = 20,        /* Gated DeltaNet: conv, norms, decay (+ conv rows)     */
  TG_K_GDN_CHUNK = 21,       /* Gated DeltaNet: per-chunk solve matrices             */
  TG_K_GDN_RECUR = 22,       /* Gated DeltaNet: the state across the chunks          */
  TG_K_GDN_OUT = 23,         /* Gated DeltaNet: gated output RMSNorm                 */
  TG_K_FOLD_NORM = 24,       /* tg_fold_norm_weight                                  */
  TG_K_COUNT = 25
} tg_kernel;

typedef struct {
  int32_t kernel;  /* tg_kernel                                           */
  int32_t layer;   /* decoder layer of a tg_prefill launch, else -1        */
  int64_t rows;    /* rows (tokens) the launch processed                    */
  float ms;        /* device time between the bracketing events             */
  double flops;    /* algorithmic FLOPs of the launch (0 if memory-bound)   */
  double bytes;    /* algorithmic bytes of the launch                       */
} tg_trace_record;

/* Starts tracing on this host thread, for at most `capacity` launches. */
tg_status tg_trace_start(int32_t capacity);
/* Stops tracing, waits for the recorded events, and copies up to `cap`
 * records into `out` (HOST array). Returns the record count, or a negative
 * tg_status on failure. */
int32_t tg_trace_stop(tg_trace_record* out, int32_t cap);
/* Static name of a tg_kernel. */
const char* tg_kernel_name(int32_t kernel);

/* ---- diagnostics -------------------------------------------------------- */

/* Static description of a status code. */
const char* tg_status_string(tg_status status);

/* The CUDA error behind the last TG_ERR_CUDA on this host thread (0 if none). */
int tg_last_cuda_error(void);

/*
 * Reads (and with clear != 0, resets) the sticky device error word of the
 * current device: 0 when no kernel has reported a problem. Nonzero bits:
 * 1 = a bounded wait ran out, 2 = an index out of range was skipped.
 * This call synchronises the current device (a diagnostic, not for hot loops).
 */
tg_status tg_device_error(uint32_t* word, int clear);

/*
 * tg_selftest_wait_timeout -- exercises the failure detection of the
 * library's kernels without a fault. A kernel waits, with the same bounded
 * wait the library's kernels use, for an event that never comes; after
 * limit_ns it gives up, sets bit value 1 of the device error word (see
 * tg_device_error) and returns, leaving the stream and the context usable.
 * For tests and health checks; the pages have no counterpart.
 *   mode 0: four warps wait on a shared-memory mbarrier (the wait of the
 *           TMA / tensor-core pipelines) that nothing completes;
 *   mode 1: the same, but the mbarrier completes: every wait succeeds;
 *   mode 2: one CTA waits at the grid barrier of the cooperative decode
 *           kernel, which no other CTA reaches.
 *   limit_ns in [1000, 1e9]; result [4] int32 device (out), 16-byte aligned:
 *   result[i] = 1 when wait i (warp i; mode 2: result[0]) completed, 0 when
 *   it gave up. ws: mode 2 only, >= 16 bytes, 16-byte aligned (the barrier's
 *   words, cleared by the call).
 */
tg_status tg_selftest_wait_timeout(int32_t mode, int64_t limit_ns, int32_t* result, void* ws,
                                   size_t ws_bytes, tg_stream stream);

/* Library version string. */
const char* tg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H */
