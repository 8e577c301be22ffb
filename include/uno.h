/*
 * uno.h -- C ABI of libuno: the Psi-Spec decode iteration of a diffusion-
 * augmented LLM ("Uno") on one NVIDIA B200 (sm_100a).
 *
 * The method ("Unlocking Lossless Speedups in LLMs via Discrete Diffusion"):
 * one causal Transformer keeps its AR weights W_base frozen and carries
 * "diffusion weights" W_diff as a gated rank-r LoRA on every layer (summary
 * page "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型", section 方法关键点).
 * One decode iteration drafts a block of B tokens in parallel with
 * W_base + W_diff from a fully noised block, the first token from W_base
 * alone; the AR path (W_base only) then scores the whole block, the longest
 * accepted prefix is kept and the first rejected position is redrawn from the
 * renormalised residual max(0, p_AR - q_diff) (blog page "不砸掉重来，给自回归
 * LLM 装一对“扩散翅膀”：Uno 的无损加速之路", sections 一句话直觉 and
 * Ψ-Spec 采样器：起草、验证、两种模式).  Draft and verify share one KV cache
 * (same page, section 一句话直觉).  Every iteration runs two forwards and
 * emits between 2 and B+1 tokens per request.
 *
 * Conventions of every call:
 *  - Return value: UNO_OK (0) or one of the UNO_ERR_* codes; no exception
 *    crosses the ABI.  uno_last_error() gives a message for the last failure
 *    of a context.
 *  - "dev" pointers are CUDA device pointers, "host" pointers host memory.
 *  - All device work is enqueued on the context's stream and is
 *    asynchronous: outputs are valid once the caller synchronises that
 *    stream.  No call inside the decode loop synchronises the host.
 *  - Weights are borrowed: caller-owned device buffers that must outlive the
 *    context.  The library owns the KV pool, the page tables and all
 *    workspaces.  Output buffers are caller-owned.
 *  - Weight matrices are row-major [out_features, in_features]
 *    (torch.nn.Linear layout), dense, in the model dtype; LoRA A is
 *    [r, in_features] and LoRA B is [out_features, r].
 */
#ifndef UNO_H_
#define UNO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque context. */
typedef struct uno_ctx uno_ctx;

/* A cudaStream_t passed as an opaque pointer (NULL: the legacy default stream). */
typedef void *uno_stream_t;

enum uno_dtype { UNO_F32 = 0, UNO_BF16 = 1 };

enum uno_status_code {
  UNO_OK = 0,
  UNO_ERR_ARG = 1,          /* invalid argument (NULL, size out of range, unknown id)   */
  UNO_ERR_OOM = 2,          /* device allocation failed                                   */
  UNO_ERR_CAPACITY = 3,     /* no free request slot or KV pages                           */
  UNO_ERR_CUDA = 4,         /* a CUDA runtime call failed                                 */
  UNO_ERR_DEVICE_CHECK = 5, /* a device-side bounds check fired (see uno_status)          */
  UNO_ERR_UNSUPPORTED = 6   /* shape or dtype this build has no kernel for                */
};

/* Projections carrying a LoRA, in this order. */
enum uno_proj {
  UNO_PROJ_Q = 0, UNO_PROJ_K, UNO_PROJ_V, UNO_PROJ_O, UNO_PROJ_GATE, UNO_PROJ_UP, UNO_PROJ_DOWN,
  UNO_N_PROJ
};

/*
 * Model shape.  Pre-RMSNorm decoder: x += o(attn(rope(q), rope(k), v)) with
 * GQA (q head h reads kv head h / (n_heads / n_kv_heads)); x += down(silu(gate)
 * * up); untied embedding / LM head; rotate-half RoPE with rope_theta; logits
 * divided by temperature.  mask_id is the reserved token id of the noised
 * block (the absorbing-state noise prior).
 */
typedef struct uno_shape {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn_dim, vocab, mask_id;
  float rope_theta, rms_eps, temperature;
  int32_t dtype; /* enum uno_dtype: UNO_F32 (all kernels in fp32) or UNO_BF16 */
} uno_shape;

/*
 * Weights (device pointers in the model dtype).  Per-layer entries are HOST
 * arrays of n_layers device pointers; the arrays are copied by uno_init.
 *   embed [vocab, d_model], lm_head [vocab, d_model], final_norm [d_model]
 *   attn_norm[l], ffn_norm[l]          [d_model]
 *   w[p][l]                             projection p of layer l, [out, in]
 *   lora_A[p][l] [r, in], lora_B[p][l]  [out, r]
 */
typedef struct uno_weights {
  const void *embed, *lm_head, *final_norm;
  const void *const *attn_norm;
  const void *const *ffn_norm;
  const void *const *w[UNO_N_PROJ];
  const void *const *lora_A[UNO_N_PROJ];
  const void *const *lora_B[UNO_N_PROJ];
} uno_weights;

/*
 * Create a context.
 *   lora_rank, lora_alpha: the LoRA scale is alpha / rank.
 *   block_B:   drafted block size B (2 <= B <= 64).
 *   max_batch: request slots; max_ctx: tokens one request may hold (prompt
 *              plus generated).  The KV pool (element type: see
 *              uno_debug_kv) holds max_batch * ceil((max_ctx + B + 2) / 64)
 *              pages of 64 tokens.  bf16 models whose pool reaches 2^31
 *              rows of head_dim (n_layers x pages x 3 planes x n_kv_heads x
 *              64) run the SIMT attention instead of the tensor-core one.
 *   seed:      Philox key of every uniform the sampler draws.
 *   stream:    every later call enqueues on this stream.
 * On success *out receives the context (free it with uno_destroy).
 */
int uno_init(const uno_shape *shape, const uno_weights *weights, int lora_rank, float lora_alpha,
             int block_B, int max_batch, int max_ctx, uint64_t seed, uno_stream_t stream,
             uno_ctx **out);

/*
 * Admit n_req requests and prefill them.
 *   prompts_dev:  int32 [n_req, prompt_stride] token ids (device).
 *   prompt_lens_host: int32 [n_req], each in [1, max_ctx].
 *   streams_host: optional uint32 [n_req] random-stream ids (NULL: the slot id).
 *   req_ids_host_out: int32 [n_req] receives each request's slot id.
 * Every prompt token but the last is run through the model with the LoRA
 * gated off and cached; the last becomes the request's pending token.
 * Fails with UNO_ERR_CAPACITY before any launch when slots run out.
 */
int uno_prefill(uno_ctx *ctx, int n_req, const int32_t *prompts_dev, int prompt_stride,
                const int32_t *prompt_lens_host, const uint32_t *streams_host,
                int32_t *req_ids_host_out);

/*
 * The training-form forward (blog page "…Uno 的无损加速之路", section Diffusion
 * Distillation：一步蒸馏 + 块级扩散): one pass over the concatenation [x, z] of
 * a clean sequence x and its noised copy z (2L rows, context 2L) with the
 * block-causal mask - a clean token sees the clean tokens up to its own
 * position; a noised token sees the clean tokens before its block (blocks of
 * B positions from position 0) and the noised tokens of its own block up to
 * its own position - and the adapter gated off on x and on on z, so one
 * forward gives the AR (teacher) logits of x and the diffusion (student)
 * logits of z.  Forward only: no loss (the pages' loss formulas are missing).
 *   tokens_dev: int32 [n_seq, 2L] (device): x_0..x_{L-1}, then z_0..z_{L-1}
 *               (z_i at position i; the noise prior's tokens, e.g. MASK).
 *   logits_dev: f32 [n_seq, 2L, vocab] (device, caller-owned), row order as
 *               the tokens.
 * Needs n_seq * 2L <= max(512, max_batch * (B + 1)) rows (else
 * UNO_ERR_CAPACITY), L <= max_ctx, and 2 n_seq free request slots (their
 * pages hold the clean and the noised keys during the call and are free
 * again after it).  Stream-ordered, no host synchronisation after the setup.
 */
int uno_train_forward(uno_ctx *ctx, int n_seq, const int32_t *tokens_dev, int L, float *logits_dev);

/*
 * One Psi-Spec iteration for n_req admitted requests (req_ids_dev: int32
 * [n_req] slot ids, distinct, device).  Outputs (device, caller-owned):
 *   out_tokens_dev int32 [n_req, B+1]: the emitted tokens (first n_new valid);
 *   n_new_dev      int32 [n_req]: emitted count, in [2, B+1].
 * The request's cache advances by n_new tokens and its pending token becomes
 * the last emitted one.  A request whose cache would exceed its pages is
 * left unchanged and raises the device check flag (see uno_status).
 */
int uno_spec_step(uno_ctx *ctx, int n_req, const int32_t *req_ids_dev, int32_t *out_tokens_dev,
                  int32_t *n_new_dev);

/*
 * Cohort-interleaved Psi-Spec steps (the gated LoRA lets one forward compute
 * both paths - blog page "…Uno 的无损加速之路", section Diffusion Distillation：
 * 一步蒸馏 + 块级扩散 - so two request cohorts can run out of phase and share
 * each weight tile of a forward).  One call runs ONE forward over
 *   the drafting cohort  (draft_ids_dev, int32 [n_draft] slots): its draft
 *                        rows [pending, MASK x B], then draft_sample; the
 *                        block and the draft logits stay with the request;
 *   the verifying cohort (verify_ids_dev, int32 [n_verify] slots, drafted by
 *                        an earlier call): its verify rows x_1..x_B (plus x_B
 *                        once more, so every request has B + 1 rows), then
 *                        spec_verify and the commit, which emit into
 *                        out_tokens_dev int32 [n_verify, B+1] and
 *                        n_new_dev int32 [n_verify].
 * A request alternates: drafted by one call, verified by a later one (any
 * number of calls in between, no uno_spec_step on it meanwhile).  Each
 * request's tokens are exactly those of uno_spec_step (same uniforms, keyed
 * by request and position).  Either cohort may be empty (not both); slots
 * must be distinct; a request in the wrong phase raises the device flag.
 * The first call allocates the per-slot buffers (once, before any stream
 * capture; 2 * max_batch * (B+1) * vocab fp32 logits).  top_p < 1:
 * UNO_ERR_UNSUPPORTED.  Graph capture as for uno_spec_step (keyed by all
 * four pointers and both counts).
 */
int uno_spec_step_cohorts(uno_ctx *ctx, int n_draft, const int32_t *draft_ids_dev, int n_verify,
                          const int32_t *verify_ids_dev, int32_t *out_tokens_dev, int32_t *n_new_dev);

/* AR-only decode (baseline): one forward, the LoRA off, one token per request
 * into out_tokens_dev int32 [n_req]. */
int uno_ar_step(uno_ctx *ctx, int n_req, const int32_t *req_ids_dev, int32_t *out_tokens_dev);

/* CUDA graphs (no counterpart on the pages: launch plumbing).  With graphs on
 * (the default), the first uno_spec_step / uno_ar_step call with a given
 * (n_req, req_ids_dev, output pointers) runs eagerly, the second captures the
 * step into a CUDA graph on an internal stream and launches it on the
 * context stream, and later calls replay it.  Calls while profiling run
 * eagerly.  enable = 0 turns capture off (already captured graphs are kept
 * but not used). */
int uno_set_graphs(uno_ctx *ctx, int enable);

/* Programmatic dependent launch (launch plumbing, on by default): each kernel
 * may start while the previous one finishes and waits inside for its data
 * (the tensor-core GEMM starts streaming weights first).  enable = 0 launches
 * kernels in plain stream order.  Changing it drops captured graphs. */
int uno_set_pdl(uno_ctx *ctx, int enable);

/* Completion counters in the fused layer pipeline (implementation choice,
 * on by default).  A kernel then waits for the one right before it through a
 * counter that kernel's CTAs increment as they finish, instead of waiting for
 * that whole grid to be retired: each projection GEMM for the epilogue that
 * wrote its input rows (its weight stream has started before either wait),
 * each epilogue for its GEMM's parts, the attention for the q|k|v epilogue
 * and the split merge for the attention (the o projection keeps the grid
 * wait on the merge).  The counters are zeroed by each pass's first kernel.
 * A wait that outlasts about a second gives up and raises the device flag
 * (uno_status returns UNO_ERR_DEVICE_CHECK).  enable = 0 uses grid
 * dependencies only.  Changing it drops captured graphs. */
int uno_set_counter_sync(uno_ctx *ctx, int enable);

/* Fused layer pipeline (implementation choice, on by default where it
 * applies: passes of at most 128 rows of bf16 models with head_dim 64 or
 * 128, d_model, ffn_dim and the q / kv widths multiples of 128, d_model <=
 * 8192, LoRA rank 0 or 128).  Each projection
 * GEMM then leaves fp32 parts that one epilogue kernel reduces and carries
 * through LoRA-B, the RMSNorm scale, RoPE and the KV write, SwiGLU or the
 * residual add; the LoRA A matrices stream with the base weights.  enable =
 * 0 runs the unfused kernels (separate rank-r GEMMs, norm, RoPE, SwiGLU).
 * Changing it drops captured graphs.  Returns UNO_ERR_UNSUPPORTED (after
 * recording the setting) when the model does not take the fused pipeline. */
int uno_set_fused(uno_ctx *ctx, int enable);

/* spec_verify's form (implementation choice): when a step's verification
 * has more than max_ctas (row, vocabulary chunk) CTAs (default 4096), it
 * runs as a reduction kernel (two chunks of a row per CTA) whose CTAs carry
 * no counters plus one CTA per request that combines the rows and decides;
 * otherwise as one fused kernel whose last CTAs combine and decide.  Both
 * give the same tokens.  0 forces the split form.  Changing it drops
 * captured graphs.  max_ctas < 0: UNO_ERR_ARG. */
int uno_set_verify_split(uno_ctx *ctx, int max_ctas);

/*
 * Benchmark tap (no counterpart on the pages; never used by the parity
 * tests): force the accepted length of every later uno_spec_step to
 * a (1 <= a <= B: the first token plus a - 1 accepted drafts), whatever the
 * accept tests say; the token after the prefix is still drawn from the
 * residual (a < B) or the bonus row (a = B).  Random-init weights accept
 * few drafts, so this gives a step at the acceptance of a trained drafter
 * (the pages convert decode steps to tokens by the average tokens per
 * forward).  a <= 0 turns it off; a > B: UNO_ERR_ARG.  Drops captured graphs.
 */
int uno_debug_set_fixed_accept(uno_ctx *ctx, int a);

/*
 * Test tap of the bounded waits (no counterpart on the pages): every later
 * completion-counter wait of the fused pipeline (see uno_set_counter_sync)
 * gives up after limit_ns nanoseconds (default 1e9), and `extra` is added to
 * every counter's target, so extra > 0 makes each such wait run out: the
 * waiting GEMM then raises the device flag (uno_status returns
 * UNO_ERR_DEVICE_CHECK) and goes on, so the step ends with meaningless
 * results instead of hanging.  extra = 0 restores normal waits.
 * limit_ns = 0: UNO_ERR_ARG.  Drops captured graphs.
 */
int uno_debug_set_dep_wait(uno_ctx *ctx, uint64_t limit_ns, uint32_t extra);

/*
 * Tree sampler (summary page "通过离散扩散实现 LLM 无损加速：扩散增强自回归模型",
 * section 方法关键点: the linear sampler serves system throughput, the tree
 * sampler per-request throughput at batch 1; the blog page's description of
 * the two candidate-set modes is lost).  With k >= 2, every later
 * uno_spec_step drafts k chains that share the AR first token x_1 - chain j
 * draws positions 2..B from the drafter's rows with its own uniforms - and
 * verifies all of them in one verify pass (k B rows per request); the walk
 * then accepts, at each position, one of the candidates by recursive
 * rejection: at position 2 every chain's token (chain order), later the
 * continuing chain's token first and then the other chains' tokens, which end
 * the block when accepted (no AR row conditions on them).  A rejection
 * replaces the target by max(0, r - q) renormalised; when every candidate is
 * rejected the token is drawn from the last target.  Emits 2 .. B+1 tokens
 * per request like the linear sampler and follows the AR distribution
 * exactly.  k = 1 is the linear sampler (the default).
 * Each request slot keeps 2 k scratch KV pages for its chains, taken from the
 * free pages when the setting is made (UNO_ERR_CAPACITY if there are too
 * few: leave spare request slots); k = 1 gives them back.  A step needs
 * n_req * k * B <= max(512, max_batch * (B + 1)) rows (else
 * UNO_ERR_CAPACITY); top_p < 1 with the tree: UNO_ERR_UNSUPPORTED.
 * Synchronises the stream; drops captured graphs.  k outside [1, 4]:
 * UNO_ERR_ARG.
 */
int uno_set_tree(uno_ctx *ctx, int k);

/*
 * Nucleus (top-p) sampling (blog page "…Uno 的无损加速之路", section 我的判断:
 * the evaluation setting is temperature 1 with top-p 0.95, and losslessness
 * holds with respect to that sampling distribution).  With top_p < 1 every
 * row a later step samples or verifies - the AR rows p and the drafter's
 * rows q alike - is restricted to its nucleus: the smallest set of most
 * probable tokens whose probability reaches top_p (tokens ordered by
 * probability, ties by token id; the token that crosses top_p is kept), and
 * renormalised.  Drafting, the accept tests, the residual max(0, p - q), the
 * bonus token and uno_ar_step all see the filtered distributions, so the
 * output follows the AR model's filtered distribution.  top_p = 1 (the
 * default) turns the filter off; top_p outside (0, 1]: UNO_ERR_ARG.  Drops
 * captured graphs.
 */
int uno_set_top_p(uno_ctx *ctx, float top_p);

/*
 * The nucleus of rows of logits as a stand-alone kernel (the filter
 * uno_set_top_p applies, one CTA per row):
 *   logits_dev: f32 [rows, vocab] (device, 16-byte aligned, vocab % 4 == 0);
 *   top_p in (0, 1);
 *   out_dev:    int32 [rows, 2] (device): per row the order-preserving key
 *               of the crossing logit l* (the float's bits b, as unsigned:
 *               ~b if the sign is set, else b | 0x80000000; -0 counts as +0)
 *               and id_cut.  Token v is in the nucleus iff key(l_v) > key
 *               or (key(l_v) == key and v <= id_cut).
 * The probability masses are summed as exact fixed-point integers (weights
 * exp(l - max) in units of 2^-40), so the result is deterministic.  Never
 * synchronises; UNO_ERR_ARG on bad sizes or pointers.
 */
int uno_top_p_filter(const float *logits_dev, int rows, int vocab, float top_p, int32_t *out_dev,
                     uno_stream_t stream);

/* Free a request's slot and pages (stream-ordered after earlier work). */
int uno_release(uno_ctx *ctx, int req_id);

/* Synchronise the context's stream, free everything. */
int uno_destroy(uno_ctx *ctx);

/* Message of the last failed call on ctx ("" if none); valid until the next call. */
const char *uno_last_error(const uno_ctx *ctx);

/* Synchronise the stream and return UNO_ERR_DEVICE_CHECK if a device-side
 * bounds check fired since the last call (the flag is then cleared). */
int uno_status(uno_ctx *ctx);

/* Read a request's state (synchronises): cached token count, pending token. */
int uno_request_state(uno_ctx *ctx, int req_id, int32_t *cached_out, int32_t *pending_out);

/*
 * Debug taps (synchronous copies of internal buffers of the LAST step, for
 * stage-by-stage parity tests; not for production use).
 *   UNO_DBG_LOGITS_DRAFT  f32   [n_req, B+1, vocab] draft-pass logits
 *   UNO_DBG_LOGITS_VERIFY f32   [n_req, B, vocab]   verify-pass logits
 *   UNO_DBG_DRAFTS        int32 [n_req, B]          drafted block x_1..x_B
 *   UNO_DBG_LOGITS_AR     f32   [n_req, vocab]      AR-step logits
 *   UNO_DBG_TOPP_DRAFT    int32 [n_req, B+1, 2]     nucleus of each draft row (top_p < 1;
 *                                                   row 1 unused; AR step: [n_req, 1, 2])
 *   UNO_DBG_TOPP_VERIFY   int32 [n_req, B, 2]       nucleus of each verify row
 *   UNO_DBG_COHORT_LOGITS f32   [2 max_batch, B+1, vocab]  cohort step: the draft logits
 *                               of each slot (rows [slot]), then the last call's
 *                               verify logits (rows [max_batch + i], i-th verified)
 *   UNO_DBG_COHORT_DRAFTS int32 [max_batch, B]      cohort step: drafted block per slot
 *   UNO_DBG_TREE_CHAINS   int32 [n_req, k, B]       tree sampler: the drafted chains
 *                               (x_1, y_j2 .. y_jB) of the last step
 *   UNO_DBG_TREE_LOGITS   f32   [n_req, k, B, vocab] tree sampler: each chain's verify logits
 *   UNO_DBG_TREE_WALK     int32 [n_req, 3]          tree sampler: c, accepted path length m,
 *                               the path's chain
 * A nucleus entry is (key, id_cut) as uno_top_p_filter writes it.  The
 * logits are those of the model (before any nucleus filter).
 * bytes must not exceed the buffer's size for max_batch requests.
 */
enum uno_debug_buf {
  UNO_DBG_LOGITS_DRAFT = 0, UNO_DBG_LOGITS_VERIFY = 1, UNO_DBG_DRAFTS = 2, UNO_DBG_LOGITS_AR = 3,
  UNO_DBG_TOPP_DRAFT = 4, UNO_DBG_TOPP_VERIFY = 5, UNO_DBG_COHORT_LOGITS = 6,
  UNO_DBG_COHORT_DRAFTS = 7, UNO_DBG_TREE_CHAINS = 8, UNO_DBG_TREE_LOGITS = 9, UNO_DBG_TREE_WALK = 10
};
int uno_debug_read(uno_ctx *ctx, int which, void *dst_host, size_t bytes);

/* Copy keys and values of positions [pos0, pos0+n) of layer `layer` of a
 * request to host buffers k_host, v_host, each [n, n_kv_heads, head_dim] in
 * the cache's element type: fp32 for fp32 models, fp16 for bf16 models (the
 * attention operands q, K, V and P of a bf16 model are fp16: two bytes like
 * bf16, with three more mantissa bits; q and K are kept as fp16 hi/lo pairs,
 * and the keys returned here are the high parts).  Synchronises.  Keys are
 * stored after RoPE. */
int uno_debug_kv(uno_ctx *ctx, int req_id, int layer, int pos0, int n, void *k_host,
                 void *v_host);

/*
 * gated_lora_linear as a stand-alone call: the projection the diffusion and
 * AR paths share, with the adapter switched per row (summary page "通过离散
 * 扩散实现 LLM 无损加速：扩散增强自回归模型", section 方法关键点: rank-r LoRA
 * diffusion weights on every layer; blog page "…Uno 的无损加速之路", section
 * Diffusion Distillation：一步蒸馏 + 块级扩散: the gate switches the adapter off
 * at clean positions and on at noised ones):
 *
 *   U = round(gate[m] * scale * X A^T)           [M, r], model dtype
 *   Y = X W^T + U Bl^T                            [M, N], fp32
 *
 *   dtype: UNO_F32 or UNO_BF16 (X, W, A, Bl in that dtype, row-major dense:
 *   X [M, K], W [N, K], A [r, K], Bl [N, r]); A == NULL: no adapter (r
 *   ignored); gate_dev: f32 [M] or NULL (all rows gated on).
 *   workspace_dev: at least uno_gated_lora_linear_workspace_bytes() bytes,
 *   256-byte aligned, zero-filled before its first use (left zeroed after);
 *   calls sharing one workspace must not overlap on the GPU.
 * bf16 shapes with K and r multiples of 64 run on the tcgen05 kernel; the
 * others on the SIMT kernel.  Never synchronises.
 */
size_t uno_gated_lora_linear_workspace_bytes(int M, int N, int K, int r, int dtype);
int uno_gated_lora_linear(int dtype, const void *X_dev, const void *W_dev, const void *A_dev,
                          const void *Bl_dev, const float *gate_dev, int M, int N, int K, int r,
                          float scale, float *Y_dev, void *workspace_dev, size_t workspace_bytes,
                          uno_stream_t stream);

/* Diagnostic (no counterpart on the pages): process-wide launch counts of
 * out[0] tensor-core GEMM, out[1] SIMT GEMM, out[2] tensor-core attention,
 * out[3] SIMT attention kernels, so a caller can tell which path ran. */
int uno_debug_launch_counts(int64_t *out);

/*
 * Profiling tap (no counterpart on the pages: measurement plumbing).
 * Kernel classes: the gated-LoRA GEMMs (incl. the LM head), attention,
 * draft_sample / AR sampling, spec_verify, and everything else (row assembly,
 * norms, RoPE/KV write, SwiGLU).
 * uno_profile_begin zeroes the counters and, for every class in
 * class_mask (bit 1 << class), records a CUDA event pair around each launch
 * on the context stream.  uno_profile_end synchronises and fills, per class
 * (arrays of UNO_K_N), the launch count (all classes), the summed event time
 * in ms (profiled classes, else 0) and the algorithmic bytes those launches
 * move (weights, activations and outputs read/written once; KV bytes are
 * not known on the host and are not included for attention).
 */
enum uno_kernel_class { UNO_K_GEMM = 0, UNO_K_ATTN, UNO_K_SAMPLE, UNO_K_VERIFY, UNO_K_OTHER, UNO_K_N };
int uno_profile_begin(uno_ctx *ctx, unsigned class_mask);
int uno_profile_end(uno_ctx *ctx, int64_t *launches, double *ms, double *bytes);
/* One profiled launch: its class, for GEMMs the shape (rows m, columns n,
 * depth k, adapter rank r or 0), and its event time. */
typedef struct uno_prof_record {
  int32_t cls, m, n, k, r;
  float ms;
} uno_prof_record;
/* Copies up to max records of the last uno_profile_end into out (may be NULL)
 * and returns how many there are (negative on a bad context). */
int uno_profile_records(uno_ctx *ctx, uno_prof_record *out, int max);

/*
 * spec_verify as a stand-alone kernel: the rejection step of speculative
 * sampling over drafted blocks (blog page "…Uno 的无损加速之路", section
 * Ψ-Spec 采样器：起草、验证、两种模式: verify the block in parallel, keep the
 * longest accepted prefix, redraw the first rejected token from the
 * renormalised residual max(0, p - q)).
 *
 *   p_dev, q_dev:  f32 [n_req, n_tests, vocab] AR / drafter logits (device);
 *                  row j of request i scores draft drafts_dev[i, j].
 *   drafts_dev:    int32 [n_req, n_tests] drafted tokens.
 *   streams_dev:   uint32 [n_req] random-stream id of each request.
 *   pos0_dev:      int32 [n_req] position of test 0; test j draws its accept
 *                  uniform at position pos0 + j, the redraw at pos0 + a.
 *   seed:          Philox key.
 *   n_out_dev      int32 [n_req]: a, the length of the accepted prefix, in
 *                  [0, n_tests].
 *   out_tokens_dev int32 [n_req, n_tests+1]: the a accepted drafts, then at
 *                  index a the token redrawn from max(0, p_a - q_a)
 *                  renormalised; -1 there when a == n_tests (no bonus row is
 *                  given, so no further token is drawn).
 *   workspace_dev: scratch of at least uno_spec_verify_workspace_bytes()
 *                  bytes, 256-byte aligned, zero-filled before its first use
 *                  (the kernels leave its counters zeroed again); calls
 *                  sharing a workspace must not overlap on the GPU.
 * Enqueues on `stream` the vocabulary reductions with the accept tests (one
 * kernel for up to 4096 (row, 8192-logit chunk) CTAs; above that a
 * reduction kernel and one deciding CTA per request), then the residual
 * redraw of each request with a rejection.  Returns UNO_ERR_ARG on bad
 * sizes; never synchronises.
 */
size_t uno_spec_verify_workspace_bytes(int n_req, int n_tests, int vocab);
int uno_spec_verify(const float *p_dev, const float *q_dev, const int32_t *drafts_dev,
                    int n_req, int n_tests, int vocab, uint64_t seed,
                    const uint32_t *streams_dev, const int32_t *pos0_dev,
                    int32_t *out_tokens_dev, int32_t *n_out_dev, void *workspace_dev,
                    size_t workspace_bytes, uno_stream_t stream);

/*
 * uno_spec_verify_noalloc: uno_spec_verify for callers that cannot allocate
 * device memory at the point of the call (the pages have no counterpart: this
 * is deployment plumbing).  Examples: a serving process whose device memory
 * is handed out up front by its own pool, where an extra cudaMalloc would fail
 * or exceed the budget; or a caller that cannot afford the device-wide
 * synchronisation that cudaMalloc / cudaFree may imply.  Instead of a
 * workspace, the call uses a fixed scratch array of
 * uno_spec_verify_noalloc_max_bytes() bytes (4 MiB) that lives in the
 * library's device image: every GPU that loads the library holds it until
 * the process exits.  It allocates nothing (no cudaMalloc, cudaFree or other
 * allocating routine).
 *   Arguments, outputs and results are those of uno_spec_verify.
 *   Every argument is checked before anything is enqueued: invalid ones give
 *   UNO_ERR_ARG, and sizes whose workspace (uno_spec_verify_workspace_bytes)
 *   exceeds the array give UNO_ERR_CAPACITY; a rejected call touches neither
 *   the array nor the stream.
 *   The first call on a device looks up the array's device address on that
 *   device (it must be the current device) and caches it with the id of the
 *   device's CUDA context; a call in a new context (after cudaDeviceReset)
 *   looks it up again.  Make the first call on a device, and the first one
 *   after a reset, before any stream capture.
 *   All calls share the one array, which keeps the previous call's contents;
 *   each call clears the part that must start at zero (its completion
 *   counters) on the given stream before the kernels.  Calls that overlap on
 *   the GPU (different streams, no ordering between them) race on the array
 *   and give wrong results: serialise them.
 */
size_t uno_spec_verify_noalloc_max_bytes(void);
int uno_spec_verify_noalloc(const float *p_dev, const float *q_dev, const int32_t *drafts_dev,
                            int n_req, int n_tests, int vocab, uint64_t seed,
                            const uint32_t *streams_dev, const int32_t *pos0_dev,
                            int32_t *out_tokens_dev, int32_t *n_out_dev, uno_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* UNO_H_ */
