/*
 * dec.h -- C ABI of a batch-1 transformer decode step run as one persistent
 * CUDA kernel per step on an NVIDIA B200 (sm_100a), or a whole generation of
 * many steps in one launch (dec_generate*).
 *
 * The problem statement follows the pages on TileRT (SemiAnalysis, "Ultra-High
 * Interactivity on NVIDIA GPUs? -- TileRT InferenceX", and "TileRT 是什么"):
 *   - decode only, batch 1: prefill runs in another engine, which hands over
 *     its KV cache (InferenceX article, PD disaggregation section);
 *   - a lifecycle of init / step / reset / cleanup (TileRT 是什么 §六 6.1: the
 *     prepare_money / show_hands / reset / go_home entry points);
 *   - the whole decode step as one persistent kernel whose tile tasks overlap
 *     weight streaming with compute, launched once for a decode lifetime
 *     (InferenceX article, "what TileRT is"; TileRT 是什么 §二 2.2, tile-level
 *     runtime engine);
 *   - model structure: dense GQA, or MLA attention with a latent kv_cache and a
 *     RoPE-key pe_cache plus a routed MoE (TileRT 是什么 §五 5.2 and 5.3).
 *
 * Conventions for every function:
 *   - return 0 (DEC_OK) on success, a negative DEC_ERR_* code on failure;
 *     dec_last_error() then describes the failure.  The library never aborts,
 *     never traps and never prints.
 *   - a dec_ctx is used by one host thread at a time.
 *   - pointers marked "host or device" are classified with
 *     cudaPointerGetAttributes; the caller keeps ownership of every buffer it
 *     passes and may free it when the call returns.  Calls that read caller
 *     device buffers (dec_load_weights, dec_set_kv_cache) first synchronise
 *     the device, so data produced on any stream is complete when read.
 *   - all work is ordered on the context's stream (dec_set_stream); calls
 *     documented as synchronous return after their results are on the host.
 */
#ifndef DEC_H_
#define DEC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ----------------------------------------------------------------- codes */
#define DEC_OK 0
#define DEC_ERR_INVALID_ARG (-1) /* bad pointer, size, shape or enum value */
#define DEC_ERR_STATE (-2)       /* call out of order (e.g. step before weights or cache) */
#define DEC_ERR_CAPACITY (-3)    /* position would reach max_seq */
#define DEC_ERR_OOM (-4)         /* device allocation failed */
#define DEC_ERR_CUDA (-5)        /* a CUDA runtime call failed */
#define DEC_ERR_TIMEOUT (-6)     /* a device-side wait gave up; context poisoned until dec_reset */
#define DEC_ERR_UNSUPPORTED (-7) /* configuration outside what the kernels implement */
#define DEC_ERR_NUMERIC (-8)     /* a router or LM-head logit was NaN or infinite (corrupt weights or
                                    activations); context poisoned until dec_reset */

/* ------------------------------------------------------------------ enums */
#define DEC_ARCH_DENSE 0   /* RMSNorm, GQA attention with RoPE, SwiGLU FFN */
#define DEC_ARCH_MLA_MOE 1 /* RMSNorm, MLA attention, dense SwiGLU first layers, then routed MoE */

#define DEC_F32 0           /* fp32 weights; activations and cache in fp32 */
#define DEC_BF16 1          /* bf16 weights; bf16 activations and cache */
#define DEC_FP8_E4M3_B128 2 /* E4M3 weights, one fp32 scale per 128x128 block; bf16 activations and cache */

#define DEC_PERSISTENT 0   /* one persistent kernel per decode step (tile task list + dependency counters) */
#define DEC_PER_OP 1       /* same tiles, one kernel launch per op */
#define DEC_PER_OP_GRAPH 2 /* same tiles, one kernel per op, replayed from a CUDA graph */

#define DEC_FLAG_TRACE 1u /* record per-task timestamps (dec_debug_dump DEC_DUMP_TRACE) */
#define DEC_FLAG_TEST_STALL 2u /* failure-path test: the first task of the first op is never published, so
                                  the persistent kernel's dependency waits run out (DEC_ERR_TIMEOUT) */

/* Weight kinds for dec_tensor.kind.  Layouts are row-major [rows][cols]; FP8
 * matrices carry scales [ceil(rows/128)][ceil(cols/128)] fp32; norm gains are
 * always fp32 vectors; the embedding table uses the activation dtype
 * (fp32 for DEC_F32, bf16 otherwise). */
enum {
  DEC_W_EMBED = 1,      /* [vocab][d_model]                          global */
  DEC_W_FINAL_NORM = 2, /* [d_model] fp32                            global */
  DEC_W_LM_HEAD = 3,    /* [vocab][d_model]                          global */
  DEC_W_ATTN_NORM = 10, /* [d_model] fp32 */
  DEC_W_Q = 11,         /* dense: [n_heads*head_dim][d_model] */
  DEC_W_K = 12,         /* dense: [n_kv_heads*head_dim][d_model] */
  DEC_W_V = 13,         /* dense: [n_kv_heads*head_dim][d_model] */
  DEC_W_O = 14,         /* dense: [d_model][n_heads*head_dim]; MLA: [d_model][n_heads*v_head] */
  DEC_W_FFN_NORM = 15,  /* [d_model] fp32 */
  DEC_W_GATE = 16,      /* dense FFN: [ffn_hidden][d_model] */
  DEC_W_UP = 17,        /* dense FFN: [ffn_hidden][d_model] */
  DEC_W_DOWN = 18,      /* dense FFN: [d_model][ffn_hidden] */
  DEC_W_Q_A = 20,       /* MLA: [q_lora][d_model] */
  DEC_W_Q_A_NORM = 21,  /* MLA: [q_lora] fp32 */
  DEC_W_Q_B = 22,       /* MLA: [n_heads*(qk_nope+qk_rope)][q_lora], per head [nope | rope] */
  DEC_W_KV_A = 23,      /* MLA: [kv_lora+qk_rope][d_model], rows [latent | rope key] */
  DEC_W_KV_A_NORM = 24, /* MLA: [kv_lora] fp32 */
  DEC_W_KV_B = 25,      /* MLA: [n_heads*(qk_nope+v_head)][kv_lora], per head [W_UK rows | W_UV rows] */
  DEC_W_ROUTER = 30,    /* MoE: [n_experts][d_model] */
  DEC_W_EXP_GATE = 31,  /* MoE routed expert e: [expert_hidden][d_model] */
  DEC_W_EXP_UP = 32,    /* MoE routed expert e: [expert_hidden][d_model] */
  DEC_W_EXP_DOWN = 33,  /* MoE routed expert e: [d_model][expert_hidden] */
  DEC_W_SH_GATE = 34,   /* MoE shared experts: [n_shared*expert_hidden][d_model] */
  DEC_W_SH_UP = 35,     /* MoE shared experts: [n_shared*expert_hidden][d_model] */
  DEC_W_SH_DOWN = 36    /* MoE shared experts: [d_model][n_shared*expert_hidden] */
};

/* dec_debug_dump selectors */
#define DEC_DUMP_KV 1       /* dense: K then V, [n_layers][n_kv_heads][len][head_dim]; MLA: latent then pe */
#define DEC_DUMP_ROUTES 2   /* MoE: int32 [n_moe_layers][top_k] expert ids of the last step */
#define DEC_DUMP_TRACE 3    /* uint64 records {cta<<48|op<<32|task, t_start, t_input_ready, t_first_stage, t_done,
                               t_published} (ns, %globaltimer) of every task of the last step */
#define DEC_DUMP_TRACE_PRODUCER 6 /* uint64 triples {cta<<48|op<<32|task, t_reached, t_first_issued} per task-list
                                     position: when the weight-streaming warp reached each task and issued its
                                     first stage (ns; 0 for a task that streams nothing) */
#define DEC_DUMP_PLAN 4     /* text: one line per op (kind, tasks, geometry) */
#define DEC_DUMP_WEIGHTS 5  /* bytes of weights read per step (uint64 x2: weights+scales, stored incl. padding) */
#define DEC_DUMP_STATUS 7   /* 64 bytes: device status word {int32 code, cta, op, task (code 0 ok, 1 timeout,
                               2 non-finite logit); uint64 winning key of the last final op (logit bits in
                               order-preserving form << 32 | ~token); uint64 0}, then the step state
                               {int32 epoch, pos, tok, last, stop, 0, 0, 0} */
#define DEC_DUMP_OP 100     /* + op index (DEC_DUMP_PLAN order): fp32 outputs of that op in the last step;
                               GEMV ops: partial sums [splits][rows]; attention ops: max [heads][chunks],
                               sum [heads][chunks], weighted values [heads][chunks][dim], concatenated */

/* ------------------------------------------------------------------ types */
typedef struct dec_ctx dec_ctx; /* opaque; owns all of its device memory */

/* Limits checked by dec_create (DEC_ERR_UNSUPPORTED otherwise): dense head_dim 64 or 128,
 * n_heads / n_kv_heads <= 8, n_heads <= 128; MLA kv_lora 512, qk_rope 64 or 128, n_heads <= 128
 * (the attention's tensor-core tile is 128 heads), bf16 or FP8 weights. */
typedef struct dec_config {
  int32_t arch;                                          /* DEC_ARCH_* */
  int32_t n_layers, d_model, vocab, max_seq;             /* max_seq: context + generated positions */
  int32_t n_heads, n_kv_heads, head_dim, ffn_hidden;     /* dense attention; ffn_hidden also sizes MLA's dense layers */
  int32_t q_lora, kv_lora, qk_nope, qk_rope, v_head;     /* MLA (the pages' model: 512, 128, 64, 128) */
  int32_t n_dense_layers, n_experts, top_k, n_shared, expert_hidden; /* MoE */
  float rope_theta, norm_eps;
  int32_t weight_dtype;   /* DEC_F32 | DEC_BF16 | DEC_FP8_E4M3_B128 */
  int32_t exec_mode;      /* DEC_PERSISTENT | DEC_PER_OP | DEC_PER_OP_GRAPH */
  int32_t device;         /* CUDA device ordinal */
  uint32_t wait_timeout_us; /* bound on every device-side wait; 0 = 1,000,000 us */
  uint32_t flags;         /* DEC_FLAG_* */
  int32_t n_ctas;         /* persistent grid size; 0 = one CTA per SM */
} dec_config;

typedef struct dec_tensor {
  int32_t kind;       /* DEC_W_* */
  int32_t layer;      /* layer index, -1 for global tensors */
  int32_t expert;     /* routed expert index for DEC_W_EXP_*, else -1 */
  const void* data;   /* host or device; layout and dtype as documented for `kind` */
  const float* scales;/* FP8 only: host or device block scales, else NULL */
  size_t bytes;       /* size of `data` in bytes (checked against the shape) */
} dec_tensor;

/* ------------------------------------------------------------- lifecycle */

/* Validate the configuration, plan the task list of one decode step and
 * allocate all device memory (weights, caches, activations, counters).
 * Defined by: TileRT 是什么 §六 6.1 (the "prepare money" call that sets up each
 * GPU's parameters and buffers) and §六 6.2 (operator decomposition, execution
 * planning and memory layout done once, at compile time, not per step).
 * On an error *out may still hold a context that carries the message for
 * dec_last_error; pass it to dec_destroy, which frees what was allocated.
 * Errors: INVALID_ARG (bad config), UNSUPPORTED, OOM, CUDA. */
int dec_create(const dec_config* cfg, dec_ctx** out);

/* Copy n weight tensors into the context, re-laid out into its tile order
 * (host-to-device or device-to-device).  Defined by: TileRT 是什么 §六 6.2
 * (weight preprocessing belongs to compile time) and §五 5.3 (each GPU manages
 * its own parameters).  May be called repeatedly; a step
 * requires every tensor of the model to have been loaded once.
 * Errors: INVALID_ARG (unknown kind, bad layer/expert, size mismatch), CUDA. */
int dec_load_weights(dec_ctx* c, const dec_tensor* t, int n);

/* Install a prefilled context of n_tokens positions (the KV cache another
 * engine produced) and set the decode position to n_tokens.  Defined by: the
 * InferenceX article's PD-disaggregation section (prefill runs in another
 * engine, which moves its KV cache to the decode node) and TileRT 是什么 §五 5.3
 * (the kv_cache and pe_cache buffers of MLA).
 * Dense: k, v as [n_layers][n_kv_heads][n_tokens][head_dim].
 * MLA:   latent [n_layers][n_tokens][kv_lora] (the kv_cache) and
 *        pe [n_layers][n_tokens][qk_rope] (the pe_cache).
 * Elements are in the activation dtype (fp32 for DEC_F32, bf16 otherwise).
 * Host or device pointers.  n_tokens == 0 clears the context.
 * Errors: INVALID_ARG, CAPACITY (n_tokens >= max_seq), CUDA. */
int dec_set_kv_cache(dec_ctx* c, const void* k_or_latent, const void* v_or_pe, int32_t n_tokens);

/* One decode step, synchronous (TileRT 是什么 §六 6.1, the "show hands" inference
 * call; InferenceX article, "what TileRT is": the step as one persistent kernel
 * of overlapped tile tasks): embed token_id at the current position,
 * run every layer, write the fp32 logits [vocab] to out_logits (nullable;
 * host or device) and the greedy token (argmax, lowest id on ties) to
 * *out_next_token (host, nullable).  token_id < 0 feeds back the previous
 * step's greedy token from device memory.
 * Errors: STATE (weights or context missing, or poisoned), CAPACITY,
 * INVALID_ARG (token_id >= vocab), TIMEOUT, NUMERIC, CUDA. */
int dec_step(dec_ctx* c, int32_t token_id, float* out_logits, int32_t* out_next_token);

/* Enqueue one decode step on the context's stream and return at once.
 * token_id < 0 feeds back the previous step's greedy token on the device, so
 * steps chain without host round trips.  Logits stay in the context.
 * Errors as dec_step except TIMEOUT and NUMERIC, which dec_sync reports. */
int dec_step_async(dec_ctx* c, int32_t token_id);

/* Wait for enqueued steps; copy the last greedy token to *out_next_token
 * (nullable) and the last logits to out_logits (nullable, host or device).
 * Errors: TIMEOUT or NUMERIC (context poisoned), CUDA. */
int dec_sync(dec_ctx* c, float* out_logits, int32_t* out_next_token);

/* Generation: a whole decode lifetime with the host out of the loop (InferenceX
 * article, "what TileRT is": the host launches the engine kernel once and the
 * decode stays on the GPU).  token_id (< 0: the previous step's greedy token) is
 * embedded at the current position; each step's greedy token is fed back on the
 * device.  In DEC_PERSISTENT mode ONE kernel launch runs all steps and writes every
 * greedy token into a host-mapped ring as soon as it is known; in DEC_PER_OP and
 * DEC_PER_OP_GRAPH modes the same steps run one launch per step with a host check
 * after each (the ablation).  The generation ends after n_steps steps, after the
 * step whose greedy token equals stop_token (-1: none), or after the step during
 * which dec_generate_stop was called.  While it runs, every call that would queue
 * work or change the context returns DEC_ERR_STATE; dec_generate_poll and
 * dec_generate_stop may be called from the same host thread at any time.
 * Errors: STATE, CAPACITY (position + n_steps > max_seq), INVALID_ARG, CUDA. */
int dec_generate_async(dec_ctx* c, int32_t token_id, int32_t n_steps, int32_t stop_token);

/* Tokens of the running generation produced so far, without waiting: copies
 * min(count, cap) tokens into out_tokens (host), *out_count = count (nullable),
 * *out_done = 1 once the generation's launches have finished (nullable).
 * Errors: STATE (no generation), INVALID_ARG, CUDA. */
int dec_generate_poll(dec_ctx* c, int32_t* out_tokens, int32_t cap, int32_t* out_count, int32_t* out_done);

/* Ask the running generation to end after the step in progress (a host-mapped
 * flag the final op of every step reads).  Returns at once. */
int dec_generate_stop(dec_ctx* c);

/* Wait for the generation to finish; copy its tokens (at most cap) to out_tokens
 * (host) and their number to *out_count (nullable).  The position advances by the
 * steps completed.  Errors: TIMEOUT or NUMERIC (context poisoned), STATE, CUDA. */
int dec_generate_wait(dec_ctx* c, int32_t* out_tokens, int32_t cap, int32_t* out_count);

/* dec_generate_async then dec_generate_wait (out_tokens holds n_steps entries). */
int dec_generate(dec_ctx* c, int32_t token_id, int32_t n_steps, int32_t stop_token, int32_t* out_tokens,
                 int32_t* out_count);

/* Forget the context (position 0), clear a poisoned state, re-zero the
 * dependency counters.  Weights are kept.  Defined by: TileRT 是什么 §六 6.1 (the
 * reset call that starts a new sequence). */
int dec_reset(dec_ctx* c);

/* Free everything the context owns.  Accepts NULL.  Defined by: TileRT 是什么
 * §六 6.1 (the "go home" call that releases the resources). */
int dec_destroy(dec_ctx* c);

/* Use `stream` (a cudaStream_t, NULL = the legacy default stream) for all
 * further work of the context, after the work already queued on the current
 * one has finished.  The caller keeps ownership: the stream must stay valid
 * until the context is destroyed or given another stream, and dec_destroy
 * synchronises it but destroys only the stream that dec_create made. */
int dec_set_stream(dec_ctx* c, void* stream);

/* Switch between DEC_PERSISTENT, DEC_PER_OP and DEC_PER_OP_GRAPH for further
 * steps.  All three run the same tiles in the same order per tile, so their
 * outputs are bit-identical; only launch and synchronisation differ (the
 * ablation of the kernel-boundary cost the InferenceX article describes).
 * Errors: INVALID_ARG, CUDA (graph capture). */
int dec_set_exec_mode(dec_ctx* c, int32_t exec_mode);

/* Current decode position (number of cached positions). */
int dec_position(const dec_ctx* c, int32_t* out_pos);

/* Copy debug state (DEC_DUMP_*) into dst (host) of capacity `bytes`;
 * *out_bytes (nullable) receives the size needed.  For tests and tools. */
int dec_debug_dump(dec_ctx* c, int32_t what, void* dst, size_t bytes, size_t* out_bytes);

/* Text of the last error on this context (never NULL). */
const char* dec_last_error(const dec_ctx* c);

/* Split-KV decode attention for one query token that allocates no device
 * memory.  The pages have no counterpart of this call; it exists for callers
 * that cannot call cudaMalloc: code running while a CUDA graph is being
 * captured, runtimes whose device memory belongs to an outside allocator that
 * forbids allocation on the serving path, and embedders that must keep a fixed
 * memory footprint once started.
 *
 * Computes, for every query head h (GQA: kv head = h / (n_heads/n_kv_heads)),
 * out[h] = softmax_t(q[h] . K[g][t] / sqrt(head_dim)) V[g][t] over t < n_pos,
 * split into position chunks whose (max, sum, weighted values) are combined
 * with a log-sum-exp rescale -- the same split-KV attention the decode step
 * runs.
 *   q        device, fp32 [n_heads][head_dim] (already RoPE'd and rounded as wanted), 4-byte aligned
 *   k_cache  device, bf16 [n_kv_heads][cache_stride][head_dim], 16-byte aligned
 *   v_cache  device, bf16 [n_kv_heads][cache_stride][head_dim], 16-byte aligned
 *   out      device, fp32 [n_heads][head_dim], 4-byte aligned
 *   stream   cudaStream_t (NULL = legacy default stream); the call is asynchronous.
 * A pointer that breaks its alignment returns INVALID_ARG before anything runs.
 * Limits: head_dim 64 or 128, n_heads a multiple of n_kv_heads with at most 8
 * query heads per kv head, 1 <= n_pos <= cache_stride, and the per-chunk
 * partials n_heads * chunks * (head_dim + 2) floats must fit the library's
 * fixed 2 MiB scratch.  The call takes about 148 / n_kv_heads chunks per kv head
 * (1 to 64, at most n_pos), which stays far inside the scratch while n_kv_heads
 * <= 148; it returns DEC_ERR_CAPACITY when even one chunk per head does not fit
 * (n_heads * (head_dim + 2) > 524288).
 * The scratch is a fixed array inside the library, held by every GPU that
 * loads it until the process exits, and shared by all calls: nothing in it has
 * to start at zero (every call writes what it reads), but calls whose kernels
 * overlap on the GPU (for example on two streams) race on it.  The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture.  The address is kept for
 * the life of the process: after cudaDeviceReset (or any other teardown of the
 * device's primary context) this function must not be called again.
 * If a CUDA error from an earlier runtime call of this library is still
 * pending, the call returns CUDA without launching and leaves it pending.
 * Errors: INVALID_ARG, CAPACITY, CUDA.  No context, no dec_last_error. */
int dec_attention_noalloc(const float* q, const void* k_cache, const void* v_cache, int32_t n_heads,
                          int32_t n_kv_heads, int32_t head_dim, int32_t n_pos, int32_t cache_stride, float* out,
                          void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DEC_H_ */
