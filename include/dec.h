/*
 * dec.h -- C ABI of a batch-1 transformer decode step run as one persistent
 * CUDA kernel per step on an NVIDIA B200 (sm_100a).
 *
 * The problem statement follows the pages on TileRT (SemiAnalysis, "Ultra-High
 * Interactivity on NVIDIA GPUs? -- TileRT InferenceX", and "TileRT 是什么"):
 *   - decode only, batch 1: prefill runs in another engine, which hands over
 *     its KV cache (InferenceX article, PD disaggregation section);
 *   - a lifecycle of init / step / reset / cleanup (TileRT 是什么 §六 6.1: the
 *     prepare_money / show_hands / reset / go_home entry points);
 *   - the whole decode step as one persistent kernel whose tile tasks overlap
 *     weight streaming with compute (InferenceX article, "what TileRT is";
 *     TileRT 是什么 §二 2.2, tile-level runtime engine);
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
#define DEC_DUMP_TRACE 3    /* uint64 records {cta<<48|op<<32|task, t_start, t_first_stage, t_done, t_published}
                               (ns, %globaltimer) of every task of the last step */
#define DEC_DUMP_TRACE_PRODUCER 6 /* uint64 pairs {cta<<48|op<<32|task, t_reached} per task-list position: when the
                                     weight-streaming warp reached each task (ns) */
#define DEC_DUMP_PLAN 4     /* text: one line per op (kind, tasks, geometry) */
#define DEC_DUMP_WEIGHTS 5  /* bytes of weights read per step (uint64 x2: weights+scales, stored incl. padding) */
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
 * On an error *out may still hold a context that carries the message for
 * dec_last_error; pass it to dec_destroy, which frees what was allocated.
 * Errors: INVALID_ARG (bad config), UNSUPPORTED, OOM, CUDA. */
int dec_create(const dec_config* cfg, dec_ctx** out);

/* Copy n weight tensors into the context, re-laid out into its tile order
 * (host-to-device or device-to-device).  May be called repeatedly; a step
 * requires every tensor of the model to have been loaded once.
 * Errors: INVALID_ARG (unknown kind, bad layer/expert, size mismatch), CUDA. */
int dec_load_weights(dec_ctx* c, const dec_tensor* t, int n);

/* Install a prefilled context of n_tokens positions (the KV cache another
 * engine produced) and set the decode position to n_tokens.
 * Dense: k, v as [n_layers][n_kv_heads][n_tokens][head_dim].
 * MLA:   latent [n_layers][n_tokens][kv_lora] (the kv_cache) and
 *        pe [n_layers][n_tokens][qk_rope] (the pe_cache).
 * Elements are in the activation dtype (fp32 for DEC_F32, bf16 otherwise).
 * Host or device pointers.  n_tokens == 0 clears the context.
 * Errors: INVALID_ARG, CAPACITY (n_tokens >= max_seq), CUDA. */
int dec_set_kv_cache(dec_ctx* c, const void* k_or_latent, const void* v_or_pe, int32_t n_tokens);

/* One decode step, synchronous: embed token_id at the current position,
 * run every layer, write the fp32 logits [vocab] to out_logits (nullable;
 * host or device) and the greedy token (argmax, lowest id on ties) to
 * *out_next_token (host, nullable).  token_id < 0 feeds back the previous
 * step's greedy token from device memory.
 * Errors: STATE (weights or context missing, or poisoned), CAPACITY,
 * INVALID_ARG (token_id >= vocab), TIMEOUT, CUDA. */
int dec_step(dec_ctx* c, int32_t token_id, float* out_logits, int32_t* out_next_token);

/* Enqueue one decode step on the context's stream and return at once.
 * token_id < 0 feeds back the previous step's greedy token on the device, so
 * steps chain without host round trips.  Logits stay in the context.
 * Errors as dec_step except TIMEOUT, which dec_sync reports. */
int dec_step_async(dec_ctx* c, int32_t token_id);

/* Wait for enqueued steps; copy the last greedy token to *out_next_token
 * (nullable) and the last logits to out_logits (nullable, host or device).
 * Errors: TIMEOUT (context poisoned), CUDA. */
int dec_sync(dec_ctx* c, float* out_logits, int32_t* out_next_token);

/* Forget the context (position 0), clear a poisoned state, re-zero the
 * dependency counters.  Weights are kept. */
int dec_reset(dec_ctx* c);

/* Free everything the context owns.  Accepts NULL. */
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
 *   q        device, fp32 [n_heads][head_dim] (already RoPE'd and rounded as wanted)
 *   k_cache  device, bf16 [n_kv_heads][cache_stride][head_dim]
 *   v_cache  device, bf16 [n_kv_heads][cache_stride][head_dim]
 *   out      device, fp32 [n_heads][head_dim]
 *   stream   cudaStream_t (NULL = legacy default stream); the call is asynchronous.
 * Limits: head_dim 64 or 128, n_heads a multiple of n_kv_heads with at most 8
 * query heads per kv head, 1 <= n_pos <= cache_stride, and the per-chunk
 * partials n_heads * chunks * (head_dim + 2) floats must fit the library's
 * fixed 2 MiB scratch (the call uses fewer chunks when needed and returns
 * DEC_ERR_CAPACITY if even one chunk per head does not fit).
 * The scratch is a fixed array inside the library, held by every GPU that
 * loads it until the process exits, and shared by all calls: nothing in it has
 * to start at zero (every call writes what it reads), but calls whose kernels
 * overlap on the GPU (for example on two streams) race on it.  The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture.
 * Errors: INVALID_ARG, CAPACITY, CUDA.  No context, no dec_last_error. */
int dec_attention_noalloc(const float* q, const void* k_cache, const void* v_cache, int32_t n_heads,
                          int32_t n_kv_heads, int32_t head_dim, int32_t n_pos, int32_t cache_stride, float* out,
                          void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DEC_H_ */
