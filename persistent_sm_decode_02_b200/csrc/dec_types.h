// Plan structures shared by the host planner and the device engine.
//
// One decode step is a static list of ops in topological order; every op is
// cut into independent tile tasks.  The persistent kernel gives each CTA a
// fixed list of (op, task) pairs; a task of op k waits until the counters of
// k's dependencies reach epoch * ntasks, runs, and adds 1 to k's counter.  The
// tile-level task decomposition with overlapped weight streaming is the
// mechanism the pages describe for TileRT's engine ("Tile A1 + Tile B1 +
// comm C1", TileRT 是什么 §二 2.2; InferenceX article, "what TileRT is").
#pragma once
#include <stdint.h>

namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;  // threads that compute
constexpr int kThreads = kConsumers + 64;        // + one producer warp (streams weights) + one signaller warp
constexpr int kStageBytes = 32768;               // one ring stage
constexpr int kStages = 5;                       // ring depth (160 KB in flight per SM)
constexpr long long kL2Bytes = 126LL << 20;      // L2 of one GPU (both dies)
constexpr int kWorkBytes = 48 * 1024;            // per-task scratch (input vector / attention state)
constexpr int kCombineOff = 40 * 1024;           // split-KV combine weights inside the scratch (<= 2048 floats)
constexpr int kMaxCombine = (kWorkBytes - kCombineOff) / 4;
constexpr int kMaxSegs = 20;
constexpr int kMaxTopK = 16;
constexpr int kMaxD = 8192;                      // longest normalised vector (d_model, q_lora)
constexpr int kMlaHeads = 128;                   // MLA attention: heads are the MMA's M dimension (zero-padded)
constexpr int kMlaBlock = 64;                    // MLA attention: cache positions per block and per task

enum WType : int { WT_F32 = 0, WT_BF16 = 1, WT_FP8 = 2 };

// GEMV stage geometry, shared by the planner and the kernels: a stage holds
// R = G * RPT rows of KCB bytes; each of the 256 consumer threads owns one
// 16-byte column chunk (CPR = KCB / 16 chunks per row, G = 256 / CPR row
// groups) of RPT rows; at most 128 rows (a tile never straddles a 128-row FP8
// scale block) and at most one 32 KB stage.
#ifdef __CUDACC__
#define DEC_HD __host__ __device__
#else
#define DEC_HD
#endif
DEC_HD constexpr int gemv_rows_per_thread(int kcb) {
  const int G = 256 / (kcb / 16);
  int r = 8;
  if (128 / G < r) r = 128 / G;
  if (32768 / (G * kcb) < r) r = 32768 / (G * kcb);
  return r < 1 ? 1 : r;
}
// Tensor-core operand layouts of MLA attention (bf16, no swizzle).  A core
// matrix is 8 rows x 8 elements, each row 16 contiguous bytes, 128 bytes in
// all.  Latent cache of a layer: blocks of kMlaBlock positions; inside a block
// the core matrix (dims 8k..8k+7, positions 8i..8i+7) sits at k * 1024 + i * 128,
// so a block is [dim group][position group][8 positions][8 dims] and the
// (kv_lora + qk_rope) dims of a position are spread over the block.  Absorbed
// query: the core matrix (dims 8k.., heads 8i..) at k * 2048 + i * 128.
DEC_HD constexpr long long mla_cache_off(int p_in_block, int d) {  // bytes inside a block
  return (long long)(d >> 3) * 1024 + (p_in_block >> 3) * 128 + (p_in_block & 7) * 16 + (d & 7) * 2;
}
DEC_HD constexpr long long mla_q_off(int h, int d) {  // bytes
  return (long long)(d >> 3) * 2048 + (h >> 3) * 128 + (h & 7) * 16 + (d & 7) * 2;
}

enum OpKind : int { OP_GEMV = 0, OP_ATTN = 1, OP_MLA = 2, OP_FINAL = 3 };
enum Pro : int {
  PRO_NONE = 0,
  PRO_RESID_NORM = 1,   // h = base + partial sums (+ routed experts); x = R(rmsnorm(h) * g)
  PRO_NORM_SUM = 2,     // x = R(rmsnorm(sum of partials) * g)
  PRO_SUM = 3,          // x = R(sum of partials) (optionally per input group)
  PRO_SWIGLU = 4,       // x = R(silu(gate) * up)
  PRO_MLA_COMBINE = 6   // x = R(split-KV combine of one head's latent output)
};

// value(e) = sum_{s < S} ptr[s * stride + off + e]
struct PSet {
  const float* ptr;
  int S, stride, off;
};

struct Seg {
  const uint8_t* w;   // tiled weights (expert 0 for routed segments)
  const float* sc;    // fp8 block scales [ceil(N/128)][ceil(K/128)] (expert 0 for routed segments)
  long long w_estride;  // bytes between experts
  long long s_estride;  // floats between experts' scale tables
  int slot;           // routed slot j: weights of the router's j-th expert; -1: fixed weights
  int N;              // rows
  int ntiles;         // row tiles of R rows
  int task0;          // first task of this segment within the op
  int out_off;        // element offset of row 0 in every split's output
  int in_group;       // prologue input variant shared by all tasks of the segment (-1: by row group)
};

struct alignas(16) OpDesc {
  int kind, ntasks, layer;
  int dep[2];  // consumer dependencies (op index or -1)
  int pdep;    // producer dependency: router op whose top-k picks the weights of routed segments
  // ---- GEMV geometry: a task = R rows x (nst stages of kc columns)
  int wtype, K, Kpad, kcb, kc, cpr, G, rpt, R, S, nst;
  int nsegs;
  Seg seg[kMaxSegs];
  int rows_per_group;  // grouped GEMV: input group = row / rows_per_group (0: one input for all rows)
  int tpt;             // GEMV units (row tile x split) per task (0 or 1: one); a task's units share a group
  void* qc;            // MLA: absorbed bf16 query in the tensor-core layout (written by absorb_q, read by attention)
  float* out;          // fp32 partial outputs [S][out_stride]
  int out_stride;
  unsigned long long* best;  // LM head: best packed (value, index) key per task, else null
  // ---- prologue
  int pro;
  int in_bf16;  // input vector dtype: 1 = bf16 (rounded), 0 = fp32
  int n;        // input vector length (<= Kpad)
  int base_embed;  // RESID_NORM: 1 = base is the embedding row of the step token
  const void* embed;
  int embed_bf16;
  const float* h_base;
  PSet add, add2;          // summed with weight 1 (ptr null = unused)
  PSet routed;             // routed expert outputs, slot j at off + j * routed_slot_stride
  int routed_slot_stride;
  int n_experts, top_k;
  int router;              // 1: the router GEMV; its last task turns the logits into the top-k
  unsigned* fin;           // router: tasks finished (cumulative over steps), to find the last one
  int* rt_ids;             // router: top-k expert ids it writes; routed GEMV ops: ids their producer reads
  float* rt_w;             // router: renormalised top-k weights it writes; RESID_NORM: weights it reads
  int* route_dump;         // router: the chosen expert ids are also stored here (debug dump)
  const float* gain;
  float eps;
  float* h_out;            // RESID_NORM: the op's task 0 stores h here
  PSet src;                // NORM_SUM / SUM
  int gstride;             // SUM: input offset per group
  PSet gate, up;           // SWIGLU; slot j reads off + j * slot_stride
  int slot_stride;
  const float* am;         // COMBINE: attention partials (max, sum, weighted values)
  const float* al;
  const float* ao;
  int nch, nheads, hdim;
  // ---- attention
  PSet qkv;       // dense: q|k|v projections; MLA: q_b output (q_pe is read from it)
  PSet qlat;      // MLA: absorbed query [H * kv_lora]
  PSet ckv;       // MLA: kv_a output (latent then RoPE key)
  const float* kvnorm_g;
  int hq, hkv, hd, gs;
  int H, kvl, rdim, nope;
  void* kcache;   // dense: K of this layer [hkv][max_seq][hd]; MLA: blocked latent cache (mla_cache_off)
  void* vcache;   // dense: V of this layer
  int cache_bf16;
  int max_seq;
  const float* rope_cos;  // [max_seq][rope_dim / 2]
  const float* rope_sin;
  int rope_dim;
  float attn_scale;
  float* m_out;
  float* l_out;
  float* o_out;
  float* o_fin;  // dense: combined attention output [hq][hd] (the last chunk task of a kv head writes it;
                 // `fin` then holds one finished-task counter per kv head)
  int np;  // positions per ring stage
  int osplit;  // MLA: tasks per cache block (1, 2 or 4: each computes S and that share of O's columns)
  // ---- final op
  const unsigned long long* fin_best;
  int fin_n;
  int vocab;
  float* logits;  // LM head output (the final op reads nothing from it; kept for dumps)
};

struct StepState {
  int epoch;  // 1-based step counter since the last reset (dependency counter targets)
  int pos;    // position of the token of the current step
  int tok;    // token of the current step (written by the host or by the previous step)
  int last;   // greedy token of the last completed step
  int stop;   // a multi-step launch ends after the step that set it (stop token or host request)
  int pad[3];
};

// A generation (dec_generate*): the final op of every step puts the greedy token into a
// host-mapped ring and may end the launch (stop token, host request).
struct GenState {
  int active;      // a generation is running
  int epoch0;      // epoch of its first step (ring index = epoch - epoch0)
  int stop_token;  // -1: none
  int pad;
};

struct Status {
  int code;  // 0 ok, 1 a bounded wait timed out, 2 a non-finite router or LM-head logit
  int cta, op, task;
  unsigned long long final_key;  // the last final op's winning (order-preserving logit bits, ~index) key
  unsigned long long pad;
};

struct KParams {
  const OpDesc* ops;
  int nops;
  const int2* tasks;     // (op, task) pairs of all CTAs
  const int* task_off;   // CTA b runs tasks[task_off[b] .. task_off[b + 1])
  unsigned* counters;    // one per op, cumulative over steps
  StepState* state;
  unsigned* started;     // CTAs that have read the step state (cumulative)
  Status* status;
  unsigned long long timeout_ns;
  int persistent;        // 1: one launch runs every op; 0: this launch runs op `op_only`
  int op_only;
  int n_ctas;
  unsigned long long* trace;  // optional per-task timestamps
  int trace_cap;
  int tok_in;                 // >= 0: token of this step given by the host; < 0: the state's token
  int test_stall;             // failure-path test: never publish task 0 of op 0
  int kv_evict_first;         // 1: cache reads take the L2 evict-first policy (the caches a step reads exceed
                              // what L2 could keep for the next step), 0: evict-last (they are re-read from L2)
  // ---- generation: a whole decode lifetime in one launch (persistent mode, n_steps > 1)
  int n_steps;                // steps this launch runs (1: one step)
  const GenState* gen;        // device: the running generation, if any
  int* tok_ring;              // host-mapped [max_seq]: greedy token of each generated step
  unsigned* tok_count;        // host-mapped: tokens written so far (after the ring entry)
  const int* stop_word;       // host-mapped: non-zero asks the generation to stop after the current step
};

}  // namespace dec
