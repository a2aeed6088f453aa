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
#include <stddef.h>
#include <stdint.h>

namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;  // threads that compute
constexpr int kThreads = kConsumers + 64;        // + one producer warp (streams weights) + one signaller warp
constexpr int kStageBytes = 32768;               // one ring stage
constexpr int kStages = 5;                       // ring depth (160 KB in flight per SM)
constexpr int kWorkBytes = 48 * 1024;            // per-task scratch (input vector / attention state)
constexpr int kCombineOff = 40 * 1024;           // split-KV combine weights inside the scratch (<= 2048 floats)
constexpr int kMaxCombine = (kWorkBytes - kCombineOff) / 4;
constexpr int kMaxSegs = 20;
constexpr int kMaxTopK = 16;
constexpr int kMaxD = 8192;                      // longest normalised vector (d_model, q_lora)
constexpr int kMlaHeads = 128;                   // MLA attention: heads are the MMA's M dimension (zero-padded)
constexpr int kMlaBlock = 64;                    // MLA attention: cache positions per block and per task
constexpr int kPieceStages = 8;                  // GEMV: longest task, in ring stages (longer row tiles are cut along K)

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
  PRO_RESID_NORM = 1,   // h = base + the previous block's output; x = R(rmsnorm(h) * g)
  PRO_NORM_SUM = 2,     // x = R(rmsnorm(sum of partials) * g)
  PRO_SUM = 3,          // x = R(sum of partials) (optionally per input group)
  PRO_SWIGLU = 4,       // x = R(silu(gate) * up)
  PRO_MLA_COMBINE = 6   // x = R(split-KV combine of one head's latent output)
};

// Fixed-point accumulators.  Every vector one op hands to another (GEMV outputs,
// the dense attention's combined output) is held as 64-bit integers in units of
// 2^-40.  A GEMV whose row tiles are split along K among tasks (and the experts,
// whose slots all add into one vector) sums its pieces with integer atomics:
// integer addition is exact and associative, so the sum does not depend on the
// order in which CTAs finish and the step stays bit-reproducible; a vector written
// by one task per row is stored plainly.  Readers have one path (two 16-byte loads
// per four values).  Range +-2^22 (a larger or non-finite value is reported as a
// numeric error); resolution 2^-40.  Every accumulator has two copies used by
// alternate steps (parity = epoch & 1): a step adds into its own copy and clears
// the other one, which the previous step finished with.
constexpr float kAccScale = 1099511627776.0f;  // 2^40
constexpr float kAccInv = 1.0f / 1099511627776.0f;
constexpr float kAccMax = 4194304.0f;          // 2^22

// value(e) = acc[par * stride + off + e] * 2^-40 for the step's parity par (acc null: unused)
struct PSet {
  const long long* acc;
  int stride, off;
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
  int out_off;        // element offset of row 0 in the op's output
  int in_group;       // prologue input variant shared by all tasks of the segment (-1: by row group)
  int zero_acc;       // accumulator ops: this segment's pieces that start at stage 0 clear the other parity
};

// Tasks are handed out at run time: when a CTA's producer warp reaches an op it takes
// the op's tasks one at a time from a global cursor (an atomic add) until none is
// left, streams each task's bytes and passes the task to its consumers through a
// shared-memory queue.  An SM that streams faster takes more tasks, so an op ends
// when the last task ends, not when the slowest SM's fixed share does.  An op whose
// tasks read different input vectors (the routed experts' down projections: one
// SwiGLU input per slot) has one cursor per input group; a CTA starts at the group
// its index maps to and moves on to the next group when one runs dry, so most CTAs
// build one input vector.  Cursors come in two copies used by alternate steps; the
// final op clears the copy of the next step.
struct alignas(16) OpDesc {
  // head (first 32 bytes, read alone by the task hand-out)
  int kind, ntasks, layer;
  int ngroups, cur_off, trace_base;  // task groups, their first cursor, first trace record
  const int* gbegin;                 // first task of each group [ngroups + 1] (null: one group of all tasks)
  int dep[2];  // consumer dependencies (op index or -1)
  int pdep;    // producer dependency: router op whose top-k picks the weights of routed segments
  // ---- GEMV geometry: a unit = R rows x nst consecutive stages of kc columns (a piece of one
  // row tile); weights are stored [row tile][nst_total stages][R rows][kcb bytes]
  int wtype, K, Kpad, kcb, kc, cpr, G, rpt, R, nst_total;
  int nsegs;
  Seg seg[kMaxSegs];
  const int4* pieces;  // per unit: x = segment, y = row tile, z = first stage, w = stages
  int rows_per_group;  // grouped GEMV: input group = row / rows_per_group (0: one input for all rows)
  int tpt;             // GEMV units per task (0 or 1: one); a task's units share an input group
  void* qc;            // MLA: absorbed bf16 query in the tensor-core layout (written by absorb_q, read by attention)
  float* out;          // fp32 outputs [out_stride] (the LM head's logits), or null when acc is set
  long long* acc;      // fixed-point output [2][out_stride]: stored (one task per row) or added (acc_add)
  int acc_add;         // the op's tasks split rows along K or add segments into the same rows
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
  PSet add;                // added to the base (ptr and acc null = unused); the FFN outputs of an MoE
                           // layer (routed experts weighted, shared expert) arrive as one accumulator
  int n_experts, top_k;
  int router;              // 1: the router GEMV; its last task turns the logits into the top-k
  unsigned* fin;           // router: tasks finished (cumulative over steps), to find the last one
  int* rt_ids;             // router: top-k expert ids it writes; routed GEMV ops: ids their producer reads
  float* rt_w;             // router: renormalised top-k weights it writes; RESID_NORM: weights it reads;
                           // routed GEMV with an accumulator: slot weights applied before the add
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
  long long* o_fin;  // dense: combined attention output [2][hq][hd], fixed point (the last chunk task of a
                    // kv head writes it; `fin` then holds one finished-task counter per kv head)
  int np;  // positions per ring stage
  // ---- final op
  const unsigned long long* fin_best;
  int fin_n;
  int vocab;
  float* logits;  // LM head output (the final op reads nothing from it; kept for dumps)
};
static_assert(offsetof(OpDesc, gbegin) == 24, "the task hand-out reads the descriptor head as int4 + pointer");

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
};

struct KParams {
  const OpDesc* ops;
  int nops;
  unsigned* cursors;     // task cursors [2][ncur] (copy epoch & 1 is this step's)
  int ncur;
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
  // ---- generation: a whole decode lifetime in one launch (persistent mode, n_steps > 1)
  int n_steps;                // steps this launch runs (1: one step)
  const GenState* gen;        // device: the running generation, if any
  int* tok_ring;              // host-mapped [max_seq]: greedy token of each generated step
  unsigned* tok_count;        // host-mapped: tokens written so far (after the ring entry)
  const int* stop_word;       // host-mapped: non-zero asks the generation to stop after the current step
};

}  // namespace dec
