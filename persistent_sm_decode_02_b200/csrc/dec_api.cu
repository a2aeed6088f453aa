// C ABI of the decode library: planning, memory, weight re-layout, cache
// install and the three execution modes (persistent kernel, one kernel per op,
// CUDA graph of the per-op kernels).  See include/dec.h for the contract.
//
// Planning happens once, at dec_create ("compile time" in the pages' terms:
// TileRT 是什么 §六 6.2 moves operator decomposition, execution planning, weight
// preprocessing and memory layout to compile time and leaves a minimal runtime
// scheduler).  Here that means: every op of the step gets a tile geometry and
// split factor, weights are stored in the tile order the ring streams them, and
// every CTA gets a fixed task list.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/dec.h"
#include "dec_types.h"
#include "engine.cuh"

using namespace dec;

namespace {

// ------------------------------------------------------------ matrices
// A weight matrix stored in tile order: [row tile][split][stage][R][kcb bytes].
struct Mat {
  int N = 0, K = 0, wb = 1, wtype = WT_F32;
  int R = 0, S = 1, nst = 1, kcb = 0, Kpad = 0, ntiles = 0;
  int n_experts = 1;
  int mode = 0;  // source layout: 0 row-major [N][K]; 1 W_UK^T of kv_b; 2 W_UV of kv_b
  size_t tile_bytes = 0;  // bytes of one expert
  size_t sc_count = 0;    // scale floats of one expert
  uint8_t* w = nullptr;
  float* sc = nullptr;
  int loaded = 0;  // experts loaded
};

struct Vec {
  float* p = nullptr;
  int n = 0;
  bool loaded = false;
};

struct Geo {
  int kcb, Kpad, cpr, G, rpt, R, nst_total;
};

Geo gemv_geometry(int K, int wb) {
  Geo g;
  const long long Kb = (long long)K * wb;
  int best = -1;
  long long best_waste = 1LL << 62;
  // Prefer 512-byte row chunks: 32 lanes cover a row, so every row reduces
  // inside one warp and tasks need no CTA-wide barrier; wider chunks only when
  // 512 would pad K too much.
  for (int kcb = 512; kcb >= 32; kcb >>= 1) {
    const long long pad = (Kb + kcb - 1) / kcb * kcb;
    const long long waste = pad - Kb;
    if (waste * 16 <= Kb) {
      best = kcb;
      break;
    }
    if (waste < best_waste) {
      best_waste = waste;
      best = kcb;
    }
  }
  g.kcb = best;
  const long long padb = (Kb + best - 1) / best * best;
  g.Kpad = (int)(padb / wb);
  g.nst_total = (int)(padb / best);
  g.cpr = best / 16;
  g.G = kConsumers / g.cpr;
  g.rpt = gemv_rows_per_thread(best);
  g.R = g.G * g.rpt;
  return g;
}

// Split-K factor S of a GEMV op, in units of ring stages on the busiest CTA: its tasks'
// stages plus a fixed cost per task, plus the consumer's prologue, which reads all S
// partial vectors (out_rows fp32 values each) on every CTA.  Every CTA reads the same lines
// at once, and that L2 read ran about 4x slower per byte than a weight stage in the device
// trace, hence the weight.
constexpr double kPrologueWeight = 4.0;
int choose_split(int ntiles, int nst_total, int n_ctas, long long out_rows, bool force_one) {
  if (force_one) return 1;
  int best = 1;
  double best_cost = 1e30;
  for (int S = 1; S <= 16 && S <= nst_total; ++S) {
    if (nst_total % S) continue;
    const long long tasks = (long long)ntiles * S;
    const long long per = (tasks + n_ctas - 1) / n_ctas;
    const double cost = per * (nst_total / (double)S + 0.75) + kPrologueWeight * S * out_rows * 4.0 / kStageBytes;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

__global__ void relayout16(const uint8_t* src, long long N, long long K, int wb, int R, int S, int nst, int kcb,
                           long long total16, uint8_t* dst) {
  // dst byte q = ((((rt*S + s)*nst + st)*R + r)*kcb + jb); one thread per 16 bytes
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total16;
       i += (long long)gridDim.x * blockDim.x) {
    const long long q = i * 16;
    const long long jb = q % kcb;
    long long rest = q / kcb;
    const long long r = rest % R;
    rest /= R;
    const long long st = rest % nst;
    rest /= nst;
    const long long s = rest % S;
    const long long rt = rest / S;
    const long long n = rt * R + r;
    const long long kb = (s * nst + st) * kcb + jb;  // byte offset in the padded row
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < N && kb < K * wb) v = *reinterpret_cast<const uint4*>(src + n * K * wb + kb);
    *reinterpret_cast<uint4*>(dst + q) = v;
  }
}

// Element-wise re-layout for the two views of kv_b (mode 1: W_UK^T, mode 2: W_UV).
__global__ void relayout_kvb(const uint8_t* src, int mode, long long N, long long K, int wb, int R, int S, int nst,
                             int kcb, long long total, int nope, int vdim, int kvl, uint8_t* dst) {
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < total;
       q += (long long)gridDim.x * blockDim.x) {
    const long long jb = q % kcb;
    long long rest = q / kcb;
    const long long r = rest % R;
    rest /= R;
    const long long st = rest % nst;
    rest /= nst;
    const long long s = rest % S;
    const long long rt = rest / S;
    const long long n = rt * R + r;
    const long long kb = (s * nst + st) * kcb + jb;
    const long long k = kb / wb, byte = kb % wb;
    uint8_t v = 0;
    if (n < N && k < K) {
      long long si;
      if (mode == 1) {  // W_UK^T: n = h*kvl + c, k = j (nope index): kv_b[(h*(nope+vdim) + j)][c]
        const long long h = n / kvl, cc = n % kvl;
        si = (h * (nope + vdim) + k) * kvl + cc;
      } else {  // W_UV: n = h*vdim + v, k = c: kv_b[(h*(nope+vdim) + nope + v)][c]
        const long long h = n / vdim, vv = n % vdim;
        si = (h * (nope + vdim) + nope + vv) * kvl + k;
      }
      v = src[si * wb + byte];
    }
    dst[q] = v;
  }
}

__global__ void set_int(int* p, int v) { *p = v; }

// Row-major latent rows [n][rowe] (bf16) <-> the blocked tensor-core cache layout
// (mla_cache_off); one thread per 16-byte chunk.
__global__ void mla_cache_convert(uint8_t* rows, uint8_t* blocked, int n, int rowe, int to_blocked) {
  const long long nck = rowe / 8, total = (long long)n * nck;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int p = (int)(i / nck), k = (int)(i % nck);
    uint4* r = reinterpret_cast<uint4*>(rows + (size_t)p * rowe * 2 + (size_t)k * 16);
    uint4* b = reinterpret_cast<uint4*>(blocked + (size_t)(p / kMlaBlock) * rowe * kMlaBlock * 2 +
                                        mla_cache_off(p % kMlaBlock, 8 * k));
    if (to_blocked)
      *b = *r;
    else
      *r = *b;
  }
}

// One engine instance per (weight type, attention kind): each compiles only its own paths.
const void* pick_kernel(int wtype, bool mla) {
  if (mla) return wtype == WT_FP8 ? (const void*)engine_kernel<WT_FP8, true> : (const void*)engine_kernel<WT_BF16, true>;
  if (wtype == WT_FP8) return (const void*)engine_kernel<WT_FP8, false>;
  if (wtype == WT_BF16) return (const void*)engine_kernel<WT_BF16, false>;
  return (const void*)engine_kernel<WT_F32, false>;
}

}  // namespace

// ====================================================================== ctx
struct dec_ctx {
  dec_config cfg{};
  int n_ctas = 0;
  cudaStream_t stream = nullptr;      // where the context's work is ordered
  cudaStream_t own_stream = nullptr;  // the stream dec_create made; the only one dec_destroy destroys
  std::string err = "";
  int wtype = WT_F32, wb = 4, act_bf16 = 0, eb = 4;
  // plan
  std::vector<OpDesc> ops;
  std::vector<std::string> op_names;
  OpDesc* d_ops = nullptr;
  int2* d_tasks = nullptr;
  int* d_task_off = nullptr;
  std::vector<int> task_off;
  int lm_op = -1, final_op = -1;
  // memory
  std::vector<void*> allocs;
  size_t bytes_alloc = 0;
  unsigned* d_counters = nullptr;
  size_t n_counters = 0;
  StepState* d_state = nullptr;
  unsigned* d_started = nullptr;
  Status* d_status = nullptr;
  unsigned long long* d_trace = nullptr;
  int trace_cap = 0;
  int* d_route_dump = nullptr;
  int n_moe = 0;
  // weights
  std::map<std::tuple<int, int>, Mat> mats;  // (kind, layer)
  std::map<std::tuple<int, int>, Vec> vecs;
  void* embed = nullptr;
  bool embed_loaded = false;
  // caches, per layer
  std::vector<void*> kc, vc;
  float* rope_cos = nullptr;
  float* rope_sin = nullptr;
  float* logits = nullptr;
  // state
  int pos = 0;
  int epoch = 1;
  bool have_ctx = false;
  bool poisoned = false;
  int pending = 0;
  cudaGraphExec_t graph = nullptr;
  int mode = DEC_PERSISTENT;
  std::vector<std::vector<void*>> seg_mats;  // per op: the Mat behind every segment
  uint8_t* staging = nullptr;
  size_t staging_bytes = 0;
  void* kvb_src = nullptr;
  const void* kernel = nullptr;  // engine instance for this model's weight type and attention kind
  size_t weight_bytes_step = 0, weight_bytes_stored = 0;
  // generation (dec_generate*): host-mapped token ring, count and stop word
  GenState* d_gen = nullptr;
  uint8_t* h_map = nullptr;  // [count u32 | stop i32 | pad | ring i32[max_seq]]
  uint8_t* d_map = nullptr;
  bool generating = false;
  int gen_epoch0 = 0, gen_steps = 0, gen_stop_token = -1;
  cudaEvent_t gen_done = nullptr;
};

static volatile unsigned* h_count(dec_ctx* c) { return reinterpret_cast<volatile unsigned*>(c->h_map); }
static volatile int* h_stop(dec_ctx* c) { return reinterpret_cast<volatile int*>(c->h_map + 4); }
static volatile int* h_ring(dec_ctx* c) { return reinterpret_cast<volatile int*>(c->h_map + 16); }

static int fail(dec_ctx* c, int code, const char* fmt, ...) __attribute__((format(printf, 3, 4)));
static int fail(dec_ctx* c, int code, const char* fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    c->err = buf;
  }
  return code;
}

#define CK(call)                                                                         \
  do {                                                                                   \
    cudaError_t e_ = (call);                                                             \
    if (e_ != cudaSuccess) return fail(c, DEC_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

template <class T>
static int dalloc(dec_ctx* c, T** p, size_t bytes) {
  void* q = nullptr;
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(c, DEC_ERR_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  c->allocs.push_back(q);
  c->bytes_alloc += bytes;
  *p = reinterpret_cast<T*>(q);
  return DEC_OK;
}

// ------------------------------------------------------------ planning
namespace {

struct SegSpec {
  Mat* mat;
  int slot;      // routed slot or -1
  int in_group;  // prologue input variant or -1
};

struct Planner {
  dec_ctx* c;
  int rc = DEC_OK;

  OpDesc base_op(int kind, int layer) {
    OpDesc o;
    memset(&o, 0, sizeof o);
    o.kind = kind;
    o.layer = layer;
    o.dep[0] = o.dep[1] = -1;
    o.pdep = -1;
    o.in_bf16 = c->act_bf16;
    o.eps = c->cfg.norm_eps;
    return o;
  }

  Mat* new_mat(int kind, int layer, int N, int K, int n_experts, int mode) {
    Mat& m = c->mats[{kind, layer}];
    m.N = N;
    m.K = K;
    m.wb = c->wb;
    m.wtype = c->wtype;
    m.n_experts = n_experts;
    m.mode = mode;
    return &m;
  }

  // Create a GEMV op over segments sharing K; returns op index.
  // whole_reader: every CTA running the consumer reads the whole output (a GEMV prologue);
  // false when each consumer task reads only its own slice (attention reading q/k/v).
  int gemv(const std::vector<SegSpec>& segs, int K, int layer, bool force_s1, const char* name,
           bool whole_reader = true) {
    OpDesc o = base_op(OP_GEMV, layer);
    const Geo g = gemv_geometry(K, c->wb);
    int ntiles = 0;
    for (auto& s : segs) ntiles += (s.mat->N + g.R - 1) / g.R;
    long long out_rows = 0;
    if (whole_reader)
      for (auto& sp : segs) out_rows += sp.mat->N;
    const int S = choose_split(ntiles, g.nst_total, c->n_ctas, out_rows, force_s1);
    o.wtype = c->wtype;
    o.K = K;
    o.Kpad = g.Kpad;
    o.kcb = g.kcb;
    o.kc = g.kcb / c->wb;
    o.cpr = g.cpr;
    o.G = g.G;
    o.rpt = g.rpt;
    o.R = g.R;
    o.S = S;
    o.nst = g.nst_total / S;
    o.n = K;
    o.nsegs = (int)segs.size();
    if (o.nsegs > kMaxSegs) {
      rc = fail(c, DEC_ERR_UNSUPPORTED, "too many segments in %s", name);
      return -1;
    }
    int task = 0, out = 0;
    for (int i = 0; i < o.nsegs; ++i) {
      Mat* m = segs[i].mat;
      m->R = g.R;
      m->S = S;
      m->nst = o.nst;
      m->kcb = g.kcb;
      m->Kpad = g.Kpad;
      m->ntiles = (m->N + g.R - 1) / g.R;
      m->tile_bytes = (size_t)m->ntiles * S * o.nst * g.R * g.kcb;
      m->sc_count = c->wtype == WT_FP8 ? (size_t)((m->N + 127) / 128) * ((m->K + 127) / 128) : 0;
      Seg& sg = o.seg[i];
      sg.slot = segs[i].slot;
      sg.in_group = segs[i].in_group;
      sg.N = m->N;
      sg.ntiles = m->ntiles;
      sg.task0 = task;
      sg.out_off = out;
      sg.w_estride = (long long)m->tile_bytes;
      sg.s_estride = (long long)m->sc_count;
      task += m->ntiles * S;
      out += m->N;
    }
    o.ntasks = task;
    o.out_stride = out;
    int arc = dalloc(c, &o.out, (size_t)o.S * o.out_stride * 4);
    if (arc) {
      rc = arc;
      return -1;
    }
    c->ops.push_back(o);
    c->op_names.push_back(name);
    std::vector<void*> sm;
    for (auto& sp : segs) sm.push_back(sp.mat);
    c->seg_mats.push_back(sm);
    return (int)c->ops.size() - 1;
  }

  int push(const OpDesc& o, const char* name) {
    c->ops.push_back(o);
    c->op_names.push_back(name);
    c->seg_mats.push_back({});
    return (int)c->ops.size() - 1;
  }
};

}  // namespace

static int alloc_mats(dec_ctx* c) {
  for (auto& kv : c->mats) {
    Mat& m = kv.second;
    int rc = dalloc(c, &m.w, m.tile_bytes * m.n_experts);
    if (rc) return rc;
    CK(cudaMemsetAsync(m.w, 0, m.tile_bytes * m.n_experts, c->stream));
    if (m.sc_count) {
      rc = dalloc(c, &m.sc, m.sc_count * m.n_experts * sizeof(float));
      if (rc) return rc;
    }
    c->weight_bytes_stored += m.tile_bytes * m.n_experts;
  }
  return DEC_OK;
}

static size_t mla_cache_bytes(const dec_config& f) {
  return (size_t)((f.max_seq + kMlaBlock - 1) / kMlaBlock) * kMlaBlock * (f.kv_lora + f.qk_rope) * 2;
}

// Grouped GEMVs whose row tiles are tiny (absorb_q: 16 KB, uv: 32 KB per tile) run a whole
// input group (one head) per task: the prologue and the task overhead are paid once per head.
static void group_tasks(OpDesc& o) {
  if (o.kind != OP_GEMV || o.S != 1 || o.rows_per_group <= 0 || o.rows_per_group % o.R) return;
  const int tpt = o.rows_per_group / o.R;
  if (tpt <= 1 || o.ntasks % tpt) return;
  for (int i = 0; i < o.nsegs; ++i)
    if (o.seg[i].ntiles % tpt || o.seg[i].task0 % tpt) return;
  o.tpt = tpt;
  o.ntasks /= tpt;
}

static float* gainp(dec_ctx* c, int kind, int layer) { return c->vecs[{kind, layer}].p; }

static int build_plan(dec_ctx* c) {
  const dec_config& f = c->cfg;
  Planner P{c};
  c->ops.reserve(16 * f.n_layers + 16);
  const int L = f.n_layers, d = f.d_model, V = f.vocab;
  const bool mla = f.arch == DEC_ARCH_MLA_MOE;
  // per-layer bookkeeping of the ops whose outputs feed the next layer's residual
  struct LayerOut {
    int ffn_op = -1;        // dense down op or MoE expert-down op
    int router_op = -1;     // MoE router op
    int mid_buf = -1;
  };
  std::vector<LayerOut> lo(L);
  std::vector<float*> h_in(L), h_mid(L);
  for (int l = 0; l < L; ++l) {
    if (dalloc(c, &h_in[l], d * 4) || dalloc(c, &h_mid[l], d * 4)) return DEC_ERR_OOM;
  }
  float* h_final = nullptr;
  if (dalloc(c, &h_final, d * 4)) return DEC_ERR_OOM;

  // residual input of layer l's attention block (and of the LM head for l == L)
  auto resid_in = [&](OpDesc& o, int l) {
    o.pro = PRO_RESID_NORM;
    o.n = d;
    o.gain = l < L ? gainp(c, DEC_W_ATTN_NORM, l) : gainp(c, DEC_W_FINAL_NORM, -1);
    if (l == 0) {
      o.base_embed = 1;
      o.embed = c->embed;
      o.embed_bf16 = c->act_bf16;
    } else {
      const LayerOut& p = lo[l - 1];
      const OpDesc& fo = c->ops[p.ffn_op];
      o.h_base = h_mid[l - 1];
      if (p.router_op < 0) {
        o.add = PSet{fo.out, fo.S, fo.out_stride, 0};
        o.dep[0] = p.ffn_op;
      } else {
        const OpDesc& ro = c->ops[p.router_op];
        o.routed = PSet{fo.out, fo.S, fo.out_stride, 0};
        o.routed_slot_stride = d;
        o.rt_w = ro.rt_w;
        o.n_experts = f.n_experts;
        o.top_k = f.top_k;
        if (f.n_shared > 0) o.add2 = PSet{fo.out, fo.S, fo.out_stride, f.top_k * d};
        o.dep[0] = p.ffn_op;
        o.dep[1] = p.router_op;
      }
    }
  };

  // split-KV chunks per head: about one attention task per CTA, at most 64 (one warp
  // combines up to 64 chunks) and few enough that the combine weights fit the scratch
  const int nch_dense = std::max(
      1, std::min({64, c->n_ctas / std::max(1, f.n_kv_heads), kMaxCombine / std::max(1, f.n_heads)}));
  // MLA: one attention task per cache block of kMlaBlock positions
  const int nch_mla = (f.max_seq + kMlaBlock - 1) / kMlaBlock;
  c->n_moe = 0;

  for (int l = 0; l < L; ++l) {
    int o_op;  // output projection op of this layer
    float* attn_buf[3];
    if (!mla) {
      const int hq = f.n_heads, hkv = f.n_kv_heads, hd = f.head_dim;
      Mat* wq = P.new_mat(DEC_W_Q, l, hq * hd, d, 1, 0);
      Mat* wk = P.new_mat(DEC_W_K, l, hkv * hd, d, 1, 0);
      Mat* wv = P.new_mat(DEC_W_V, l, hkv * hd, d, 1, 0);
      int qkv = P.gemv({{wq, -1, 0}, {wk, -1, 0}, {wv, -1, 0}}, d, l, false, "qkv", false);
      if (qkv < 0) return P.rc;
      {
        OpDesc& o = c->ops[qkv];
        resid_in(o, l);
        o.h_out = h_in[l];
      }
      // attention
      OpDesc a = P.base_op(OP_ATTN, l);
      a.hq = hq;
      a.hkv = hkv;
      a.hd = hd;
      a.gs = hq / hkv;
      {
        const OpDesc& p = c->ops[qkv];
        a.qkv = PSet{p.out, p.S, p.out_stride, 0};
      }
      a.nch = nch_dense;
      a.ntasks = hkv * a.nch;
      a.dep[0] = qkv;
      a.cache_bf16 = c->act_bf16;
      a.max_seq = f.max_seq;
      a.rope_dim = hd;
      a.attn_scale = (float)(1.0 / std::sqrt((double)hd));
      a.np = kStageBytes / (2 * hd * c->eb);
      for (int i = 0; i < 3; ++i) {
        size_t n = (size_t)hq * a.nch * (i == 2 ? hd : 1);
        if (dalloc(c, &attn_buf[i], n * 4)) return DEC_ERR_OOM;
      }
      a.m_out = attn_buf[0];
      a.l_out = attn_buf[1];
      a.o_out = attn_buf[2];
      if (dalloc(c, &a.o_fin, (size_t)hq * hd * 4)) return DEC_ERR_OOM;
      a.kcache = c->kc[l];
      a.vcache = c->vc[l];
      a.rope_cos = c->rope_cos;
      a.rope_sin = c->rope_sin;
      const int attn = P.push(a, "attn");
      Mat* wo = P.new_mat(DEC_W_O, l, d, hq * hd, 1, 0);
      o_op = P.gemv({{wo, -1, 0}}, hq * hd, l, false, "o_proj");
      if (o_op < 0) return P.rc;
      OpDesc& oo = c->ops[o_op];
      oo.pro = PRO_SUM;  // the attention op's last chunk task per kv head combined the chunks
      oo.n = hq * hd;
      oo.src = PSet{c->ops[attn].o_fin, 1, hq * hd, 0};
      oo.dep[0] = attn;
    } else {
      const int H = f.n_heads, nope = f.qk_nope, rd = f.qk_rope, vh = f.v_head, kvl = f.kv_lora;
      Mat* qa = P.new_mat(DEC_W_Q_A, l, f.q_lora, d, 1, 0);
      Mat* kva = P.new_mat(DEC_W_KV_A, l, kvl + rd, d, 1, 0);
      int s1 = P.gemv({{qa, -1, 0}, {kva, -1, 0}}, d, l, false, "q_a|kv_a");
      if (s1 < 0) return P.rc;
      {
        OpDesc& o = c->ops[s1];
        resid_in(o, l);
        o.h_out = h_in[l];
      }
      Mat* qb = P.new_mat(DEC_W_Q_B, l, H * (nope + rd), f.q_lora, 1, 0);
      int s2 = P.gemv({{qb, -1, 0}}, f.q_lora, l, false, "q_b", false);  // absorb_q reads one head per task
      if (s2 < 0) return P.rc;
      {
        OpDesc& o = c->ops[s2];
        const OpDesc& p = c->ops[s1];
        o.pro = PRO_NORM_SUM;
        o.n = f.q_lora;
        o.gain = gainp(c, DEC_W_Q_A_NORM, l);
        o.src = PSet{p.out, p.S, p.out_stride, 0};
        o.dep[0] = s1;
      }
      Mat* uk = P.new_mat(DEC_W_KV_B * 16 + 1, l, H * kvl, nope, 1, 1);  // W_UK^T view of kv_b
      int s3 = P.gemv({{uk, -1, -1}}, nope, l, true, "absorb_q");
      if (s3 < 0) return P.rc;
      // bf16 absorbed query [q_lat | q_pe] of all kMlaHeads (zero-padded) in the tensor-core layout
      void* qc = nullptr;
      {
        const size_t qb = (size_t)(kvl + rd) / 8 * 2048;
        if (dalloc(c, reinterpret_cast<uint8_t**>(&qc), qb)) return DEC_ERR_OOM;
        CK(cudaMemsetAsync(qc, 0, qb, c->stream));
      }
      {
        OpDesc& o = c->ops[s3];
        const OpDesc& p = c->ops[s2];
        o.pro = PRO_SUM;
        o.n = nope;
        o.src = PSet{p.out, p.S, p.out_stride, 0};
        o.gstride = nope + rd;
        o.rows_per_group = kvl;
        o.dep[0] = s2;
        o.qc = qc;
        o.nope = nope;
        o.rdim = rd;
        o.rope_cos = c->rope_cos;
        o.rope_sin = c->rope_sin;
        // an extra last task appends the step's latent row (normalised c, RoPE'd k_pe) to the cache
        const OpDesc& p1 = c->ops[s1];
        o.ckv = PSet{p1.out, p1.S, p1.out_stride, f.q_lora};
        o.kvnorm_g = gainp(c, DEC_W_KV_A_NORM, l);
        o.kcache = c->kc[l];
        group_tasks(o);
        o.ntasks += 1;  // the last task appends the step's latent row (on a CTA with no GEMV task here)
      }
      OpDesc a = P.base_op(OP_MLA, l);
      {
        const OpDesc& p1 = c->ops[s1];
        a.H = H;
        a.kvl = kvl;
        a.rdim = rd;
        a.nope = nope;
        a.nch = nch_mla;
        // few blocks (short caches): two or four tasks per block, each with that share of O's
        // columns, so that the output work goes to more CTAs
        a.osplit = kvl != 512 ? 1 : 4 * nch_mla <= c->n_ctas ? 4 : 2 * nch_mla <= c->n_ctas ? 2 : 1;
        a.ntasks = nch_mla * a.osplit;
        a.qc = qc;
        a.ckv = PSet{p1.out, p1.S, p1.out_stride, f.q_lora};
        a.dep[0] = s3;
        a.pdep = s3;  // the producer streams the absorbed query
        a.max_seq = f.max_seq;
        a.cache_bf16 = 1;
        a.rope_dim = rd;
        a.attn_scale = (float)(1.0 / std::sqrt((double)(nope + rd)));
        for (int i = 0; i < 3; ++i) {
          size_t n = (size_t)H * a.nch * (i == 2 ? kvl : 1);
          if (dalloc(c, &attn_buf[i], n * 4)) return DEC_ERR_OOM;
          CK(cudaMemsetAsync(attn_buf[i], 0, n * 4, c->stream));
        }
        a.m_out = attn_buf[0];
        a.l_out = attn_buf[1];
        a.o_out = attn_buf[2];
      }
      a.kcache = c->kc[l];
      a.rope_cos = c->rope_cos;
      a.rope_sin = c->rope_sin;
      a.kvnorm_g = gainp(c, DEC_W_KV_A_NORM, l);
      const int attn = P.push(a, "mla_attn");
      Mat* uv = P.new_mat(DEC_W_KV_B * 16 + 2, l, H * vh, kvl, 1, 2);  // W_UV view of kv_b
      int s5 = P.gemv({{uv, -1, -1}}, kvl, l, false, "uv");
      if (s5 < 0) return P.rc;
      {
        OpDesc& o = c->ops[s5];
        o.pro = PRO_MLA_COMBINE;
        o.n = kvl;
        o.am = attn_buf[0];
        o.al = attn_buf[1];
        o.ao = attn_buf[2];
        o.nch = nch_mla;
        o.nheads = H;
        o.hdim = kvl;
        o.rows_per_group = vh;
        o.dep[0] = attn;
        group_tasks(o);
      }
      Mat* wo = P.new_mat(DEC_W_O, l, d, H * vh, 1, 0);
      o_op = P.gemv({{wo, -1, 0}}, H * vh, l, false, "o_proj");
      if (o_op < 0) return P.rc;
      {
        OpDesc& o = c->ops[o_op];
        const OpDesc& p = c->ops[s5];
        o.pro = PRO_SUM;
        o.n = H * vh;
        o.src = PSet{p.out, p.S, p.out_stride, 0};
        o.dep[0] = s5;
      }
    }
    // ---- FFN
    const OpDesc& oo = c->ops[o_op];
    const PSet o_out{oo.out, oo.S, oo.out_stride, 0};
    auto ffn_resid = [&](OpDesc& o, bool write_h) {
      o.pro = PRO_RESID_NORM;
      o.n = d;
      o.gain = gainp(c, DEC_W_FFN_NORM, l);
      o.h_base = h_in[l];
      o.add = o_out;
      o.dep[0] = o_op;
      o.h_out = write_h ? h_mid[l] : nullptr;
    };
    if (!mla || l < f.n_dense_layers) {
      const int ff = f.ffn_hidden;
      Mat* wg = P.new_mat(DEC_W_GATE, l, ff, d, 1, 0);
      Mat* wu = P.new_mat(DEC_W_UP, l, ff, d, 1, 0);
      int gu = P.gemv({{wg, -1, 0}, {wu, -1, 0}}, d, l, false, "gate|up");
      if (gu < 0) return P.rc;
      ffn_resid(c->ops[gu], true);
      Mat* wd = P.new_mat(DEC_W_DOWN, l, d, ff, 1, 0);
      int dn = P.gemv({{wd, -1, 0}}, ff, l, false, "down");
      if (dn < 0) return P.rc;
      {
        OpDesc& o = c->ops[dn];
        const OpDesc& p = c->ops[gu];
        o.pro = PRO_SWIGLU;
        o.n = ff;
        o.gate = PSet{p.out, p.S, p.out_stride, 0};
        o.up = PSet{p.out, p.S, p.out_stride, ff};
        o.slot_stride = 0;
        o.dep[0] = gu;
      }
      lo[l].ffn_op = dn;
    } else {
      const int E = f.n_experts, k = f.top_k, eh = f.expert_hidden;
      Mat* wr = P.new_mat(DEC_W_ROUTER, l, E, d, 1, 0);
      int ro = P.gemv({{wr, -1, 0}}, d, l, false, "router");
      if (ro < 0) return P.rc;
      ffn_resid(c->ops[ro], true);
      {
        OpDesc& o = c->ops[ro];
        o.router = 1;
        o.n_experts = E;
        o.top_k = k;
        if (dalloc(c, &o.rt_ids, (size_t)k * 4) || dalloc(c, &o.rt_w, (size_t)k * 4)) return DEC_ERR_OOM;
        CK(cudaMemsetAsync(o.rt_ids, 0, (size_t)k * 4, c->stream));
        CK(cudaMemsetAsync(o.rt_w, 0, (size_t)k * 4, c->stream));
      }
      Mat* eg = P.new_mat(DEC_W_EXP_GATE, l, eh, d, E, 0);
      Mat* eu = P.new_mat(DEC_W_EXP_UP, l, eh, d, E, 0);
      Mat* sg = nullptr;
      Mat* su = nullptr;
      std::vector<SegSpec> segs;
      for (int j = 0; j < k; ++j) {
        segs.push_back({eg, j, 0});
        segs.push_back({eu, j, 0});
      }
      if (f.n_shared > 0) {
        sg = P.new_mat(DEC_W_SH_GATE, l, eh * f.n_shared, d, 1, 0);
        su = P.new_mat(DEC_W_SH_UP, l, eh * f.n_shared, d, 1, 0);
        segs.push_back({sg, -1, 0});
        segs.push_back({su, -1, 0});
      }
      int egu = P.gemv(segs, d, l, false, "exp_gate|up");
      if (egu < 0) return P.rc;
      int* rids = c->ops[ro].rt_ids;
      {
        OpDesc& o = c->ops[egu];
        ffn_resid(o, false);
        o.pdep = ro;
        o.rt_ids = rids;
        o.n_experts = E;
        o.top_k = k;
      }
      Mat* ed = P.new_mat(DEC_W_EXP_DOWN, l, d, eh, E, 0);
      Mat* sd = nullptr;
      std::vector<SegSpec> dsegs;
      for (int j = 0; j < k; ++j) dsegs.push_back({ed, j, j});
      if (f.n_shared > 0) {
        sd = P.new_mat(DEC_W_SH_DOWN, l, d, eh * f.n_shared, 1, 0);
        dsegs.push_back({sd, -1, k});
      }
      int edn = P.gemv(dsegs, eh, l, false, "exp_down");
      if (edn < 0) return P.rc;
      {
        OpDesc& o = c->ops[edn];
        const OpDesc& p = c->ops[egu];
        o.pro = PRO_SWIGLU;
        o.n = eh;
        o.gate = PSet{p.out, p.S, p.out_stride, 0};
        o.up = PSet{p.out, p.S, p.out_stride, eh};
        o.slot_stride = 2 * eh;
        o.dep[0] = egu;
        o.pdep = ro;
        o.rt_ids = rids;
        o.n_experts = E;
        o.top_k = k;
      }
      lo[l].ffn_op = edn;
      lo[l].router_op = ro;
      ++c->n_moe;
    }
  }
  // ---- LM head + argmax
  Mat* lm = P.new_mat(DEC_W_LM_HEAD, -1, V, d, 1, 0);
  int lmop = P.gemv({{lm, -1, 0}}, d, -1, true, "lm_head");
  if (lmop < 0) return P.rc;
  {
    OpDesc& o = c->ops[lmop];
    resid_in(o, L);
    o.h_out = h_final;
  }
  c->lm_op = lmop;
  OpDesc fin = P.base_op(OP_FINAL, -1);
  fin.ntasks = 1;
  fin.dep[0] = lmop;
  c->final_op = P.push(fin, "final");

  {
    OpDesc& o = c->ops[lmop];
    if (dalloc(c, &o.best, (size_t)o.ntasks * 8)) return DEC_ERR_OOM;
    c->logits = o.out;
    OpDesc& fo = c->ops[c->final_op];
    fo.fin_best = o.best;
    fo.fin_n = o.ntasks;
    fo.vocab = V;
    fo.logits = o.out;
  }
  return DEC_OK;
}

// ---------------------------------------------------------- task lists
// Each op's tasks are cut into n_ctas contiguous runs, one per CTA, starting
// at a CTA that rotates from op to op so that the remainders spread evenly.
// Contiguous runs keep a CTA on one input group (expert slot, head) so that
// the prologue building that group's input runs once per CTA, not per task.
static int assign_tasks(dec_ctx* c) {
  std::vector<std::vector<int2>> lists(c->n_ctas);
  const int nc = c->n_ctas;
  int rr = 0;
  for (int op = 0; op < (int)c->ops.size(); ++op) {
    const long long n = c->ops[op].ntasks;
    for (int i = 0; i < nc; ++i) {
      const int b = (rr + i) % nc;
      for (long long t = i * n / nc; t < (i + 1) * n / nc; ++t) lists[b].push_back(make_int2(op, (int)t));
    }
    rr = (int)((rr + n) % nc);
  }
  std::vector<int2> flat;
  c->task_off.assign(c->n_ctas + 1, 0);
  for (int b = 0; b < c->n_ctas; ++b) {
    c->task_off[b] = (int)flat.size();
    flat.insert(flat.end(), lists[b].begin(), lists[b].end());
  }
  c->task_off[c->n_ctas] = (int)flat.size();
  if (dalloc(c, &c->d_tasks, flat.size() * sizeof(int2))) return DEC_ERR_OOM;
  if (dalloc(c, &c->d_task_off, c->task_off.size() * sizeof(int))) return DEC_ERR_OOM;
  CK(cudaMemcpy(c->d_tasks, flat.data(), flat.size() * sizeof(int2), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(c->d_task_off, c->task_off.data(), c->task_off.size() * sizeof(int), cudaMemcpyHostToDevice));
  return DEC_OK;
}

static int upload_ops(dec_ctx* c) {
  // segment weight pointers are known once the matrices are allocated
  for (size_t i = 0; i < c->ops.size(); ++i) {
    OpDesc& o = c->ops[i];
    for (int s = 0; s < o.nsegs; ++s) {
      Mat* m = reinterpret_cast<Mat*>(c->seg_mats[i][s]);
      o.seg[s].w = m->w;
      o.seg[s].sc = m->sc;
    }
  }
  if (!c->d_ops && dalloc(c, &c->d_ops, c->ops.size() * sizeof(OpDesc))) return DEC_ERR_OOM;
  CK(cudaMemcpy(c->d_ops, c->ops.data(), c->ops.size() * sizeof(OpDesc), cudaMemcpyHostToDevice));
  return DEC_OK;
}

static int validate(const dec_config* f, dec_ctx* c) {
  auto bad = [&](const char* what) { return fail(c, DEC_ERR_INVALID_ARG, "invalid config: %s", what); };
  auto uns = [&](const char* what) { return fail(c, DEC_ERR_UNSUPPORTED, "unsupported config: %s", what); };
  if (f->arch != DEC_ARCH_DENSE && f->arch != DEC_ARCH_MLA_MOE) return bad("arch");
  if (f->weight_dtype < DEC_F32 || f->weight_dtype > DEC_FP8_E4M3_B128) return bad("weight_dtype");
  if (f->exec_mode < DEC_PERSISTENT || f->exec_mode > DEC_PER_OP_GRAPH) return bad("exec_mode");
  if (f->n_layers < 1 || f->d_model < 16 || f->vocab < 1 || f->max_seq < 2) return bad("sizes");
  if (!(f->norm_eps >= 0.f) || !(f->rope_theta > 0.f)) return bad("norm_eps / rope_theta");
  if (f->d_model > kMaxD) return uns("d_model > 8192");
  const int wb = f->weight_dtype == DEC_F32 ? 4 : f->weight_dtype == DEC_BF16 ? 2 : 1;
  auto k_ok = [&](long long K) { return K > 0 && (K * wb) % 16 == 0; };
  if (!k_ok(f->d_model)) return uns("d_model * weight bytes must be a multiple of 16");
  if (f->arch == DEC_ARCH_DENSE) {
    if (f->n_heads < 1 || f->n_kv_heads < 1 || f->n_heads % f->n_kv_heads) return bad("heads");
    if (f->n_heads / f->n_kv_heads > kConsumerWarps) return uns("GQA group > 8");
    if (f->n_heads > 128) return uns("n_heads > 128");
    if (f->head_dim != 64 && f->head_dim != 128) return uns("head_dim must be 64 or 128");
    if (f->ffn_hidden < 1 || !k_ok(f->ffn_hidden)) return uns("ffn_hidden alignment");
    if (!k_ok((long long)f->n_heads * f->head_dim)) return uns("n_heads*head_dim alignment");
  } else {
    if (f->weight_dtype == DEC_F32) return uns("MLA needs bf16 activations (bf16 or fp8 weights)");
    // tensor-core attention: heads fill (at most) the MMA's 128 rows; 64-dim K chunks; 256-dim O halves
    if (f->kv_lora != 512) return uns("kv_lora must be 512");
    if (f->qk_rope != 64 && f->qk_rope != 128) return uns("qk_rope must be 64 or 128");
    if (f->n_heads > kMlaHeads) return uns("MLA n_heads > 128");
    if (f->qk_nope < 16 || !k_ok(f->qk_nope)) return uns("qk_nope");
    if (f->v_head < 8 || !k_ok((long long)f->n_heads * f->v_head)) return uns("v_head");
    if (f->n_heads < 1 || f->n_heads > 1024) return bad("n_heads");
    if (f->q_lora < 16 || f->q_lora > kMaxD || !k_ok(f->q_lora)) return uns("q_lora");
    if (f->n_dense_layers < 0 || f->n_dense_layers > f->n_layers) return bad("n_dense_layers");
    if (f->n_dense_layers > 0 && (f->ffn_hidden < 1 || !k_ok(f->ffn_hidden))) return uns("ffn_hidden");
    if (f->n_dense_layers < f->n_layers) {
      if (f->n_experts < 1 || f->n_experts > 256) return uns("n_experts must be 1..256");
      if (f->top_k < 1 || f->top_k > kMaxTopK || f->top_k > f->n_experts) return bad("top_k");
      if (f->n_shared < 0 || f->n_shared > 1) return uns("n_shared must be 0 or 1");
      if (f->expert_hidden < 1 || !k_ok(f->expert_hidden)) return uns("expert_hidden");
      if (2 * f->top_k + 2 > kMaxSegs) return uns("top_k too large");
    }
  }
  return DEC_OK;
}

static int check_work_area(dec_ctx* c) {
  // The prologues read partial sums with 16-byte loads: every vector they read
  // must start, and every split must be strided, at a multiple of 4 floats.
  auto al = [](const PSet& p) { return !p.ptr || (p.off % 4 == 0 && p.stride % 4 == 0); };
  for (size_t i = 0; i < c->ops.size(); ++i) {
    const OpDesc& o = c->ops[i];
    const char* nm = c->op_names[i].c_str();
    if (o.kind != OP_GEMV) continue;
    const int cap = o.pro == PRO_MLA_COMBINE ? kCombineOff : kWorkBytes;
    if ((long long)o.Kpad * (o.in_bf16 ? 2 : 4) > cap)
      return fail(c, DEC_ERR_UNSUPPORTED, "input vector of op %zu (%s) exceeds the work area", i, nm);
    if (o.n % 4 || o.Kpad % 4 || !al(o.add) || !al(o.add2) || !al(o.routed) || !al(o.src) || !al(o.gate) ||
        !al(o.up) || o.routed_slot_stride % 4 || o.slot_stride % 4 || o.gstride % 4 || o.hdim % 4)
      return fail(c, DEC_ERR_UNSUPPORTED, "op %zu (%s): vector lengths and offsets must be multiples of 4", i, nm);
    if (o.pro == PRO_MLA_COMBINE && o.nch > kMaxCombine)
      return fail(c, DEC_ERR_UNSUPPORTED, "op %zu (%s): too many split-KV chunks", i, nm);
  }
  return DEC_OK;
}

static void free_all(dec_ctx* c) {
  if (c->graph) cudaGraphExecDestroy(c->graph);
  c->graph = nullptr;
  if (c->gen_done) cudaEventDestroy(c->gen_done);
  c->gen_done = nullptr;
  if (c->h_map) cudaFreeHost(c->h_map);
  c->h_map = nullptr;
  for (void* p : c->allocs) cudaFree(p);
  c->allocs.clear();
  if (c->staging) cudaFree(c->staging);
  c->staging = nullptr;
}

extern "C" int dec_create(const dec_config* cfg, dec_ctx** out) {
  if (!cfg || !out) return DEC_ERR_INVALID_ARG;
  *out = nullptr;
  dec_ctx* c = new dec_ctx();
  c->cfg = *cfg;
  int rc = validate(cfg, c);
  if (rc) {
    *out = c;  // so that dec_last_error works; caller must still destroy
    return rc;
  }
  const dec_config& f = c->cfg;
  c->wtype = f.weight_dtype == DEC_F32 ? WT_F32 : f.weight_dtype == DEC_BF16 ? WT_BF16 : WT_FP8;
  c->wb = f.weight_dtype == DEC_F32 ? 4 : f.weight_dtype == DEC_BF16 ? 2 : 1;
  c->act_bf16 = f.weight_dtype == DEC_F32 ? 0 : 1;
  c->eb = c->act_bf16 ? 2 : 4;
  c->mode = f.exec_mode;
  *out = c;
  CK(cudaSetDevice(f.device));
  int sms = 0, coop = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, f.device));
  CK(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, f.device));
  c->kernel = pick_kernel(c->wtype, f.arch == DEC_ARCH_MLA_MOE);
  CK(cudaFuncSetAttribute(c->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes));
  int per_sm = 0;
  CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, c->kernel, kThreads, kSmemBytes));
  if (per_sm < 1 || !coop) return fail(c, DEC_ERR_UNSUPPORTED, "device cannot host the persistent kernel");
  c->n_ctas = f.n_ctas > 0 ? std::min(f.n_ctas, sms * per_sm) : sms;
  CK(cudaStreamCreateWithFlags(&c->own_stream, cudaStreamNonBlocking));
  c->stream = c->own_stream;
  const int L = f.n_layers, d = f.d_model;
  const bool mla = f.arch == DEC_ARCH_MLA_MOE;
  // embedding, gains, caches, RoPE tables (referenced by the plan)
  if ((rc = dalloc(c, reinterpret_cast<uint8_t**>(&c->embed), (size_t)f.vocab * d * c->eb))) return rc;
  auto vec = [&](int kind, int layer, int n) -> int {
    Vec& v = c->vecs[{kind, layer}];
    v.n = n;
    return dalloc(c, &v.p, (size_t)n * 4);
  };
  if ((rc = vec(DEC_W_FINAL_NORM, -1, d))) return rc;
  for (int l = 0; l < L; ++l) {
    if ((rc = vec(DEC_W_ATTN_NORM, l, d)) || (rc = vec(DEC_W_FFN_NORM, l, d))) return rc;
    if (mla && ((rc = vec(DEC_W_Q_A_NORM, l, f.q_lora)) || (rc = vec(DEC_W_KV_A_NORM, l, f.kv_lora)))) return rc;
  }
  c->kc.assign(L, nullptr);
  c->vc.assign(L, nullptr);
  for (int l = 0; l < L; ++l) {
    if (!mla) {
      const size_t n = (size_t)f.n_kv_heads * f.max_seq * f.head_dim * c->eb;
      if ((rc = dalloc(c, reinterpret_cast<uint8_t**>(&c->kc[l]), n))) return rc;
      if ((rc = dalloc(c, reinterpret_cast<uint8_t**>(&c->vc[l]), n))) return rc;
      CK(cudaMemsetAsync(c->kc[l], 0, n, c->stream));
      CK(cudaMemsetAsync(c->vc[l], 0, n, c->stream));
    } else {  // whole blocks, zeroed: an MMA reads the unused tail rows of the last block (with P = 0)
      const size_t n = mla_cache_bytes(f);
      if ((rc = dalloc(c, reinterpret_cast<uint8_t**>(&c->kc[l]), n))) return rc;
      CK(cudaMemsetAsync(c->kc[l], 0, n, c->stream));
    }
  }
  {
    // RoPE tables: angle p * theta^(-2j/D), computed in double, stored as fp32
    const int D = mla ? f.qk_rope : f.head_dim;
    std::vector<float> cs((size_t)f.max_seq * (D / 2)), sn(cs.size());
    for (int p = 0; p < f.max_seq; ++p)
      for (int j = 0; j < D / 2; ++j) {
        const double ang = p * std::pow((double)f.rope_theta, -2.0 * j / D);
        cs[(size_t)p * (D / 2) + j] = (float)std::cos(ang);
        sn[(size_t)p * (D / 2) + j] = (float)std::sin(ang);
      }
    if ((rc = dalloc(c, &c->rope_cos, cs.size() * 4)) || (rc = dalloc(c, &c->rope_sin, sn.size() * 4))) return rc;
    CK(cudaMemcpy(c->rope_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(c->rope_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice));
  }
  if ((rc = build_plan(c))) return rc;
  if ((rc = check_work_area(c))) return rc;
  if ((rc = alloc_mats(c))) return rc;
  // routing dump: one row of top_k ids per MoE layer
  if (c->n_moe > 0) {
    if ((rc = dalloc(c, &c->d_route_dump, (size_t)c->n_moe * f.top_k * 4))) return rc;
    int i = 0;
    for (auto& o : c->ops)
      if (o.router) o.route_dump = c->d_route_dump + f.top_k * i++;
  }
  // Counters, one array that dec_reset zeroes: per op the dependency counter and
  // (routers) the finished-task counter, the latter at ops.size() + op; per dense
  // attention op one finished-task counter per kv head, after those.
  c->n_counters = 2 * c->ops.size();
  for (auto& o : c->ops)
    if (o.kind == OP_ATTN) c->n_counters += o.hkv;
  if ((rc = dalloc(c, &c->d_counters, c->n_counters * 4))) return rc;
  CK(cudaMemsetAsync(c->d_counters, 0, c->n_counters * 4, c->stream));
  {
    unsigned* next = c->d_counters + 2 * c->ops.size();
    for (size_t i = 0; i < c->ops.size(); ++i) {
      OpDesc& o = c->ops[i];
      if (o.router) o.fin = c->d_counters + c->ops.size() + i;
      if (o.kind == OP_ATTN) {
        o.fin = next;
        next += o.hkv;
      }
    }
  }
  if ((rc = upload_ops(c))) return rc;
  if ((rc = assign_tasks(c))) return rc;
  if ((rc = dalloc(c, &c->d_state, sizeof(StepState)))) return rc;
  if ((rc = dalloc(c, &c->d_gen, sizeof(GenState)))) return rc;
  CK(cudaMemsetAsync(c->d_gen, 0, sizeof(GenState), c->stream));
  {  // the token ring the device writes and the host reads while a generation runs
    const size_t mb = 16 + (size_t)f.max_seq * 4;
    cudaError_t e = cudaHostAlloc(&c->h_map, mb, cudaHostAllocMapped);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      c->h_map = nullptr;
      return fail(c, DEC_ERR_OOM, "mapped host memory for the token ring: %s", cudaGetErrorString(e));
    }
    memset(c->h_map, 0, mb);
    CK(cudaHostGetDevicePointer(reinterpret_cast<void**>(&c->d_map), c->h_map, 0));
    CK(cudaEventCreateWithFlags(&c->gen_done, cudaEventDisableTiming));
  }
  if ((rc = dalloc(c, &c->d_started, 4))) return rc;
  if ((rc = dalloc(c, &c->d_status, sizeof(Status)))) return rc;
  if (f.flags & DEC_FLAG_TRACE) {
    int total = 0;
    for (auto& o : c->ops) total += o.ntasks;
    c->trace_cap = total;
    if ((rc = dalloc(c, &c->d_trace, (2 + 9 * (size_t)total) * 8))) return rc;
  }
  // bytes a step reads from the weight store (active weights + scales)
  for (auto& kv : c->mats) {
    const Mat& m = kv.second;
    const int kind = std::get<0>(kv.first);
    const int nact = (kind == DEC_W_EXP_GATE || kind == DEC_W_EXP_UP || kind == DEC_W_EXP_DOWN) ? f.top_k : 1;
    c->weight_bytes_step += (m.tile_bytes + m.sc_count * 4) * nact;
  }
  CK(cudaStreamSynchronize(c->stream));
  return dec_reset(c);
}

extern "C" int dec_destroy(dec_ctx* c) {
  if (!c) return DEC_OK;
  if (c->own_stream) {  // creation got as far as the stream: the device is set up
    cudaSetDevice(c->cfg.device);
    cudaStreamSynchronize(c->stream);
  }
  free_all(c);
  if (c->own_stream) cudaStreamDestroy(c->own_stream);  // a stream given by dec_set_stream stays the caller's
  (void)cudaGetLastError();
  delete c;
  return DEC_OK;
}

extern "C" const char* dec_last_error(const dec_ctx* c) { return c ? c->err.c_str() : "null context"; }

extern "C" int dec_set_stream(dec_ctx* c, void* stream) {
  if (!c) return DEC_ERR_INVALID_ARG;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is running; call dec_generate_wait");
  CK(cudaStreamSynchronize(c->stream));
  if (c->graph) {
    cudaGraphExecDestroy(c->graph);
    c->graph = nullptr;
  }
  c->stream = reinterpret_cast<cudaStream_t>(stream);
  return DEC_OK;
}

extern "C" int dec_position(const dec_ctx* c, int32_t* out_pos) {
  if (!c || !out_pos) return DEC_ERR_INVALID_ARG;
  *out_pos = c->pos;
  return DEC_OK;
}

extern "C" int dec_reset(dec_ctx* c) {
  if (!c) return DEC_ERR_INVALID_ARG;
  CK(cudaSetDevice(c->cfg.device));
  cudaStreamSynchronize(c->stream);
  (void)cudaGetLastError();
  CK(cudaMemsetAsync(c->d_counters, 0, c->n_counters * 4, c->stream));
  CK(cudaMemsetAsync(c->d_started, 0, 4, c->stream));
  CK(cudaMemsetAsync(c->d_status, 0, sizeof(Status), c->stream));
  CK(cudaMemsetAsync(c->d_gen, 0, sizeof(GenState), c->stream));
  StepState st{1, 0, 0, 0};
  CK(cudaMemcpyAsync(c->d_state, &st, sizeof st, cudaMemcpyHostToDevice, c->stream));
  CK(cudaStreamSynchronize(c->stream));
  c->generating = false;
  c->pos = 0;
  c->epoch = 1;
  c->have_ctx = false;
  c->poisoned = false;
  c->pending = 0;
  return DEC_OK;
}

// --------------------------------------------------------------- weights
static int staging_for(dec_ctx* c, size_t bytes) {
  if (c->staging_bytes >= bytes) return DEC_OK;
  if (c->staging) cudaFree(c->staging);
  c->staging = nullptr;
  c->staging_bytes = 0;
  if (cudaMalloc(&c->staging, bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(c, DEC_ERR_OOM, "staging buffer of %zu bytes", bytes);
  }
  c->staging_bytes = bytes;
  return DEC_OK;
}

static bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// Source bytes on the device (staged if the caller passed host memory).
static int device_source(dec_ctx* c, const void* data, size_t bytes, const uint8_t** out) {
  if (is_device_ptr(data)) {
    *out = reinterpret_cast<const uint8_t*>(data);
    return DEC_OK;
  }
  int rc = staging_for(c, bytes);
  if (rc) return rc;
  CK(cudaMemcpyAsync(c->staging, data, bytes, cudaMemcpyDefault, c->stream));
  *out = c->staging;
  return DEC_OK;
}

static int load_matrix(dec_ctx* c, Mat& m, int expert, const void* data, const float* scales, size_t bytes,
                       const char* what) {
  const size_t want = (size_t)m.N * m.K * m.wb;
  if (bytes != want) return fail(c, DEC_ERR_INVALID_ARG, "%s: %zu bytes given, %zu expected", what, bytes, want);
  if (m.wtype == WT_FP8 && !scales) return fail(c, DEC_ERR_INVALID_ARG, "%s: FP8 weights need scales", what);
  const uint8_t* src = nullptr;
  int rc = device_source(c, data, bytes, &src);
  if (rc) return rc;
  uint8_t* dst = m.w + (size_t)expert * m.tile_bytes;
  const long long total16 = (long long)(m.tile_bytes / 16);
  const int grid = (int)std::min<long long>((total16 + 255) / 256, 148 * 16);
  relayout16<<<std::max(grid, 1), 256, 0, c->stream>>>(src, m.N, m.K, m.wb, m.R, m.S, m.nst, m.kcb, total16, dst);
  CK(cudaGetLastError());
  if (m.sc_count) CK(cudaMemcpyAsync(m.sc + (size_t)expert * m.sc_count, scales, m.sc_count * 4, cudaMemcpyDefault, c->stream));
  CK(cudaStreamSynchronize(c->stream));
  m.loaded |= 1;
  return DEC_OK;
}

static int load_kvb(dec_ctx* c, int layer, const void* data, const float* scales, size_t bytes) {
  const dec_config& f = c->cfg;
  const int H = f.n_heads, nope = f.qk_nope, vh = f.v_head, kvl = f.kv_lora;
  const size_t want = (size_t)H * (nope + vh) * kvl * c->wb;
  if (bytes != want) return fail(c, DEC_ERR_INVALID_ARG, "kv_b: %zu bytes given, %zu expected", bytes, want);
  if (c->wtype == WT_FP8 && !scales) return fail(c, DEC_ERR_INVALID_ARG, "kv_b: FP8 weights need scales");
  if ((nope % 128 || vh % 128) && c->wtype == WT_FP8)
    return fail(c, DEC_ERR_UNSUPPORTED, "FP8 kv_b needs qk_nope and v_head multiples of 128");
  const uint8_t* src = nullptr;
  int rc = device_source(c, data, bytes, &src);
  if (rc) return rc;
  for (int mode = 1; mode <= 2; ++mode) {
    Mat& m = c->mats[{DEC_W_KV_B * 16 + mode, layer}];
    const long long total = (long long)m.tile_bytes;
    const int grid = (int)std::min<long long>((total + 255) / 256, 148 * 16);
    relayout_kvb<<<std::max(grid, 1), 256, 0, c->stream>>>(src, mode, m.N, m.K, m.wb, m.R, m.S, m.nst, m.kcb, total,
                                                           nope, vh, kvl, m.w);
    CK(cudaGetLastError());
  }
  if (c->wtype == WT_FP8) {
    // kv_b scales [H*(nope+vh)/128][kvl/128]; views: W_UK^T block (h*kvl/128 + cb, j/128), W_UV (h*vh/128 + vb, cb)
    const int rb_per_head = (nope + vh) / 128, nkb = kvl / 128;
    std::vector<float> s((size_t)H * rb_per_head * nkb);
    CK(cudaMemcpy(s.data(), scales, s.size() * 4, cudaMemcpyDefault));
    Mat& uk = c->mats[{DEC_W_KV_B * 16 + 1, layer}];
    Mat& uv = c->mats[{DEC_W_KV_B * 16 + 2, layer}];
    const int uk_nkb = (nope + 127) / 128, uv_nkb = nkb;
    std::vector<float> suk(uk.sc_count), suv(uv.sc_count);
    for (int h = 0; h < H; ++h) {
      for (int cb = 0; cb < nkb; ++cb)
        for (int jb = 0; jb < nope / 128; ++jb)
          suk[((size_t)h * nkb + cb) * uk_nkb + jb] = s[((size_t)h * rb_per_head + jb) * nkb + cb];
      for (int vb = 0; vb < vh / 128; ++vb)
        for (int cb = 0; cb < nkb; ++cb)
          suv[((size_t)h * (vh / 128) + vb) * uv_nkb + cb] = s[((size_t)h * rb_per_head + nope / 128 + vb) * nkb + cb];
    }
    CK(cudaMemcpy(uk.sc, suk.data(), suk.size() * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(uv.sc, suv.data(), suv.size() * 4, cudaMemcpyHostToDevice));
  }
  CK(cudaStreamSynchronize(c->stream));
  c->mats[{DEC_W_KV_B * 16 + 1, layer}].loaded |= 1;
  c->mats[{DEC_W_KV_B * 16 + 2, layer}].loaded |= 1;
  return DEC_OK;
}

extern "C" int dec_load_weights(dec_ctx* c, const dec_tensor* t, int n) {
  if (!c || (!t && n > 0) || n < 0) return DEC_ERR_INVALID_ARG;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is running; call dec_generate_wait");
  CK(cudaSetDevice(c->cfg.device));
  // Device sources may have been produced on any stream: read them only after
  // all work already submitted to the device has finished.
  CK(cudaDeviceSynchronize());
  const dec_config& f = c->cfg;
  for (int i = 0; i < n; ++i) {
    const dec_tensor& x = t[i];
    if (!x.data) return fail(c, DEC_ERR_INVALID_ARG, "tensor %d: null data", i);
    const int layer = x.layer;
    const bool global = x.kind == DEC_W_EMBED || x.kind == DEC_W_FINAL_NORM || x.kind == DEC_W_LM_HEAD;
    if (global ? layer != -1 : (layer < 0 || layer >= f.n_layers))
      return fail(c, DEC_ERR_INVALID_ARG, "tensor %d: bad layer %d for kind %d", i, layer, x.kind);
    int rc = DEC_OK;
    if (x.kind == DEC_W_EMBED) {
      const size_t want = (size_t)f.vocab * f.d_model * c->eb;
      if (x.bytes != want) return fail(c, DEC_ERR_INVALID_ARG, "embed: %zu bytes, %zu expected", x.bytes, want);
      CK(cudaMemcpyAsync(c->embed, x.data, want, cudaMemcpyDefault, c->stream));
      CK(cudaStreamSynchronize(c->stream));
      c->embed_loaded = true;
      continue;
    }
    auto vit = c->vecs.find({x.kind, layer});
    if (vit != c->vecs.end()) {
      Vec& v = vit->second;
      if (x.bytes != (size_t)v.n * 4) return fail(c, DEC_ERR_INVALID_ARG, "norm %d: %zu bytes", x.kind, x.bytes);
      CK(cudaMemcpyAsync(v.p, x.data, x.bytes, cudaMemcpyDefault, c->stream));
      CK(cudaStreamSynchronize(c->stream));
      v.loaded = true;
      continue;
    }
    if (x.kind == DEC_W_KV_B && f.arch == DEC_ARCH_MLA_MOE) {
      if ((rc = load_kvb(c, layer, x.data, x.scales, x.bytes))) return rc;
      continue;
    }
    auto mit = c->mats.find({x.kind, layer});
    if (mit == c->mats.end())
      return fail(c, DEC_ERR_INVALID_ARG, "tensor %d: kind %d does not exist in layer %d of this model", i, x.kind,
                  layer);
    Mat& m = mit->second;
    int e = 0;
    if (m.n_experts > 1 || x.kind == DEC_W_EXP_GATE || x.kind == DEC_W_EXP_UP || x.kind == DEC_W_EXP_DOWN) {
      if (x.expert < 0 || x.expert >= m.n_experts)
        return fail(c, DEC_ERR_INVALID_ARG, "tensor %d: expert %d out of range", i, x.expert);
      e = x.expert;
    }
    char what[64];
    snprintf(what, sizeof what, "kind %d layer %d expert %d", x.kind, layer, e);
    if ((rc = load_matrix(c, m, e, x.data, x.scales, x.bytes, what))) return rc;
  }
  return DEC_OK;
}

static bool all_loaded(dec_ctx* c) {
  if (!c->embed_loaded) return false;
  for (auto& kv : c->vecs)
    if (!kv.second.loaded) return false;
  for (auto& kv : c->mats)
    if (!kv.second.loaded) return false;
  return true;
}

// ------------------------------------------------------------------ cache
extern "C" int dec_set_kv_cache(dec_ctx* c, const void* k_or_latent, const void* v_or_pe, int32_t n_tokens) {
  if (!c) return DEC_ERR_INVALID_ARG;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is running; call dec_generate_wait");
  const dec_config& f = c->cfg;
  if (n_tokens < 0) return fail(c, DEC_ERR_INVALID_ARG, "n_tokens < 0");
  if (n_tokens >= f.max_seq) return fail(c, DEC_ERR_CAPACITY, "context of %d tokens needs max_seq > %d", n_tokens, n_tokens);
  if (n_tokens > 0 && (!k_or_latent || !v_or_pe)) return fail(c, DEC_ERR_INVALID_ARG, "null cache pointer");
  CK(cudaSetDevice(f.device));
  CK(cudaDeviceSynchronize());  // device sources may come from any stream
  int rc = dec_reset(c);
  if (rc) return rc;
  const bool mla = f.arch == DEC_ARCH_MLA_MOE;
  uint8_t* rows = nullptr;  // MLA only: [n][kv_lora | qk_rope] rows of one layer, freed on every path
  auto copy_layers = [&]() -> int {
    for (int l = 0; l < f.n_layers && n_tokens > 0; ++l) {
      if (!mla) {
        const size_t row = (size_t)n_tokens * f.head_dim * c->eb;  // one kv head
        const size_t src_layer = (size_t)f.n_kv_heads * row;
        const size_t dpitch = (size_t)f.max_seq * f.head_dim * c->eb;
        CK(cudaMemcpy2DAsync(c->kc[l], dpitch, (const uint8_t*)k_or_latent + l * src_layer, row, row, f.n_kv_heads,
                             cudaMemcpyDefault, c->stream));
        CK(cudaMemcpy2DAsync(c->vc[l], dpitch, (const uint8_t*)v_or_pe + l * src_layer, row, row, f.n_kv_heads,
                             cudaMemcpyDefault, c->stream));
      } else {  // rows [n][kv_lora | qk_rope] in a scratch buffer, then the blocked layout
        const size_t lat = (size_t)f.kv_lora * 2, pe = (size_t)f.qk_rope * 2, rowb = lat + pe;
        if (!rows) {
          cudaError_t e = cudaMalloc(&rows, (size_t)n_tokens * rowb);
          if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return fail(c, DEC_ERR_OOM, "cache scratch of %zu bytes: %s", (size_t)n_tokens * rowb, cudaGetErrorString(e));
          }
        }
        CK(cudaMemcpy2DAsync(rows, rowb, (const uint8_t*)k_or_latent + (size_t)l * n_tokens * lat, lat, lat, n_tokens,
                             cudaMemcpyDefault, c->stream));
        CK(cudaMemcpy2DAsync(rows + lat, rowb, (const uint8_t*)v_or_pe + (size_t)l * n_tokens * pe, pe, pe, n_tokens,
                             cudaMemcpyDefault, c->stream));
        mla_cache_convert<<<1184, 256, 0, c->stream>>>(rows, (uint8_t*)c->kc[l], n_tokens, f.kv_lora + f.qk_rope, 1);
        CK(cudaGetLastError());
      }
    }
    return DEC_OK;
  };
  rc = copy_layers();
  if (rows) {
    const cudaError_t es = cudaStreamSynchronize(c->stream);
    const cudaError_t ef = cudaFree(rows);
    if (!rc && (es != cudaSuccess || ef != cudaSuccess))
      return fail(c, DEC_ERR_CUDA, "cache scratch: %s", cudaGetErrorString(es != cudaSuccess ? es : ef));
  }
  if (rc) return rc;
  StepState st{1, n_tokens, 0, 0};
  CK(cudaMemcpyAsync(c->d_state, &st, sizeof st, cudaMemcpyHostToDevice, c->stream));
  CK(cudaStreamSynchronize(c->stream));
  c->pos = n_tokens;
  c->have_ctx = true;
  return DEC_OK;
}

// ------------------------------------------------------------------ steps
static KParams kparams(dec_ctx* c, int persistent, int op, int tok_in) {
  KParams P;
  memset(&P, 0, sizeof P);
  P.ops = c->d_ops;
  P.nops = (int)c->ops.size();
  P.tasks = c->d_tasks;
  P.task_off = c->d_task_off;
  P.counters = c->d_counters;
  P.state = c->d_state;
  P.started = c->d_started;
  P.status = c->d_status;
  const unsigned us = c->cfg.wait_timeout_us ? c->cfg.wait_timeout_us : 1000000u;
  P.timeout_ns = (unsigned long long)us * 1000ull;
  P.persistent = persistent;
  P.op_only = op;
  P.n_ctas = c->n_ctas;
  P.trace = c->d_trace;
  P.trace_cap = c->trace_cap;
  P.tok_in = tok_in;
  P.test_stall = (c->cfg.flags & DEC_FLAG_TEST_STALL) ? 1 : 0;
  {
    // cache bytes one step reads at the current position (all layers), against 3/4 of L2
    const dec_config& f = c->cfg;
    const long long row = f.arch == DEC_ARCH_MLA_MOE ? (long long)(f.kv_lora + f.qk_rope) * c->eb
                                                     : 2LL * f.n_kv_heads * f.head_dim * c->eb;
    P.kv_evict_first = (long long)(c->pos + 1) * f.n_layers * row > kL2Bytes / 4 * 3 ? 1 : 0;
  }
  P.n_steps = 1;
  P.gen = c->d_gen;
  P.tok_count = reinterpret_cast<unsigned*>(c->d_map);
  P.stop_word = reinterpret_cast<const int*>(c->d_map + 4);
  P.tok_ring = reinterpret_cast<int*>(c->d_map + 16);
  return P;
}

static int launch_per_op(dec_ctx* c, int tok_in) {
  for (int op = 0; op < (int)c->ops.size(); ++op) {
    KParams P = kparams(c, 0, op, op == 0 ? tok_in : -1);
    const int grid = std::min(c->ops[op].ntasks, c->n_ctas);
    void* args[] = {&P};
    CK(cudaLaunchKernel(c->kernel, dim3(grid), dim3(kThreads), args, kSmemBytes, c->stream));
  }
  return DEC_OK;
}

static int ensure_graph(dec_ctx* c) {
  if (c->graph) return DEC_OK;
  cudaGraph_t g = nullptr;
  CK(cudaStreamBeginCapture(c->stream, cudaStreamCaptureModeThreadLocal));
  int rc = launch_per_op(c, -1);
  cudaError_t e = cudaStreamEndCapture(c->stream, &g);
  if (rc) {
    if (g) cudaGraphDestroy(g);
    return rc;
  }
  if (e != cudaSuccess) return fail(c, DEC_ERR_CUDA, "graph capture: %s", cudaGetErrorString(e));
  e = cudaGraphInstantiate(&c->graph, g, 0);
  cudaGraphDestroy(g);
  if (e != cudaSuccess) return fail(c, DEC_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
  return DEC_OK;
}

static int enqueue_step(dec_ctx* c, int32_t token_id) {
  const dec_config& f = c->cfg;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is running; call dec_generate_wait");
  if (c->poisoned) return fail(c, DEC_ERR_STATE, "context poisoned by an earlier device failure; call dec_reset");
  if (!all_loaded(c)) return fail(c, DEC_ERR_STATE, "not every weight tensor has been loaded");
  if (!c->have_ctx) return fail(c, DEC_ERR_STATE, "no context: call dec_set_kv_cache first");
  if (c->pos + 1 > f.max_seq) return fail(c, DEC_ERR_CAPACITY, "position %d reaches max_seq %d", c->pos, f.max_seq);
  if (token_id >= f.vocab) return fail(c, DEC_ERR_INVALID_ARG, "token %d >= vocab %d", token_id, f.vocab);
  if (token_id < 0 && c->epoch == 1)  // epoch 1: no step since the last reset / context install
    return fail(c, DEC_ERR_STATE, "no previous greedy token to feed back");
  CK(cudaSetDevice(f.device));
  if (c->d_trace) CK(cudaMemsetAsync(c->d_trace, 0, (2 + 9 * (size_t)c->trace_cap) * 8, c->stream));
  int rc = DEC_OK;
  if (c->mode == DEC_PERSISTENT) {
    KParams P = kparams(c, 1, -1, token_id);
    void* args[] = {&P};
    CK(cudaLaunchCooperativeKernel(c->kernel, dim3(c->n_ctas), dim3(kThreads), args, kSmemBytes, c->stream));
  } else if (c->mode == DEC_PER_OP) {
    rc = launch_per_op(c, token_id);
  } else {
    if ((rc = ensure_graph(c))) return rc;
    if (token_id >= 0) {
      set_int<<<1, 1, 0, c->stream>>>(&c->d_state->tok, token_id);
      CK(cudaGetLastError());
    }
    CK(cudaGraphLaunch(c->graph, c->stream));
  }
  if (rc) return rc;
  c->pos += 1;
  c->epoch += 1;
  c->pending += 1;
  return DEC_OK;
}

static int finish(dec_ctx* c, float* out_logits, int32_t* out_next) {
  Status st;
  StepState ss;
  CK(cudaMemcpyAsync(&st, c->d_status, sizeof st, cudaMemcpyDeviceToHost, c->stream));
  CK(cudaMemcpyAsync(&ss, c->d_state, sizeof ss, cudaMemcpyDeviceToHost, c->stream));
  CK(cudaStreamSynchronize(c->stream));
  c->pending = 0;
  if (st.code != 0) {
    c->poisoned = true;
    const char* nm = st.op >= 0 && st.op < (int)c->op_names.size() ? c->op_names[st.op].c_str() : "?";
    if (st.code == 2)
      return fail(c, DEC_ERR_NUMERIC, "non-finite logit (cta %d, op %d '%s', task %d)", st.cta, st.op, nm, st.task);
    return fail(c, DEC_ERR_TIMEOUT, "device wait timed out (cta %d, op %d '%s', task %d)", st.cta, st.op, nm,
                st.task);
  }
  if (out_next) *out_next = ss.last;
  if (out_logits) {
    CK(cudaMemcpyAsync(out_logits, c->logits, (size_t)c->cfg.vocab * 4, cudaMemcpyDefault, c->stream));
    CK(cudaStreamSynchronize(c->stream));
  }
  return DEC_OK;
}

extern "C" int dec_step(dec_ctx* c, int32_t token_id, float* out_logits, int32_t* out_next_token) {
  if (!c) return DEC_ERR_INVALID_ARG;
  int rc = enqueue_step(c, token_id);
  if (rc) return rc;
  return finish(c, out_logits, out_next_token);
}

extern "C" int dec_step_async(dec_ctx* c, int32_t token_id) {
  if (!c) return DEC_ERR_INVALID_ARG;
  return enqueue_step(c, token_id);
}

extern "C" int dec_sync(dec_ctx* c, float* out_logits, int32_t* out_next_token) {
  if (!c) return DEC_ERR_INVALID_ARG;
  return finish(c, out_logits, out_next_token);
}

// ------------------------------------------------------------- generation
// A decode lifetime with the host out of the loop: in DEC_PERSISTENT mode one kernel
// launch runs every step, feeding each greedy token back on the device and writing it
// to a host-mapped ring as soon as it is known (InferenceX article, "what TileRT is":
// the host launches once for the whole decode).  The other modes run the same steps
// one launch per step (per op, or a CUDA graph per step) with a host check of the stop
// condition after each step: the ablation of what the single launch removes.
extern "C" int dec_generate_async(dec_ctx* c, int32_t token_id, int32_t n_steps, int32_t stop_token) {
  if (!c) return DEC_ERR_INVALID_ARG;
  const dec_config& f = c->cfg;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is already running");
  if (n_steps < 1) return fail(c, DEC_ERR_INVALID_ARG, "n_steps < 1");
  if (c->pos + n_steps > f.max_seq)
    return fail(c, DEC_ERR_CAPACITY, "position %d + %d steps exceeds max_seq %d", c->pos, n_steps, f.max_seq);
  if (c->poisoned) return fail(c, DEC_ERR_STATE, "context poisoned by an earlier device failure; call dec_reset");
  if (!all_loaded(c)) return fail(c, DEC_ERR_STATE, "not every weight tensor has been loaded");
  if (!c->have_ctx) return fail(c, DEC_ERR_STATE, "no context: call dec_set_kv_cache first");
  if (token_id >= f.vocab) return fail(c, DEC_ERR_INVALID_ARG, "token %d >= vocab %d", token_id, f.vocab);
  if (token_id < 0 && c->epoch == 1) return fail(c, DEC_ERR_STATE, "no previous greedy token to feed back");
  CK(cudaSetDevice(f.device));
  CK(cudaStreamSynchronize(c->stream));  // the ring and stop word are reused: nothing may still write them
  *h_count(c) = 0;
  *h_stop(c) = 0;
  GenState g{1, c->epoch, stop_token, 0};
  CK(cudaMemcpyAsync(c->d_gen, &g, sizeof g, cudaMemcpyHostToDevice, c->stream));
  c->gen_epoch0 = c->epoch;
  c->gen_steps = n_steps;
  c->gen_stop_token = stop_token;
  if (c->d_trace) CK(cudaMemsetAsync(c->d_trace, 0, (2 + 9 * (size_t)c->trace_cap) * 8, c->stream));
  if (c->mode == DEC_PERSISTENT) {
    KParams P = kparams(c, 1, -1, token_id);
    P.n_steps = n_steps;
    void* args[] = {&P};
    CK(cudaLaunchCooperativeKernel(c->kernel, dim3(c->n_ctas), dim3(kThreads), args, kSmemBytes, c->stream));
  } else {  // one launch per step; the host checks the stop condition after each
    for (int i = 0; i < n_steps; ++i) {
      int rc = c->mode == DEC_PER_OP ? launch_per_op(c, i == 0 ? token_id : -1) : DEC_OK;
      if (c->mode == DEC_PER_OP_GRAPH) {
        if ((rc = ensure_graph(c))) return rc;
        if (i == 0 && token_id >= 0) {
          set_int<<<1, 1, 0, c->stream>>>(&c->d_state->tok, token_id);
          CK(cudaGetLastError());
        }
        CK(cudaGraphLaunch(c->graph, c->stream));
      }
      if (rc) return rc;
      CK(cudaStreamSynchronize(c->stream));
      const unsigned n = *h_count(c);
      if (n < (unsigned)(i + 1) || (n > 0 && h_ring(c)[n - 1] == stop_token) || *h_stop(c)) break;
    }
  }
  CK(cudaEventRecord(c->gen_done, c->stream));
  c->generating = true;
  return DEC_OK;
}

extern "C" int dec_generate_poll(dec_ctx* c, int32_t* out_tokens, int32_t cap, int32_t* out_count,
                                 int32_t* out_done) {
  if (!c || cap < 0 || (cap > 0 && !out_tokens)) return DEC_ERR_INVALID_ARG;
  if (!c->generating) return fail(c, DEC_ERR_STATE, "no generation is running");
  const unsigned n = *h_count(c);  // the device writes a ring entry before the count
  for (unsigned i = 0; i < n && (int)i < cap; ++i) out_tokens[i] = h_ring(c)[i];
  if (out_count) *out_count = (int32_t)n;
  if (out_done) {
    const cudaError_t e = cudaEventQuery(c->gen_done);
    if (e != cudaSuccess && e != cudaErrorNotReady) return fail(c, DEC_ERR_CUDA, "%s", cudaGetErrorString(e));
    (void)cudaGetLastError();
    *out_done = e == cudaSuccess;
  }
  return DEC_OK;
}

extern "C" int dec_generate_stop(dec_ctx* c) {
  if (!c) return DEC_ERR_INVALID_ARG;
  *h_stop(c) = 1;
  return DEC_OK;
}

extern "C" int dec_generate_wait(dec_ctx* c, int32_t* out_tokens, int32_t cap, int32_t* out_count) {
  if (!c || cap < 0 || (cap > 0 && !out_tokens)) return DEC_ERR_INVALID_ARG;
  if (!c->generating) return fail(c, DEC_ERR_STATE, "no generation is running");
  CK(cudaSetDevice(c->cfg.device));
  Status st;
  StepState ss;
  const GenState off{0, 0, -1, 0};
  CK(cudaMemcpyAsync(&st, c->d_status, sizeof st, cudaMemcpyDeviceToHost, c->stream));
  CK(cudaMemcpyAsync(&ss, c->d_state, sizeof ss, cudaMemcpyDeviceToHost, c->stream));
  CK(cudaMemcpyAsync(c->d_gen, &off, sizeof off, cudaMemcpyHostToDevice, c->stream));
  CK(cudaStreamSynchronize(c->stream));
  c->generating = false;
  const int done = ss.epoch - c->gen_epoch0;  // steps completed
  c->pos += done;
  c->epoch += done;
  const unsigned n = *h_count(c);
  for (unsigned i = 0; i < n && (int)i < cap; ++i) out_tokens[i] = h_ring(c)[i];
  if (out_count) *out_count = (int32_t)n;
  if (st.code != 0) {
    c->poisoned = true;
    const char* nm = st.op >= 0 && st.op < (int)c->op_names.size() ? c->op_names[st.op].c_str() : "?";
    if (st.code == 2)
      return fail(c, DEC_ERR_NUMERIC, "non-finite logit (cta %d, op %d '%s', task %d)", st.cta, st.op, nm, st.task);
    return fail(c, DEC_ERR_TIMEOUT, "device wait timed out (cta %d, op %d '%s', task %d)", st.cta, st.op, nm,
                st.task);
  }
  return DEC_OK;
}

extern "C" int dec_generate(dec_ctx* c, int32_t token_id, int32_t n_steps, int32_t stop_token, int32_t* out_tokens,
                            int32_t* out_count) {
  int rc = dec_generate_async(c, token_id, n_steps, stop_token);
  if (rc) return rc;
  return dec_generate_wait(c, out_tokens, n_steps, out_count);
}

extern "C" int dec_set_exec_mode(dec_ctx* c, int32_t mode) {
  if (!c || mode < DEC_PERSISTENT || mode > DEC_PER_OP_GRAPH) return DEC_ERR_INVALID_ARG;
  if (c->generating) return fail(c, DEC_ERR_STATE, "a generation is running; call dec_generate_wait");
  CK(cudaStreamSynchronize(c->stream));
  c->mode = mode;
  if (mode == DEC_PER_OP_GRAPH) return ensure_graph(c);
  return DEC_OK;
}

// ------------------------------------------------------------------ debug
extern "C" int dec_debug_dump(dec_ctx* c, int32_t what, void* dst, size_t bytes, size_t* out_bytes) {
  if (!c) return DEC_ERR_INVALID_ARG;
  const dec_config& f = c->cfg;
  CK(cudaStreamSynchronize(c->stream));
  if (what == DEC_DUMP_KV) {
    const bool mla = f.arch == DEC_ARCH_MLA_MOE;
    const int n = c->pos;
    size_t need;
    if (!mla)
      need = 2ull * f.n_layers * f.n_kv_heads * n * f.head_dim * c->eb;
    else
      need = (size_t)f.n_layers * n * (f.kv_lora + f.qk_rope) * 2;
    if (out_bytes) *out_bytes = need;
    if (!dst) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    uint8_t* o = reinterpret_cast<uint8_t*>(dst);
    uint8_t* rows = nullptr;  // MLA only: one layer's [n][kv_lora | qk_rope] rows
    struct FreeRows {         // freed on every return, the CK(...) error returns included
      uint8_t*& p;
      ~FreeRows() {
        if (p) cudaFree(p);
      }
    } free_rows{rows};
    for (int l = 0; l < f.n_layers && n > 0; ++l) {
      if (!mla) {
        const size_t row = (size_t)n * f.head_dim * c->eb, sp = (size_t)f.max_seq * f.head_dim * c->eb;
        const size_t half = need / 2, lb = (size_t)f.n_kv_heads * row;
        CK(cudaMemcpy2D(o + l * lb, row, c->kc[l], sp, row, f.n_kv_heads, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy2D(o + half + l * lb, row, c->vc[l], sp, row, f.n_kv_heads, cudaMemcpyDeviceToHost));
      } else {
        const size_t lat = (size_t)f.kv_lora * 2, pe = (size_t)f.qk_rope * 2, rowb = lat + pe;
        const size_t nl = (size_t)f.n_layers * n;
        if (!rows) {
          cudaError_t e = cudaMalloc(&rows, (size_t)n * rowb);
          if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return fail(c, DEC_ERR_OOM, "dump scratch: %s", cudaGetErrorString(e));
          }
        }
        mla_cache_convert<<<1184, 256, 0, c->stream>>>(rows, (uint8_t*)c->kc[l], n, f.kv_lora + f.qk_rope, 0);
        CK(cudaGetLastError());
        CK(cudaStreamSynchronize(c->stream));
        CK(cudaMemcpy2D(o + (size_t)l * n * lat, lat, rows, rowb, lat, n, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy2D(o + nl * lat + (size_t)l * n * pe, pe, rows + lat, rowb, pe, n, cudaMemcpyDeviceToHost));
      }
    }
    if (rows) {
      const cudaError_t e = cudaFree(rows);
      rows = nullptr;
      if (e != cudaSuccess) return fail(c, DEC_ERR_CUDA, "dump scratch: %s", cudaGetErrorString(e));
    }
    return DEC_OK;
  }
  if (what == DEC_DUMP_ROUTES) {
    const size_t need = (size_t)c->n_moe * f.top_k * 4;
    if (out_bytes) *out_bytes = need;
    if (!dst || need == 0) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    CK(cudaMemcpy(dst, c->d_route_dump, need, cudaMemcpyDeviceToHost));
    return DEC_OK;
  }
  if (what == DEC_DUMP_TRACE) {
    if (!c->d_trace) return fail(c, DEC_ERR_STATE, "context created without DEC_FLAG_TRACE");
    unsigned long long hdr[2];
    CK(cudaMemcpy(hdr, c->d_trace, 16, cudaMemcpyDeviceToHost));
    const size_t nrec = std::min<size_t>((unsigned)hdr[0], (size_t)c->trace_cap);
    const size_t need = nrec * 48;
    if (out_bytes) *out_bytes = need;
    if (!dst) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    CK(cudaMemcpy(dst, c->d_trace + 2, need, cudaMemcpyDeviceToHost));
    return DEC_OK;
  }
  if (what == DEC_DUMP_TRACE_PRODUCER) {
    if (!c->d_trace) return fail(c, DEC_ERR_STATE, "context created without DEC_FLAG_TRACE");
    const size_t need = (size_t)c->trace_cap * 24;
    if (out_bytes) *out_bytes = need;
    if (!dst) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    CK(cudaMemcpy(dst, c->d_trace + 2 + 6 * (size_t)c->trace_cap, need, cudaMemcpyDeviceToHost));
    return DEC_OK;
  }
  if (what == DEC_DUMP_PLAN) {
    std::string s;
    char line[512];
    for (size_t i = 0; i < c->ops.size(); ++i) {
      const OpDesc& o = c->ops[i];
      snprintf(line, sizeof line,
               "%zu %s layer=%d kind=%d tasks=%d K=%d Kpad=%d kcb=%d R=%d S=%d nst=%d segs=%d dep=%d,%d pdep=%d nch=%d\n",
               i, c->op_names[i].c_str(), o.layer, o.kind, o.ntasks, o.K, o.Kpad, o.kcb, o.R, o.S, o.nst, o.nsegs,
               o.dep[0], o.dep[1], o.pdep, o.nch);
      s += line;
    }
    snprintf(line, sizeof line, "ctas=%d smem=%d stages=%d stage_bytes=%d\n", c->n_ctas, kSmemBytes, kStages,
             kStageBytes);
    s += line;
    if (out_bytes) *out_bytes = s.size() + 1;
    if (!dst) return DEC_OK;
    if (bytes < s.size() + 1) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", s.size() + 1);
    memcpy(dst, s.c_str(), s.size() + 1);
    return DEC_OK;
  }
  if (what == DEC_DUMP_STATUS) {
    static_assert(sizeof(Status) + sizeof(StepState) == 64, "status dump layout");
    const size_t need = sizeof(Status) + sizeof(StepState);
    if (out_bytes) *out_bytes = need;
    if (!dst) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    CK(cudaMemcpy(dst, c->d_status, sizeof(Status), cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(reinterpret_cast<uint8_t*>(dst) + sizeof(Status), c->d_state, sizeof(StepState),
                  cudaMemcpyDeviceToHost));
    return DEC_OK;
  }
  if (what == DEC_DUMP_WEIGHTS) {
    if (out_bytes) *out_bytes = 16;
    if (!dst) return DEC_OK;
    if (bytes < 16) return fail(c, DEC_ERR_INVALID_ARG, "dump needs 16 bytes");
    uint64_t v[2] = {c->weight_bytes_step, c->weight_bytes_stored};
    memcpy(dst, v, 16);
    return DEC_OK;
  }
  if (what >= DEC_DUMP_OP && what < DEC_DUMP_OP + (int)c->ops.size()) {
    const OpDesc& o = c->ops[what - DEC_DUMP_OP];
    std::vector<std::pair<const float*, size_t>> parts;
    if (o.kind == OP_GEMV) {
      parts.push_back({o.out, (size_t)o.S * o.out_stride});
    } else if (o.kind == OP_ATTN || o.kind == OP_MLA) {
      const int heads = o.kind == OP_ATTN ? o.hq : o.H, dim = o.kind == OP_ATTN ? o.hd : o.kvl;
      parts.push_back({o.m_out, (size_t)heads * o.nch});
      parts.push_back({o.l_out, (size_t)heads * o.nch});
      parts.push_back({o.o_out, (size_t)heads * o.nch * dim});
    }
    size_t need = 0;
    for (auto& p : parts) need += p.second * 4;
    if (out_bytes) *out_bytes = need;
    if (!dst) return DEC_OK;
    if (bytes < need) return fail(c, DEC_ERR_INVALID_ARG, "dump needs %zu bytes", need);
    uint8_t* o8 = reinterpret_cast<uint8_t*>(dst);
    for (auto& p : parts) {
      CK(cudaMemcpy(o8, p.first, p.second * 4, cudaMemcpyDeviceToHost));
      o8 += p.second * 4;
    }
    return DEC_OK;
  }
  return fail(c, DEC_ERR_INVALID_ARG, "unknown dump selector %d", what);
}
