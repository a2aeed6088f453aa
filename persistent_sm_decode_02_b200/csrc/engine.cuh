// Device engine of the decode step: tile tasks and the persistent scheduler.
//
// A CTA runs three warp roles:
//   * 8 consumer warps compute the tasks;
//   * 1 producer warp walks the CTA's task list and streams every task's bytes
//     (weights, KV rows) from HBM into a kStages-deep shared-memory ring with
//     1-D TMA bulk copies.  It never waits for activation dependencies
//     (weights are static), so the next tasks' weights are in flight while
//     the consumers wait for the previous layer; only routed-expert weights
//     wait, because their address comes from the router's top-k;
//   * 1 signaller warp publishes each finished task: it receives the task from
//     the consumers through a 16-slot mailbox guarded by mbarriers and does
//     the gpu-scope fence and counter release, off the consumers' path.
// Consumers wait on the dependency counters of the task's op (one thread polls,
// then a barrier), build the task's input vector in shared memory (norm /
// combine / SwiGLU prologue, once per op and input group), consume the ring
// stages and write fp32 partial outputs.  Op descriptors are staged in shared
// memory when the op changes; the next task-list entry is prefetched a task
// ahead.  Every wait is bounded by a global-timer deadline: on expiry the CTA
// records the failure in a status word, finishes the task it is in on stale
// data (so that every thread meets the same barriers), stops, and drains the
// copies still in flight.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "dec_types.h"
#include "ptx.cuh"

namespace dec {

constexpr int kMail = 16;  // mailbox slots between consumers and the signaller
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kSignalWarp = kConsumerWarps + 1;
constexpr int kOdBytes = (int)((sizeof(OpDesc) + 15) / 16 * 16);

struct Misc {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t sig_done[kMail];  // consumers -> signaller: task in mailbox slot finished (8 warp arrivals)
  uint64_t sig_free[kMail];  // signaller -> consumers: mailbox slot published and free again
  uint64_t mma_bar;          // tensor-core MMAs of the current MLA task completed (tcgen05.commit)
  uint64_t fin_bar;          // every MMA completed before TMEM is freed
  uint32_t tmem;             // TMEM base address (MLA engine instances)
  int prod_dep_op;           // op whose producer dependency the producer already waited for
  int last_task;             // the current task is the last of its op (router) or kv head (attention) to finish
  StepState st;
  volatile int abort;
  int x_op, x_group;     // identity of the input vector currently in the work area
  int consumed;          // ring stages consumed (consumer thread 0)
  int issued;            // ring stages issued (producer lane 0)
  int prod_route_op;     // router op whose top-k is in prod_idx
  int prod_idx[kMaxTopK];
  float cons_w[kMaxTopK];
  int mail_op[kMail], mail_task[kMail];
  unsigned long long mail_t[kMail][4];  // trace: task start, input vector ready, first stage available, compute done
  unsigned long long tr_pro;            // trace: when the current task's input vector was ready
  unsigned long long tr_data;           // trace: when the current task's first stage was available
  float red[256];
  unsigned long long redk[8];
};

constexpr int kRingBytes = kStages * kStageBytes;
constexpr int kSmemBytes = kRingBytes + kWorkBytes + 2 * kOdBytes + (int)sizeof(Misc);

struct Smem {
  uint8_t* ring;
  uint8_t* work;
  OpDesc* cod;  // consumers' copy of the current op descriptor
  OpDesc* pod;  // producer's copy
  Misc* m;
};

__device__ __forceinline__ Smem smem_layout(uint8_t* base) {
  Smem s;
  s.ring = base;
  s.work = base + kRingBytes;
  s.cod = reinterpret_cast<OpDesc*>(base + kRingBytes + kWorkBytes);
  s.pod = reinterpret_cast<OpDesc*>(base + kRingBytes + kWorkBytes + kOdBytes);
  s.m = reinterpret_cast<Misc*>(base + kRingBytes + kWorkBytes + 2 * kOdBytes);
  return s;
}

// Copy an op descriptor from global to shared memory (nthr threads with ids 0..nthr-1).
__device__ __forceinline__ void copy_od(OpDesc* dst, const OpDesc* src, int id, int nthr) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int i = id; i < kOdBytes / 16; i += nthr) d[i] = __ldg(s + i);
}

// ------------------------------------------------------------ error / waits
__device__ __forceinline__ void report_timeout(const KParams& P, int op, int task) {
  if (atomicCAS(&P.status->code, 0, 1) == 0) {
    P.status->cta = blockIdx.x;
    P.status->op = op;
    P.status->task = task;
  }
}

// A router or LM-head logit is NaN or infinite (a corrupt weight or activation): the
// step's greedy token and expert choice are meaningless.  Recorded like a timeout, so
// the other CTAs' cross-CTA waits stop early and the host poisons the context.
__device__ __noinline__ void report_nonfinite(const KParams& P, int op, int task) {
  if (atomicCAS(&P.status->code, 0, 2) == 0) {
    P.status->cta = blockIdx.x;
    P.status->op = op;
    P.status->task = task;
  }
}

// true unless v is an infinity or a NaN (all exponent bits set), tested on the bits
__device__ __forceinline__ bool finite_bits(float v) { return (__float_as_uint(v) & 0x7F800000u) != 0x7F800000u; }

// Spin until ready(); false if this CTA gave up (deadline passed or the CTA's
// abort flag set).  Waits on another CTA (cross_cta) also watch the global status
// word, so that a failure anywhere stops them; waits inside the CTA only read
// the CTA's own flag (many threads spin on those: they must not load global
// memory while they wait).
template <class F>
__device__ __forceinline__ bool bounded_wait(F ready, const KParams& P, volatile int* abort, int op, int task,
                                             bool cross_cta) {
  if (ready()) return true;
  const uint64_t t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
    if (ready()) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (cross_cta && ld_volatile_int(&P.status->code) != 0) {
        *abort = 1;
        return false;
      }
      if (globaltimer() - t0 > P.timeout_ns) {
        report_timeout(P, op, task);
        *abort = 1;
        return false;
      }
    }
    if (cross_cta) __nanosleep(64);
  }
}

__device__ __forceinline__ bool wait_counter(const KParams& P, int dop, unsigned epoch, volatile int* abort,
                                             int op, int task) {
  if (dop < 0) return true;
  const unsigned target = epoch * (unsigned)__ldg(&P.ops[dop].ntasks);
  const unsigned* c = &P.counters[dop];
  return bounded_wait([&] { return (int)(ld_acquire_gpu(c) - target) >= 0; }, P, abort, op, task, true);
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t par, const KParams& P, volatile int* abort,
                                          int op, int task) {
  return bounded_wait([&] { return mbar_try_wait(bar, par); }, P, abort, op, task, false);
}

// ------------------------------------------------------- block reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over the 256 consumer threads (all must call).
__device__ __forceinline__ float consumer_sum(float v, Misc* m) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  v = warp_sum(v);
  if (lane == 0) m->red[w] = v;
  named_bar_sync(1, kConsumers);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kConsumerWarps; ++i) s += m->red[i];
  named_bar_sync(1, kConsumers);
  return s;
}

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float pset(const PSet& p, int e) {
  float v = 0.f;
  for (int s = 0; s < p.S; ++s) v += ldcg(p.ptr + (size_t)s * p.stride + p.off + e);
  return v;
}

__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void add4(float4& a, const float4 b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}
__device__ __forceinline__ void fma4(float4& a, float w, const float4 b) {
  a.x = fmaf(w, b.x, a.x);
  a.y = fmaf(w, b.y, a.y);
  a.z = fmaf(w, b.z, a.z);
  a.w = fmaf(w, b.w, a.w);
}

// Sum over splits of 4 consecutive elements (e multiple of 4, offsets 16-byte aligned).
__device__ __forceinline__ float4 pset4(const PSet& p, int e) {
  const float* b = p.ptr + p.off + e;
  float4 v = ldcg4(b);  // first split unconditionally, so callers' loads can be issued together
  for (int s = 1; s < p.S; ++s) add4(v, ldcg4(b + (size_t)s * p.stride));
  return v;
}

__device__ __forceinline__ float rnd(float v, int bf16) { return bf16 ? bf16_round(v) : v; }

__device__ __forceinline__ void store_x(uint8_t* work, int in_bf16, int e, float v) {
  if (in_bf16)
    reinterpret_cast<__nv_bfloat16*>(work)[e] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(work)[e] = v;
}

// Four consecutive input elements (e multiple of 4), rounded to the input dtype.
__device__ __forceinline__ void store_x4(uint8_t* work, int in_bf16, int e, float4 v) {
  if (in_bf16) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(work + 2 * e) = u;
  } else {
    *reinterpret_cast<float4*>(work + 4 * e) = v;
  }
}

// Router logits: sum of the S split-K partials of each of E experts, in split order, one
// expert per consumer thread (its S loads in flight together).  Out of line: it runs once per
// MoE layer and must not add to the register budget of the hot loops.
__device__ __noinline__ void router_sum(const float* out, int S, int stride, int E, float* dst) {
  for (int e = threadIdx.x; e < E; e += kConsumers) {
    float v = 0.f;
    for (int s0 = 0; s0 < S; ++s0) v += ldcg(out + (size_t)s0 * stride + e);
    dst[e] = v;
  }
}

// Softmax top-k router (one warp, all 32 lanes call) over E <= 256 summed logits in
// shared memory: pick the k largest logits,
// ties to the lower expert id, weights renormalised over the chosen k:
// w_j = exp(r_j - r_max) / sum_i exp(r_i - r_max).  Returns false (every lane) if
// any logit is NaN or infinite; the ids and weights are then still written.
__device__ __forceinline__ bool warp_route(const float* logits, int E, int k, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  int taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = lane + 32 * i < E ? logits[lane + 32 * i] : 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (lane + 32 * i >= E)
      v[i] = -INFINITY;
    else
      bad |= !finite_bits(v[i]);
  }
  bad = __any_sync(0xffffffffu, bad);
  float top[kMaxTopK];
  int id[kMaxTopK];
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1) && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= E) {  // only reachable with NaN logits (reported): fall back to id 0
      bi = 0;
      bv = -INFINITY;
    }
    if ((bi & 31) == lane) taken |= 1 << (bi >> 5);
    top[j] = bv;
    id[j] = bi;
  }
  float den = 0.f;
  for (int j = 0; j < k; ++j) den += expf(top[j] - top[0]);
  if (!(den > 0.f)) den = 1.f;
  if (lane == 0) {
    for (int j = 0; j < k; ++j) {
      if (idx_out) idx_out[j] = id[j];
      if (w_out) w_out[j] = expf(top[j] - top[0]) / den;
    }
  }
  __syncwarp();
  return !bad;
}

// ------------------------------------------------------------- prologues
// Every prologue reads its sources with 16-byte loads, several independent
// loads in flight per thread, so it is bound by L2 bandwidth, not latency.
constexpr int kMaxQ = kMaxD / 4 / kConsumers;  // float4 chunks per thread for vectors <= kMaxD
constexpr int kSrcBatch = 2;                    // residual sources loaded together

// Split-KV log-sum-exp weights of one head: w_c = e^(m_c - M) / sum_c e^(m_c - M) l_c over
// the chunks with data (l_c > 0), M = max m_c.  One warp; stores nch weights.
__device__ __forceinline__ void combine_weights(const float* am, const float* al, int nch, float* w) {
  const int lane = threadIdx.x & 31;
  float M = -INFINITY;
  for (int c = lane; c < nch; c += 32)
    if (ldcg(al + c) > 0.f) M = fmaxf(M, ldcg(am + c));
  M = warp_max(M);
  float den = 0.f;
  for (int c = lane; c < nch; c += 32) {
    const float l = ldcg(al + c);
    const float e = l > 0.f ? expf(ldcg(am + c) - M) : 0.f;  // empty chunks (l = 0) get weight 0
    den += e * l;
    w[c] = e;
  }
  den = warp_sum(den);
  const float inv = den > 0.f ? 1.0f / den : 0.f;
  __syncwarp();
  for (int c = lane; c < nch; c += 32) w[c] *= inv;
}

// Build the input vector of (op, group) in the work area, all 256 consumer threads.
__device__ __forceinline__ void prologue(const OpDesc& od, int group, int task, const Smem& S) {
  Misc* m = S.m;
  const int tid = threadIdx.x;
  uint8_t* x = S.work;
  const int n = od.n;
  const int bf = od.in_bf16;
  switch (od.pro) {
    case PRO_RESID_NORM:
    case PRO_NORM_SUM: {
      const bool resid = od.pro == PRO_RESID_NORM;
      if (resid && od.routed.ptr) {
        if (tid < od.top_k) m->cons_w[tid] = __ldcg(od.rt_w + tid);  // written by the router's last task
        named_bar_sync(1, kConsumers);
      }
      float4 v[kMaxQ];
      // The gains (often read from HBM) are copied asynchronously into the work area
      // behind the input vector, so their latency overlaps the base and source loads;
      // each thread later reads back only the chunks it copied itself.
      const int goff = ((od.Kpad * (bf ? 2 : 4)) + 15) & ~15;
      float* gs = reinterpret_cast<float*>(S.work + goff);
      const bool stage_g = goff + 4 * n <= kWorkBytes;
      if (stage_g) {
        for (int e = 4 * tid; e < n; e += 4 * kConsumers) cp_async16(gs + e, od.gain + e);
        cp_async_commit();
      }
      // base
#pragma unroll
      for (int i = 0; i < kMaxQ; ++i) {
        const int e = 4 * (tid + i * kConsumers);
        v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < n) {
          if (!resid) {
            v[i] = pset4(od.src, e);
          } else if (od.base_embed) {
            const size_t row = (size_t)m->st.tok * n;
            if (od.embed_bf16) {
              const uint2 u = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(od.embed) + row + e));
              v[i] = make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
            } else {
              v[i] = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(od.embed) + row + e));
            }
          } else {
            v[i] = ldcg4(od.h_base + e);
          }
        }
      }
      if (resid) {
        // Added sources: every split of `add` and `add2` (weight 1) and of each routed
        // expert slot j (weight w_j).  kSrcBatch sources are loaded per batch so
        // that each thread has up to kSrcBatch * kMaxQ 16-byte loads in flight.
        const int na = od.add.ptr ? od.add.S : 0, nb = od.add2.ptr ? od.add2.S : 0;
        const int nr = od.routed.ptr ? od.top_k * od.routed.S : 0;
        const int nsrc = na + nb + nr;
        auto src = [&](int k, float& wk) -> const float* {
          wk = 1.f;
          if (k < na) return od.add.ptr + od.add.off + (size_t)k * od.add.stride;
          k -= na;
          if (k < nb) return od.add2.ptr + od.add2.off + (size_t)k * od.add2.stride;
          k -= nb;
          const int j = k / od.routed.S, s = k % od.routed.S;
          wk = m->cons_w[j];
          return od.routed.ptr + od.routed.off + (size_t)j * od.routed_slot_stride + (size_t)s * od.routed.stride;
        };
        for (int k0 = 0; k0 < nsrc; k0 += kSrcBatch) {
          float w3[kSrcBatch];
          const float* p3[kSrcBatch];
          float4 u[kSrcBatch][kMaxQ];
#pragma unroll
          for (int b = 0; b < kSrcBatch; ++b) {
            p3[b] = k0 + b < nsrc ? src(k0 + b, w3[b]) : nullptr;
            if (!p3[b]) w3[b] = 0.f;
          }
#pragma unroll
          for (int b = 0; b < kSrcBatch; ++b)
#pragma unroll
            for (int i = 0; i < kMaxQ; ++i) {
              const int e = 4 * (tid + i * kConsumers);
              u[b][i] = (p3[b] && e < n) ? ldcg4(p3[b] + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
          for (int b = 0; b < kSrcBatch; ++b)
#pragma unroll
            for (int i = 0; i < kMaxQ; ++i) fma4(v[i], w3[b], u[b][i]);  // w = 1: exact add
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxQ; ++i) ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
      if (stage_g) cp_async_wait_all();
      const float tot = consumer_sum(ss, m);
      const float inv = 1.0f / sqrtf(tot / (float)n + od.eps);
#pragma unroll
      for (int i = 0; i < kMaxQ; ++i) {
        const int e = 4 * (tid + i * kConsumers);
        if (e < n) {
          const float4 g = stage_g ? *reinterpret_cast<const float4*>(gs + e)
                                   : __ldg(reinterpret_cast<const float4*>(od.gain + e));
          float4 y;
          y.x = v[i].x * inv * g.x;
          y.y = v[i].y * inv * g.y;
          y.z = v[i].z * inv * g.z;
          y.w = v[i].w * inv * g.w;
          store_x4(x, bf, e, y);
          if (resid && od.h_out && task == 0) *reinterpret_cast<float4*>(od.h_out + e) = v[i];
        }
      }
      break;
    }
    case PRO_SUM: {
      PSet p = od.src;
      p.off += group * od.gstride;
      for (int e0 = 4 * tid; e0 < n; e0 += 4 * 4 * kConsumers) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * 4 * kConsumers;
          if (e < n) v[u] = pset4(p, e);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * 4 * kConsumers;
          if (e < n) store_x4(x, bf, e, v[u]);
        }
      }
      break;
    }
    case PRO_SWIGLU: {
      PSet gp = od.gate, up = od.up;
      gp.off += group * od.slot_stride;
      up.off += group * od.slot_stride;
      for (int e0 = 4 * tid; e0 < n; e0 += 4 * 4 * kConsumers) {
        float4 gv[4], uv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * 4 * kConsumers;
          if (e < n) {
            gv[u] = pset4(gp, e);
            uv[u] = pset4(up, e);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = e0 + u * 4 * kConsumers;
          if (e < n) {
            float4 y;
            y.x = gv[u].x / (1.0f + expf(-gv[u].x)) * uv[u].x;
            y.y = gv[u].y / (1.0f + expf(-gv[u].y)) * uv[u].y;
            y.z = gv[u].z / (1.0f + expf(-gv[u].z)) * uv[u].z;
            y.w = gv[u].w / (1.0f + expf(-gv[u].w)) * uv[u].w;
            store_x4(x, bf, e, y);
          }
        }
      }
      break;
    }
    case PRO_MLA_COMBINE: {
      // per-chunk weights of the group's head, then the weighted sum of its chunk outputs
      const int h0 = group, nh = 1;
      float* wt = reinterpret_cast<float*>(S.work + kCombineOff);  // [nh][nch]
      const int warp = tid >> 5;
      const int hd = od.hdim;
      // MLA blocks past position pos hold no partials
      const int nc = min(od.nch, m->st.pos / kMlaBlock + 1);
      if (n == 4 * kConsumers / 2 && hd == n) {
        // One head of 512 columns: each half of the threads sums half of the blocks for its
        // 4 columns (the first kB partial loads issued before the combine weights are known),
        // and the two halves meet in shared memory.
        constexpr int kB = 9;
        const int hf = tid / (kConsumers / 2), e = 4 * (tid % (kConsumers / 2));
        const int mid = (nc + 1) / 2, cb = hf ? mid : 0, ce = hf ? nc : mid;
        const float* src = od.ao + (size_t)h0 * od.nch * hd + e;
        float4 a[kB];
#pragma unroll
        for (int b = 0; b < kB; ++b) a[b] = cb + b < ce ? ldcg4(src + (size_t)(cb + b) * hd) : make_float4(0.f, 0.f, 0.f, 0.f);
        if (warp == 0) combine_weights(od.am + (size_t)h0 * od.nch, od.al + (size_t)h0 * od.nch, od.nch, wt);
        named_bar_sync(1, kConsumers);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = cb; c0 < ce; c0 += kB) {
          if (c0 != cb)
#pragma unroll
            for (int b = 0; b < kB; ++b)
              a[b] = c0 + b < ce ? ldcg4(src + (size_t)(c0 + b) * hd) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int b = 0; b < kB; ++b)
            if (c0 + b < ce) fma4(acc, wt[c0 + b], a[b]);
        }
        float4* other = reinterpret_cast<float4*>(S.work + kCombineOff) + 64;  // behind the weights
        if (hf) other[tid % (kConsumers / 2)] = acc;
        named_bar_sync(1, kConsumers);
        if (!hf) {
          const float4 o2 = other[tid];
          acc.x += o2.x;
          acc.y += o2.y;
          acc.z += o2.z;
          acc.w += o2.w;
          store_x4(x, bf, e, acc);
        }
        break;
      }
      for (int h = warp; h < nh; h += kConsumerWarps)
        combine_weights(od.am + (size_t)(h0 + h) * od.nch, od.al + (size_t)(h0 + h) * od.nch, od.nch,
                        wt + h * od.nch);
      named_bar_sync(1, kConsumers);
      for (int e = 4 * tid; e < n; e += 4 * kConsumers) {
        const int h = e / hd, d = e % hd;
        const float* w = wt + h * od.nch;
        const float* src = od.ao + ((size_t)(h0 + h) * od.nch) * hd + d;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int c = 0;
        for (; c + 4 <= nc; c += 4) {
          const float4 a0 = ldcg4(src + (size_t)c * hd), a1 = ldcg4(src + (size_t)(c + 1) * hd);
          const float4 a2 = ldcg4(src + (size_t)(c + 2) * hd), a3 = ldcg4(src + (size_t)(c + 3) * hd);
          fma4(acc, w[c], a0);
          fma4(acc, w[c + 1], a1);
          fma4(acc, w[c + 2], a2);
          fma4(acc, w[c + 3], a3);
        }
        for (; c < nc; ++c) fma4(acc, w[c], ldcg4(src + (size_t)c * hd));
        store_x4(x, bf, e, acc);
      }
      break;
    }
    default:
      break;
  }
  // zero padding up to Kpad (n and Kpad are multiples of 4)
  for (int e = n + 4 * tid; e < od.Kpad; e += 4 * kConsumers) store_x4(x, bf, e, make_float4(0.f, 0.f, 0.f, 0.f));
  named_bar_sync(1, kConsumers);
}

// ------------------------------------------------------------ GEMV tasks
struct TaskGeo {
  int si, rt, s, group;
};

__device__ __forceinline__ TaskGeo gemv_geo(const OpDesc& od, int t) {
  TaskGeo g;
  int si = 0;
  while (si + 1 < od.nsegs && t >= od.seg[si + 1].task0) ++si;
  const Seg& sg = od.seg[si];
  const int local = t - sg.task0;
  g.si = si;
  g.rt = local / od.S;
  g.s = local % od.S;
  g.group = sg.in_group >= 0 ? sg.in_group : (od.rows_per_group ? (g.rt * od.R) / od.rows_per_group : 0);
  return g;
}

__device__ __forceinline__ void wait_full(const KParams& P, const Smem& S, uint32_t g, int op, int task) {
  mbar_wait(&S.m->full[g % kStages], (g / kStages) & 1, P, &S.m->abort, op, task);
}

__device__ __forceinline__ void release_stage(const Smem& S, uint32_t g) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&S.m->empty[g % kStages]);
}

// Order-preserving key of (logit, index): larger logit wins, then the smaller index.
// The bits are taken through an opaque move so that the sign-bit or/xor below stays
// integer work: written on a plain bitcast, the compiler may turn it into float
// negate/absolute-value, whose result for a NaN input is an unspecified NaN, and a NaN
// logit must keep its all-ones key for the final op to see it.
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t u;
  asm("mov.b32 %0, %1;" : "=r"(u) : "f"(v));
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

// This thread's 16-byte chunks of a ring stage: chunk c of rows rg, rg + G, ... (rpt rows).
// They are taken into registers first so that the stage can go back to the producer before
// the arithmetic: the slot's next copy then overlaps this stage's compute.
template <int RPT>
__device__ __forceinline__ void gemv_load(const uint8_t* stage, int kcb, int G, int rpt, int c, int rg, uint4* wv) {
#pragma unroll
  for (int i = 0; i < RPT; ++i)
    if (i < rpt) wv[i] = *reinterpret_cast<const uint4*>(stage + (rg + G * i) * kcb + c * 16);
}

template <int WT, int RPT>
__device__ __forceinline__ void gemv_stage(const uint4* wv, const uint8_t* x, int k0, int rpt, int c, float scale,
                                           float* acc) {
  if constexpr (WT == WT_FP8) {
    const uint4* xv = reinterpret_cast<const uint4*>(x + 2 * (k0 + c * 16));
    const uint4 xa = xv[0], xb = xv[1];
    float xf[16];
    const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      xf[2 * i] = bf16lo(xw[i]);
      xf[2 * i + 1] = bf16hi(xw[i]);
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (i >= rpt) break;
      const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
      float part = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 lo = __half22float2(e4m3x2_to_half2((uint16_t)(ww[q] & 0xFFFF)));
        const float2 hi = __half22float2(e4m3x2_to_half2((uint16_t)(ww[q] >> 16)));
        part = fmaf(lo.x, xf[4 * q + 0], part);
        part = fmaf(lo.y, xf[4 * q + 1], part);
        part = fmaf(hi.x, xf[4 * q + 2], part);
        part = fmaf(hi.y, xf[4 * q + 3], part);
      }
      acc[i] = fmaf(scale, part, acc[i]);
    }
  } else if constexpr (WT == WT_BF16) {
    const uint4 xa = *reinterpret_cast<const uint4*>(x + 2 * (k0 + c * 8));
    const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w};
    float xf[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xf[2 * i] = bf16lo(xw[i]);
      xf[2 * i + 1] = bf16hi(xw[i]);
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (i >= rpt) break;
      const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
      float a = acc[i];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a = fmaf(bf16lo(ww[q]), xf[2 * q], a);
        a = fmaf(bf16hi(ww[q]), xf[2 * q + 1], a);
      }
      acc[i] = a;
    }
  } else {
    const float4 xa = *reinterpret_cast<const float4*>(x + 4 * (k0 + c * 4));
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (i >= rpt) break;
      const float4 w4 = make_float4(__uint_as_float(wv[i].x), __uint_as_float(wv[i].y), __uint_as_float(wv[i].z),
                                    __uint_as_float(wv[i].w));
      float a = acc[i];
      a = fmaf(w4.x, xa.x, a);
      a = fmaf(w4.y, xa.y, a);
      a = fmaf(w4.z, xa.z, a);
      a = fmaf(w4.w, xa.w, a);
      acc[i] = a;
    }
  }
}

// One GEMV task, geometry fixed at compile time by the stage's bytes per row
// (KCB): CPR 16-byte chunks per row, G row groups, RPT rows per thread.
template <int WT, int KCB>
__device__ __forceinline__ void gemv_task(const KParams& P, const OpDesc& od, int op, int t, const Smem& S,
                                          uint32_t& g, const TaskGeo& geo) {
  constexpr int CPR = KCB / 16, G = kConsumers / CPR, RPT = gemv_rows_per_thread(KCB), R = G * RPT;
  constexpr int SPAN = CPR < 32 ? CPR : 32, PARTS = CPR / SPAN;
  constexpr int KC = KCB / (WT == WT_FP8 ? 1 : WT == WT_BF16 ? 2 : 4);
  const Seg& sg = od.seg[geo.si];
  Misc* m = S.m;
  const int tid = threadIdx.x;
  const int c = tid % CPR, rg = tid / CPR;
  const int nst = od.nst;
  float acc[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) acc[i] = 0.f;
  const float* sc = nullptr;
  const int nkb = (od.K + 127) / 128;
  if constexpr (WT == WT_FP8) {
    sc = sg.sc + (size_t)((geo.rt * R) / 128) * nkb;
    if (sg.slot >= 0) sc += (size_t)m->prod_idx[sg.slot] * sg.s_estride;  // read after the first stage landed
  }
  for (int st = 0; st < nst; ++st) {
    wait_full(P, S, g, op, t);  // on failure the task runs to its end on stale data; the caller stops after it
    if (P.trace && st == 0 && tid == 0) m->tr_data = globaltimer();
    const uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    const int k0 = (geo.s * nst + st) * KC;
    float scale = 1.f;
    if constexpr (WT == WT_FP8) {
      if (st == 0 && sg.slot >= 0) {  // the producer wrote the expert id before this stage's copy
        sc = sg.sc + (size_t)((geo.rt * R) / 128) * nkb + (size_t)m->prod_idx[sg.slot] * sg.s_estride;
      }
      const int cb = (k0 + c * 16) >> 7;
      scale = cb < nkb ? __ldg(sc + cb) : 0.f;
    }
    uint4 wv[RPT];
    gemv_load<RPT>(stage, KCB, G, RPT, c, rg, wv);
    release_stage(S, g);
    gemv_stage<WT, RPT>(wv, S.work, k0, RPT, c, scale, acc);
    ++g;
  }
  // reduce the CPR partials of every row
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = SPAN >> 1; o > 0; o >>= 1)
#pragma unroll
    for (int i = 0; i < RPT; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (PARTS == 1 && !od.best) {
    // a row's chunks all live in one warp: its first lane holds the row sum, no CTA barrier needed
    if ((lane & (SPAN - 1)) == 0) {
      float* out = od.out + (size_t)geo.s * od.out_stride + sg.out_off;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int row = geo.rt * R + rg + G * i;
        if (row < sg.N) {
          out[row] = acc[i];
          if (od.qc)
            reinterpret_cast<__nv_bfloat16*>(od.qc)[mla_q_off(row / od.rows_per_group, row % od.rows_per_group) / 2] =
                __float2bfloat16_rn(acc[i]);
        }
      }
    }
    return;
  }
  if ((lane & (SPAN - 1)) == 0) {
    const int part = CPR >= 32 ? (warp * 32 % CPR) / 32 : 0;
#pragma unroll
    for (int i = 0; i < RPT; ++i) m->red[(i * G + rg) * PARTS + part] = acc[i];
  }
  named_bar_sync(1, kConsumers);
  unsigned long long key = 0ull;
  if (tid < R) {
    const int i = tid / G, rg2 = tid % G;
    float y = 0.f;
#pragma unroll
    for (int p = 0; p < PARTS; ++p) y += m->red[(i * G + rg2) * PARTS + p];
    const int row = geo.rt * R + tid;
    if (row < sg.N) {
      od.out[(size_t)geo.s * od.out_stride + sg.out_off + row] = y;
      if (od.qc)
        reinterpret_cast<__nv_bfloat16*>(od.qc)[mla_q_off(row / od.rows_per_group, row % od.rows_per_group) / 2] =
            __float2bfloat16_rn(y);
      if (od.best) key = argmax_key(y, sg.out_off + row);
    }
  }
  if (od.best) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, o);
      key = ok > key ? ok : key;
    }
    if (lane == 0) m->redk[warp] = key;
    named_bar_sync(1, kConsumers);
    if (tid == 0) {
      unsigned long long b = 0ull;
      for (int w = 0; w < kConsumerWarps; ++w) b = m->redk[w] > b ? m->redk[w] : b;
      od.best[t] = b;
    }
  }
}

// MLA: the step's new latent cache row, c = bf16(RMSNorm(kv_a latent) * g) and
// k_pe = bf16(RoPE(kv_a rope part)), stored at position pos of the blocked cache
// (all consumer threads; absorb_q's extra last task, before attention reads the block).
__device__ __forceinline__ void mla_new_row(const OpDesc& od, const Smem& S) {
  Misc* m = S.m;
  const int tid = threadIdx.x, pos = m->st.pos;
  const int kvl = od.rows_per_group, rd = od.rdim, rowe = kvl + rd;
  __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(S.work + kCombineOff);  // [rowe]
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (4 * tid < kvl) v = pset4(od.ckv, 4 * tid);  // 16-byte loads of the split partials
  const float tot = consumer_sum(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w, m);
  const float inv = 1.0f / sqrtf(tot / (float)kvl + od.eps);
  if (4 * tid < kvl) {
    const float4 g4 = __ldg(reinterpret_cast<const float4*>(od.kvnorm_g + 4 * tid));
    reinterpret_cast<__nv_bfloat162*>(row)[2 * tid] = __floats2bfloat162_rn(v.x * inv * g4.x, v.y * inv * g4.y);
    reinterpret_cast<__nv_bfloat162*>(row)[2 * tid + 1] = __floats2bfloat162_rn(v.z * inv * g4.z, v.w * inv * g4.w);
  }
  const int rq = tid - kvl / 4;  // RoPE: 4 pairs (j, j + rd/2) per thread
  if (rq >= 0 && 4 * rq < rd / 2) {
    const int j = 4 * rq;
    const float4 a = pset4(od.ckv, kvl + j), b = pset4(od.ckv, kvl + j + rd / 2);
    const float4 cs = __ldg(reinterpret_cast<const float4*>(od.rope_cos + (size_t)pos * (rd / 2) + j));
    const float4 sn = __ldg(reinterpret_cast<const float4*>(od.rope_sin + (size_t)pos * (rd / 2) + j));
    __nv_bfloat162* lo = reinterpret_cast<__nv_bfloat162*>(row + kvl + j);
    __nv_bfloat162* hi = reinterpret_cast<__nv_bfloat162*>(row + kvl + j + rd / 2);
    lo[0] = __floats2bfloat162_rn(a.x * cs.x - b.x * sn.x, a.y * cs.y - b.y * sn.y);
    lo[1] = __floats2bfloat162_rn(a.z * cs.z - b.z * sn.z, a.w * cs.w - b.w * sn.w);
    hi[0] = __floats2bfloat162_rn(a.x * sn.x + b.x * cs.x, a.y * sn.y + b.y * cs.y);
    hi[1] = __floats2bfloat162_rn(a.z * sn.z + b.z * cs.z, a.w * sn.w + b.w * cs.w);
  }
  named_bar_sync(1, kConsumers);
  uint8_t* blk = reinterpret_cast<uint8_t*>(od.kcache) + (size_t)(pos / kMlaBlock) * rowe * kMlaBlock * 2;
  for (int k = tid; k < rowe / 8; k += kConsumers)
    *reinterpret_cast<uint4*>(blk + mla_cache_off(pos % kMlaBlock, 8 * k)) = reinterpret_cast<const uint4*>(row)[k];
}

template <int WT>
__device__ __forceinline__ void gemv_unit(const KParams& P, const OpDesc& od, int op, int u, const Smem& S,
                                          uint32_t& g, const TaskGeo& geo) {
  switch (od.kcb) {
    case 4096: gemv_task<WT, 4096>(P, od, op, u, S, g, geo); break;
    case 2048: gemv_task<WT, 2048>(P, od, op, u, S, g, geo); break;
    case 1024: gemv_task<WT, 1024>(P, od, op, u, S, g, geo); break;
    case 512: gemv_task<WT, 512>(P, od, op, u, S, g, geo); break;
    case 256: gemv_task<WT, 256>(P, od, op, u, S, g, geo); break;
    case 128: gemv_task<WT, 128>(P, od, op, u, S, g, geo); break;
    case 64: gemv_task<WT, 64>(P, od, op, u, S, g, geo); break;
    default: gemv_task<WT, 32>(P, od, op, u, S, g, geo); break;
  }
}

template <int WT>
__device__ __forceinline__ void gemv_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S,
                                             uint32_t& g) {
  Misc* m = S.m;
  if (od.qc && t == od.ntasks - 1) {  // absorb_q's extra task: the step's latent cache row
    mla_new_row(od, S);
    fence_async_global();  // read by bulk copies of other CTAs after the op's counter
    return;
  }
  const int tpt = od.tpt > 1 ? od.tpt : 1;
  for (int i = 0; i < tpt; ++i) {  // a task's units (row tiles) share the input group
  const int u = t * tpt + i;
  const TaskGeo geo = gemv_geo(od, u);
  if (m->x_op != op || m->x_group != geo.group) {
    prologue(od, geo.group, u, S);
    if (threadIdx.x == 0) {
      m->x_op = op;
      m->x_group = geo.group;
      if (P.trace && i == 0) m->tr_pro = globaltimer();
    }
  }
  gemv_unit<WT>(P, od, op, u, S, g, geo);
  if (od.router) {
    // The task that finishes the router op last sums the logits' split-K
    // partials and stores the top-k ids and weights once for all readers.
    __threadfence();
    named_bar_sync(1, kConsumers);
    if (threadIdx.x == 0) {
      const unsigned prev = atomicAdd(od.fin, 1u);
      m->last_task = prev + 1 == (unsigned)m->st.epoch * (unsigned)od.ntasks;
    }
    named_bar_sync(1, kConsumers);
    if (m->last_task) {
      __threadfence();
      // every consumer thread sums one expert's split-K partials, in split order (all of them
      // in flight at once); one warp then takes the top-k from shared memory
      router_sum(od.out, od.S, od.out_stride, od.n_experts, m->red);
      named_bar_sync(1, kConsumers);
    }
    if (m->last_task && threadIdx.x < 32) {
      if (!warp_route(m->red, od.n_experts, od.top_k, od.rt_ids, od.rt_w) && threadIdx.x == 0)
        report_nonfinite(P, op, t);
      if (od.route_dump && threadIdx.x < od.top_k) od.route_dump[threadIdx.x] = __ldcg(od.rt_ids + threadIdx.x);
    }
  }
  if (od.qc) {
    // absorb_q also feeds the tensor-core MLA attention: gemv_task stored q_lat
    // rows in bf16; the first tile of head h adds its RoPE'd q_pe (bf16).
    if (geo.s == 0 && (geo.rt * od.R) % od.rows_per_group == 0) {
      const int h = geo.rt * od.R / od.rows_per_group, rd = od.rdim, kvl = od.rows_per_group;
      const int pos = m->st.pos;
      __nv_bfloat16* q = reinterpret_cast<__nv_bfloat16*>(od.qc);
      for (int j = threadIdx.x; j < rd / 2; j += kConsumers) {
        const float a = pset(od.src, h * od.gstride + od.nope + j), b = pset(od.src, h * od.gstride + od.nope + j + rd / 2);
        const float cs = od.rope_cos[(size_t)pos * (rd / 2) + j], sn = od.rope_sin[(size_t)pos * (rd / 2) + j];
        q[mla_q_off(h, kvl + j) / 2] = __float2bfloat16_rn(a * cs - b * sn);
        q[mla_q_off(h, kvl + j + rd / 2) / 2] = __float2bfloat16_rn(a * sn + b * cs);
      }
    }
  }
  }  // units
  if (od.qc) fence_async_global();  // Qc is read by bulk copies of other CTAs after the op's counter
}

// ------------------------------------------------------- attention tasks
struct ChunkB {
  int t0, t1, tc;  // chunk [t0, t1) of positions 0..pos; cached part [t0, tc)
  bool has_new;
};

__device__ __forceinline__ ChunkB chunk_bounds(int c, int nch, int pos) {
  ChunkB b;
  const int T = pos + 1;
  b.t0 = (int)(((long long)c * T) / nch);
  b.t1 = (int)(((long long)(c + 1) * T) / nch);
  b.tc = b.t1 < pos ? b.t1 : pos;
  if (b.tc < b.t0) b.tc = b.t0;
  b.has_new = b.t1 == T && b.t0 < b.t1;
  return b;
}

// Dense GQA split-KV attention: task = (kv head, position chunk c), all gs query heads of
// the kv head (GQA: query head i reads kv head i * hkv / hq).  Each head keeps a running
// (max m, sum l, weighted values o) over the chunk (online softmax, Milakov & Gimelshein
// 2018) and publishes them for the log-sum-exp combine in the output projection's prologue.
// Work split, so that the chunk streams at the ring's rate on CUDA cores: warp w takes
// positions w, w + 8, ... of every ring stage; lane l holds dims [dpl l, dpl l + dpl) of
// the G (gs rounded up to a power of two) query heads.  Per position the G partial dot
// products are reduced over the warp by one multi-value butterfly (after it, lane l holds
// the full score of one head), the G scores are broadcast, and every lane updates its
// warp's state with base-2 exponentials.  The 8 warps' states merge once per task.
template <int G>
__device__ __forceinline__ float group_reduce(float (&v)[G], int lane) {
#pragma unroll
  for (int cnt = G, b = 16; cnt > 1; cnt >>= 1, b >>= 1) {
    const bool up = (lane & b) != 0;
#pragma unroll
    for (int i = 0; i < cnt / 2; ++i) {
      const float send = up ? v[i] : v[i + cnt / 2];
      const float keep = up ? v[i + cnt / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, b);
    }
  }
  constexpr int kLog = G >= 8 ? 3 : G >= 4 ? 2 : G >= 2 ? 1 : 0;
#pragma unroll
  for (int b = 16 >> kLog; b >= 1; b >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], b);
  return v[0];
}

// Lane that holds head h's score after group_reduce<G>.
template <int G>
__device__ __forceinline__ int group_holder(int h) {
  constexpr int kLog = G >= 8 ? 3 : G >= 4 ? 2 : G >= 2 ? 1 : 0;
  int lane = 0;
#pragma unroll
  for (int k = 0; k < kLog; ++k) lane |= ((h >> (kLog - 1 - k)) & 1) << (4 - k);
  return lane;
}

template <int DPL>
__device__ __forceinline__ void load_dims(const uint8_t* row, int cbf, int lane, float (&x)[DPL]) {
  if (cbf) {
    if constexpr (DPL == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(row + lane * 8);
      x[0] = bf16lo(u.x);
      x[1] = bf16hi(u.x);
      x[2] = bf16lo(u.y);
      x[3] = bf16hi(u.y);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 4);
      x[0] = bf16lo(u);
      x[1] = bf16hi(u);
    }
  } else {
    if constexpr (DPL == 4) {
      const float4 f = *reinterpret_cast<const float4*>(row + lane * 16);
      x[0] = f.x;
      x[1] = f.y;
      x[2] = f.z;
      x[3] = f.w;
    } else {
      const float2 f = *reinterpret_cast<const float2*>(row + lane * 8);
      x[0] = f.x;
      x[1] = f.y;
    }
  }
}

// G: query heads of the kv head rounded up to a power of two; DPL = head_dim / 32.
// A warp carries at most 4 heads: for G = 8 the warps form two sets of 4 (heads 0-3 and
// 4-7), each set taking every 4th position.
template <int G, int DPL>
__device__ __forceinline__ void attn_task(const KParams& P, const OpDesc& od, int op, int t, const Smem& S,
                                          uint32_t& g) {
  constexpr int HW = G < 4 ? G : 4;        // heads per warp
  constexpr int SETS = G / HW;             // warp sets (1 or 2)
  constexpr int WPS = kConsumerWarps / SETS;  // warps per set
  Misc* m = S.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int set = warp / WPS, wi = warp % WPS;
  const int nch = od.nch, np = od.np;
  const int kvh = t / nch, c = t % nch;
  const int pos = m->st.pos;
  const ChunkB b = chunk_bounds(c, nch, pos);
  const int hd = od.hd, gs = od.gs, cbf = od.cache_bf16, cb = cbf ? 2 : 4;
  const int rowb = hd * cb;
  float* q_s = reinterpret_cast<float*>(S.work);                   // [gs][hd]
  uint8_t* new_s = S.work + gs * hd * 4;                            // K row then V row (cache dtype)
  float* mg = reinterpret_cast<float*>(S.work + 8192);             // merge area: [8 warps][HW][hd + 2]
  const int half = hd / 2;
  const float* cosr = od.rope_cos + (size_t)pos * (od.rope_dim / 2);
  const float* sinr = od.rope_sin + (size_t)pos * (od.rope_dim / 2);
  // queries of the group (RoPE, rounded), and the new K/V row if this chunk holds position pos
  for (int e = tid; e < gs * half; e += kConsumers) {
    const int i = e / half, j = e % half;
    const int qh = kvh * gs + i;
    const float a = pset(od.qkv, qh * hd + j), bq = pset(od.qkv, qh * hd + j + half);
    q_s[i * hd + j] = rnd(a * cosr[j] - bq * sinr[j], cbf);
    q_s[i * hd + j + half] = rnd(a * sinr[j] + bq * cosr[j], cbf);
  }
  if (b.has_new) {
    const int koff = od.hq * hd + kvh * hd, voff = (od.hq + od.hkv) * hd + kvh * hd;
    const size_t crow = ((size_t)kvh * od.max_seq + pos) * hd;
    for (int j = tid; j < half; j += kConsumers) {
      const float a = pset(od.qkv, koff + j), bk = pset(od.qkv, koff + j + half);
      const float k0 = rnd(a * cosr[j] - bk * sinr[j], cbf);
      const float k1 = rnd(a * sinr[j] + bk * cosr[j], cbf);
      if (cbf) {
        reinterpret_cast<__nv_bfloat16*>(new_s)[j] = __float2bfloat16_rn(k0);
        reinterpret_cast<__nv_bfloat16*>(new_s)[j + half] = __float2bfloat16_rn(k1);
        reinterpret_cast<__nv_bfloat16*>(od.kcache)[crow + j] = __float2bfloat16_rn(k0);
        reinterpret_cast<__nv_bfloat16*>(od.kcache)[crow + j + half] = __float2bfloat16_rn(k1);
      } else {
        reinterpret_cast<float*>(new_s)[j] = k0;
        reinterpret_cast<float*>(new_s)[j + half] = k1;
        reinterpret_cast<float*>(od.kcache)[crow + j] = k0;
        reinterpret_cast<float*>(od.kcache)[crow + j + half] = k1;
      }
    }
    for (int j = tid; j < hd; j += kConsumers) {
      const float v = rnd(pset(od.qkv, voff + j), cbf);
      if (cbf) {
        reinterpret_cast<__nv_bfloat16*>(new_s + rowb)[j] = __float2bfloat16_rn(v);
        reinterpret_cast<__nv_bfloat16*>(od.vcache)[crow + j] = __float2bfloat16_rn(v);
      } else {
        reinterpret_cast<float*>(new_s + rowb)[j] = v;
        reinterpret_cast<float*>(od.vcache)[crow + j] = v;
      }
    }
  }
  named_bar_sync(1, kConsumers);
  // this lane's dims of the warp's heads (heads past gs are zero)
  float q[HW][DPL], o[HW][DPL], mr[HW], lr[HW];
#pragma unroll
  for (int h = 0; h < HW; ++h) {
    const int qh = set * HW + h;
    mr[h] = -INFINITY;
    lr[h] = 0.f;
#pragma unroll
    for (int d = 0; d < DPL; ++d) {
      q[h][d] = qh < gs ? q_s[qh * hd + lane * DPL + d] : 0.f;
      o[h][d] = 0.f;
    }
  }
  const float sl2 = od.attn_scale * 1.4426950408889634f;  // scores in base-2 units
  auto position = [&](const uint8_t* krow, const uint8_t* vrow) {
    float kf[DPL], vf[DPL], v[HW];
    load_dims<DPL>(krow, cbf, lane, kf);
    load_dims<DPL>(vrow, cbf, lane, vf);
#pragma unroll
    for (int h = 0; h < HW; ++h) {
      float x = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d) x = fmaf(q[h][d], kf[d], x);
      v[h] = x;
    }
    const float mine = group_reduce<HW>(v, lane);
#pragma unroll
    for (int h = 0; h < HW; ++h) {
      const float s = __shfl_sync(0xffffffffu, mine, group_holder<HW>(h)) * sl2;
      const float mn = fmaxf(mr[h], s);
      const float corr = ex2_approx(mr[h] - mn), p = ex2_approx(s - mn);
      lr[h] = lr[h] * corr + p;
#pragma unroll
      for (int d = 0; d < DPL; ++d) o[h][d] = fmaf(p, vf[d], o[h][d] * corr);
      mr[h] = mn;
    }
  };
  // two positions per step: independent loads, dots and butterflies overlap, and one
  // correction factor serves both
  auto position2 = [&](const uint8_t* k0, const uint8_t* v0, const uint8_t* k1, const uint8_t* v1, bool two) {
    float ka[DPL], va[DPL], kb[DPL], vb[DPL], xa[HW], xb[HW];
    load_dims<DPL>(k0, cbf, lane, ka);
    load_dims<DPL>(v0, cbf, lane, va);
    load_dims<DPL>(k1, cbf, lane, kb);
    load_dims<DPL>(v1, cbf, lane, vb);
#pragma unroll
    for (int h = 0; h < HW; ++h) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int d = 0; d < DPL; ++d) {
        x = fmaf(q[h][d], ka[d], x);
        y = fmaf(q[h][d], kb[d], y);
      }
      xa[h] = x;
      xb[h] = y;
    }
    const float ma = group_reduce<HW>(xa, lane);
    const float mb = group_reduce<HW>(xb, lane);
#pragma unroll
    for (int h = 0; h < HW; ++h) {
      const float sa = __shfl_sync(0xffffffffu, ma, group_holder<HW>(h)) * sl2;
      const float sbv = __shfl_sync(0xffffffffu, mb, group_holder<HW>(h)) * sl2;
      const float sb = two ? sbv : -INFINITY;
      const float mn = fmaxf(mr[h], fmaxf(sa, sb));
      const float corr = ex2_approx(mr[h] - mn), pa = ex2_approx(sa - mn), pb = ex2_approx(sb - mn);
      lr[h] = lr[h] * corr + pa + pb;
#pragma unroll
      for (int d = 0; d < DPL; ++d) o[h][d] = fmaf(pb, vb[d], fmaf(pa, va[d], o[h][d] * corr));
      mr[h] = mn;
    }
  };
  const int nst = (b.tc - b.t0 + np - 1) / np;
  for (int st = 0; st < nst; ++st) {
    wait_full(P, S, g, op, t);
    const uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    const int a = b.t0 + st * np;
    const int n = (b.tc - a) < np ? (b.tc - a) : np;
    for (int tt = wi; tt < n; tt += 2 * WPS) {
      const bool two = tt + WPS < n;
      const int t2 = two ? tt + WPS : tt;  // a lone position reads its own row twice, weight 0
      position2(stage + (size_t)tt * rowb, stage + (size_t)(np + tt) * rowb, stage + (size_t)t2 * rowb,
                stage + (size_t)(np + t2) * rowb, two);
    }
    release_stage(S, g);
    ++g;
  }
  if (b.has_new && wi == 0) position(new_s, new_s + rowb);
  // merge the warps of each head's set: M = max m_w, o = sum 2^(m_w - M) o_w, l = sum 2^(m_w - M) l_w
  const int stride = hd + 2;
#pragma unroll
  for (int h = 0; h < HW; ++h) {
    float* rec = mg + (warp * HW + h) * stride;
    if (lane == 0) {
      rec[hd] = mr[h];
      rec[hd + 1] = lr[h];
    }
#pragma unroll
    for (int d = 0; d < DPL; ++d) rec[lane * DPL + d] = o[h][d];
  }
  named_bar_sync(1, kConsumers);
  for (int e = tid; e < gs * hd; e += kConsumers) {
    const int qh = e / hd, d = e % hd;
    const int st2 = qh / HW, h = qh % HW;
    float M = -INFINITY;
    for (int w = st2 * WPS; w < (st2 + 1) * WPS; ++w) M = fmaxf(M, mg[(w * HW + h) * stride + hd]);
    float acc = 0.f, l = 0.f;
    if (M != -INFINITY)
      for (int w = st2 * WPS; w < (st2 + 1) * WPS; ++w) {
        const float* rec = mg + (w * HW + h) * stride;
        const float f = ex2_approx(rec[hd] - M);
        acc = fmaf(f, rec[d], acc);
        l = fmaf(f, rec[hd + 1], l);
      }
    const size_t pi = (size_t)(kvh * gs + qh) * nch + c;
    od.o_out[pi * hd + d] = acc;
    if (d == 0) {
      od.m_out[pi] = M == -INFINITY ? -INFINITY : M * 0.6931471805599453f;  // base 2 -> natural log
      od.l_out[pi] = l;
    }
  }
  // The task that finishes the kv head's chunks last combines them once (split-KV
  // log-sum-exp), so that the output projection reads one vector instead of every chunk.
  __threadfence();
  named_bar_sync(1, kConsumers);  // also: the merge area is free again
  if (tid == 0) m->last_task = atomicAdd(od.fin + kvh, 1u) + 1 == (unsigned)m->st.epoch * (unsigned)nch;
  named_bar_sync(1, kConsumers);
  if (m->last_task) {
    __threadfence();
    float* wt = reinterpret_cast<float*>(S.work + kCombineOff);  // [gs][nch]
    if (warp < gs) {
      const int qh = kvh * gs + warp;
      combine_weights(od.m_out + (size_t)qh * nch, od.l_out + (size_t)qh * nch, nch, wt + warp * nch);
    }
    named_bar_sync(1, kConsumers);
    for (int e = tid; e < gs * hd; e += kConsumers) {
      const int h = e / hd, d = e % hd, qh = kvh * gs + h;
      const float* src = od.o_out + (size_t)qh * nch * hd + d;
      float acc = 0.f;
      for (int c0 = 0; c0 < nch; c0 += 8) {
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = c0 + u < nch ? ldcg(src + (size_t)(c0 + u) * hd) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c0 + u < nch) acc = fmaf(wt[h * nch + c0 + u], a[u], acc);
      }
      od.o_fin[(size_t)qh * hd + d] = acc;
    }
  }
}

template <int DPL>
__device__ __forceinline__ void attn_consume_dpl(const KParams& P, const OpDesc& od, int op, int t, const Smem& S,
                                                 uint32_t& g) {
  const int gs = od.gs;
  if (gs <= 1)
    attn_task<1, DPL>(P, od, op, t, S, g);
  else if (gs <= 2)
    attn_task<2, DPL>(P, od, op, t, S, g);
  else if (gs <= 4)
    attn_task<4, DPL>(P, od, op, t, S, g);
  else
    attn_task<8, DPL>(P, od, op, t, S, g);
}

__device__ __forceinline__ void attn_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S, uint32_t& g) {
  if (od.hd == 128)
    attn_consume_dpl<4>(P, od, op, t, S, g);
  else
    attn_consume_dpl<2>(P, od, op, t, S, g);
}

// MLA absorbed-latent attention on the tensor cores (tcgen05): task c = cache
// block c (positions [64c, 64c + 64) clipped to 0..pos) for all heads at once,
// the heads being the MMA's M = 128 rows (DeepSeek-V3 absorbed form, the
// "MLA" model structure of the pages).
//   S = Q . C^T : Q = [q_lat | q_pe] bf16 [128 x (kvl + rdim)], C = the block's
//                 cache rows [64 x (kvl + rdim)]; nine 64-dim K-chunks, each
//                 ring stage carrying Q's chunk (16 KB) and C's chunk (8 KB).
//   P = exp(S * scale - m) per head (8 warps, each 32 heads x 32 positions of TMEM),
//       split into bf16 hi + lo parts so that P keeps ~16 mantissa bits.
//   O = P . C_lat : two ring stages of 256 latent dims (32 KB each); C is
//                 read MN-major from the same bytes the S step read K-major.
// The task publishes (m, l, O) for the split-KV log-sum-exp combine in the uv
// projection's prologue.  The step's new latent row is already in the cache:
// absorb_q's extra last task writes it (mla_new_row).
// TMEM: 512 fp32 columns x 128 lanes; S uses columns 0..63 and is read out
// before O (columns 0..511) overwrites it.
__device__ __forceinline__ void mla_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S, uint32_t& g,
                                            uint32_t& nmma) {
  Misc* m = S.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pos = m->st.pos, T = pos + 1, nch = od.nch, H = od.H;
  const int os = od.osplit > 1 ? od.osplit : 1, part = t % os;  // part: which half of O's columns
  const int c = t / os, t0 = c * kMlaBlock;
  if (t0 >= T) {  // block beyond the sequence: empty partial (l = 0)
    for (int h = tid; h < H && part == 0; h += kConsumers) {
      od.m_out[(size_t)h * nch + c] = -INFINITY;
      od.l_out[(size_t)h * nch + c] = 0.f;
    }
    return;
  }
  const int n = T - t0 < kMlaBlock ? T - t0 : kMlaBlock;
  const int kvl = od.kvl, rd = od.rdim, rowe = kvl + rd;
  uint8_t* Phi = S.work;                                                   // [64 pos] x [128 heads] bf16, A layout
  uint8_t* Plo = S.work + 16384;
  const uint32_t tm = m->tmem;
  constexpr uint32_t kIdS = umma_idesc_bf16(128, kMlaBlock, false);
  constexpr uint32_t kIdO = umma_idesc_bf16(128, 256, true);
  constexpr uint32_t kIdO4 = umma_idesc_bf16(128, 128, true);  // a quarter of the columns
  // ---- S = Q . C^T over (kvl + rd) / 64 stages
  const int nS = rowe / 64;
  for (int j = 0; j < nS; ++j) {
    wait_full(P, S, g, op, t);
    uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    if (warp == 0) {
      if (lane == 0) {
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 4; ++s)  // K = 16 dims = two core matrices per MMA
          tc_mma(tm, umma_desc(stage + s * 4096, 2048, 128), umma_desc(stage + 16384 + s * 2048, 1024, 128), kIdS,
                 (j | s) != 0);
        tc_commit(&m->empty[g % kStages]);  // the stage is free once these MMAs have read it
      }
      __syncwarp();
    } else {
      release_stage(S, g);
    }
    ++g;
  }
  if (tid == 0) tc_commit(&m->mma_bar);
  // ---- softmax: all 8 warps; warp w reads TMEM lanes 32 (w % 4).. (heads) and
  // columns 32 (w / 4).. (positions); row max and sum meet in shared memory.
  const int quad = warp & 3, half = warp >> 2;
  const int h = 32 * quad + lane;
  float* red = m->red;  // [2][128]
  mbar_wait(&m->mma_bar, nmma & 1, P, &m->abort, op, t);
  __syncwarp();
  tc_fence_after();
  {
    uint32_t r[32];
    tmem_ld32(tm + ((uint32_t)(32 * quad) << 16) + 32 * half, r);
    tmem_wait_ld();
    const float sl2 = od.attn_scale * 1.4426950408889634f;  // scale * log2(e): p = 2^(s * sl2 - max)
    const int nv = n - 32 * half;                             // valid columns of this half
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nv) mx = fmaxf(mx, __uint_as_float(r[i]) * sl2);
    red[128 * half + h] = mx;
    named_bar_sync(1, kConsumers);
    mx = fmaxf(red[h], red[128 + h]);  // n >= 1: finite
    float l = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // positions 32 half + 8q .. + 7
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = 8 * q + 2 * e;
        const float p0 = i0 < nv ? ex2_approx(__uint_as_float(r[i0]) * sl2 - mx) : 0.f;
        const float p1 = i0 + 1 < nv ? ex2_approx(__uint_as_float(r[i0 + 1]) * sl2 - mx) : 0.f;
        l += p0 + p1;
        const __nv_bfloat162 ph = __floats2bfloat162_rn(p0, p1);
        const float2 phf = __bfloat1622float2(ph);
        const __nv_bfloat162 pl = __floats2bfloat162_rn(p0 - phf.x, p1 - phf.y);
        hi[e] = *reinterpret_cast<const uint32_t*>(&ph);
        lo[e] = *reinterpret_cast<const uint32_t*>(&pl);
      }
      const int off = (4 * half + q) * 2048 + (h >> 3) * 128 + (h & 7) * 16;
      *reinterpret_cast<uint4*>(Phi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(Plo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    named_bar_sync(1, kConsumers);  // both halves read red[] before it is reused
    red[128 * half + h] = l;
    fence_async_smem();
    tc_fence_before();
    named_bar_sync(1, kConsumers);
    if (half == 0 && h < H && part == 0) {  // (m, l) in natural-log units for the combine
      od.m_out[(size_t)h * nch + c] = mx * 0.6931471805599453f;  // log2 units -> natural log
      od.l_out[(size_t)h * nch + c] = red[h] + red[128 + h];
    }
  }
  // ---- O = P . C_lat over kvl / 256 stages (hi and lo parts of P)
  const int nks = (n + 15) / 16;
  for (int o = 0; o < (os == 4 ? 1 : kvl / 256); ++o) {
    if (os == 2 && o != part) continue;  // the other half of the columns is the other task's
    wait_full(P, S, g, op, t);
    uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    if (warp == 0) {
      if (lane == 0) {
        tc_fence_after();
        // TMEM columns of this stage's O: 256 o (halves), 128 part (quarters)
        const uint32_t dcol = os == 4 ? 128 * part : 256 * o;
        for (int s = 0; s < nks; ++s) {  // K = 16 positions
          const uint64_t b = umma_desc(stage + s * 256, 128, 1024);  // MN-major: K step 128 B, N step 1024 B
          tc_mma(tm + dcol, umma_desc(Phi + s * 4096, 2048, 128), b, os == 4 ? kIdO4 : kIdO, s != 0);
          tc_mma(tm + dcol, umma_desc(Plo + s * 4096, 2048, 128), b, os == 4 ? kIdO4 : kIdO, 1);
        }
        tc_commit(&m->empty[g % kStages]);
      }
      __syncwarp();
    } else {
      release_stage(S, g);
    }
    ++g;
  }
  if (tid == 0) tc_commit(&m->mma_bar);
  // ---- epilogue: warp w reads lanes 32 (w % 4).. and columns col0.. (its half of the
  // task's columns); each
  // 32 x 32 tile goes through shared memory so that the stores are coalesced
  mbar_wait(&m->mma_bar, (nmma + 1) & 1, P, &m->abort, op, t);
  __syncwarp();
  tc_fence_after();
  // this task's kvl / os columns, half of them per warp half, 32 per read
  const int ncols = kvl / os, ncc = ncols / 64, col0 = ncols * part + (ncols / 2) * half;
  float* tile = reinterpret_cast<float*>(S.work) + warp * (32 * 36);  // [32 heads][36] (P is dead)
#pragma unroll 1
  for (int cc = 0; cc < ncc; ++cc) {
    uint32_t r[32];
    tmem_ld32(tm + ((uint32_t)(32 * quad) << 16) + col0 + 32 * cc, r);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<float4*>(tile + lane * 36 + 4 * q) =
          make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                      __uint_as_float(r[4 * q + 3]));
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 8; ++it) {  // 4 heads x 32 columns per instruction
      const int i = 4 * it + (lane >> 3), q = lane & 7;
      const int hh = 32 * quad + i;
      if (hh < H)
        *reinterpret_cast<float4*>(od.o_out + ((size_t)hh * nch + c) * kvl + col0 + 32 * cc + 4 * q) =
            *reinterpret_cast<const float4*>(tile + i * 36 + 4 * q);
    }
    __syncwarp();
  }
  tc_fence_before();
  nmma += 2;
}

// Final op: greedy token = argmax over the LM-head tasks' best keys; advance the step state.
__device__ __forceinline__ void final_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S) {
  Misc* m = S.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned long long key = 0ull;
  for (int i = tid; i < od.fin_n; i += kConsumers) {
    const unsigned long long k = __ldcg(od.fin_best + i);
    key = k > key ? k : key;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long ok = __shfl_xor_sync(0xffffffffu, key, o);
    key = ok > key ? ok : key;
  }
  if (lane == 0) m->redk[warp] = key;
  named_bar_sync(1, kConsumers);
  if (tid == 0) {
    unsigned long long b = 0ull;
    for (int w = 0; w < kConsumerWarps; ++w) b = m->redk[w] > b ? m->redk[w] : b;
    int next = (int)(0xFFFFFFFFu - (uint32_t)(b & 0xFFFFFFFFull));
    // the winning logit, decoded from its order-preserving key
    const uint32_t kb = (uint32_t)(b >> 32);
    const float best = __uint_as_float((kb & 0x80000000u) ? (kb & 0x7FFFFFFFu) : ~kb);
    const bool bad = next < 0 || next >= od.vocab || !finite_bits(best);
    if (next < 0 || next >= od.vocab) next = 0;
    if (P.persistent) {
      // every CTA must have read this step's state before it changes
      const unsigned target = (unsigned)m->st.epoch * (unsigned)P.n_ctas;
      bounded_wait([&] { return (int)(ld_acquire_gpu(P.started) - target) >= 0; }, P, &m->abort, op, t, true);
    } else {
      atomicAdd(P.started, (unsigned)P.n_ctas);  // keep started == epoch * n_ctas across modes
    }
    StepState ns;
    ns.epoch = m->st.epoch + 1;
    ns.pos = m->st.pos + 1;
    ns.tok = next;
    ns.last = next;
    ns.stop = 0;
    ns.pad[0] = ns.pad[1] = ns.pad[2] = 0;
    if (P.gen && __ldcg(&P.gen->active)) {  // generation: the token goes to the host as soon as it is known
      const int s = m->st.epoch - __ldcg(&P.gen->epoch0);
      reinterpret_cast<volatile int*>(P.tok_ring)[s] = next;
      __threadfence_system();
      *reinterpret_cast<volatile unsigned*>(P.tok_count) = (unsigned)(s + 1);
      if (next == __ldcg(&P.gen->stop_token) || *reinterpret_cast<const volatile int*>(P.stop_word) != 0)
        ns.stop = 1;
    }
    *P.state = ns;
    P.status->final_key = b;  // the winning packed key, for dumps
    if (bad) report_nonfinite(P, op, t);  // after the state: a stopped step still advances consistently
  }
}

// ------------------------------------------------------------ task lists
// Walks this CTA's (op, task) list; the entry after the current one is loaded a
// task ahead so the list read never sits on the critical path.
struct TaskIter {
  const int2* list;
  int i, end, op, stride, persistent;
  int2 nxt;
  __device__ void init(const KParams& p) {
    persistent = p.persistent;
    if (persistent) {
      list = p.tasks;
      i = p.task_off[blockIdx.x];
      end = p.task_off[blockIdx.x + 1];
      stride = 1;
      if (i < end) nxt = __ldg(list + i);
    } else {
      list = nullptr;
      op = p.op_only;
      i = blockIdx.x;
      end = __ldg(&p.ops[op].ntasks);
      stride = gridDim.x;
    }
  }
  __device__ bool next(int& o, int& t) {
    if (i >= end) return false;
    if (persistent) {
      o = nxt.x;
      t = nxt.y;
      if (i + 1 < end) nxt = __ldg(list + i + 1);
    } else {
      o = op;
      t = i;
    }
    i += stride;
    return true;
  }
};

// --------------------------------------------------------------- producer
__device__ void producer_loop(const KParams& P, const Smem& S) {
  Misc* m = S.m;
  const int lane = threadIdx.x & 31;
  const uint64_t pol_w = policy_evict_first();  // weights: streamed once per step
  // caches: re-read every step, so kept in L2 while they fit there; past that they only push
  // other lines out and are streamed like the weights
  const uint64_t pol_kv = P.kv_evict_first ? policy_evict_first() : policy_evict_last();
  uint32_t g = 0;
  TaskIter it;
  it.init(P);
  int op, t, cur = -1;
  const int pos0 = m->st.pos;
  const unsigned epoch0 = (unsigned)m->st.epoch;
  const OpDesc& od = *S.pod;
  unsigned long long* tr_first = nullptr;  // trace: where the current task's first issue time goes (lane 0)
  auto issue = [&](const void* src, uint32_t bytes, const void* src2, uint32_t bytes2, uint32_t off2,
                   uint64_t pol) -> bool {
    uint64_t* eb = &m->empty[g % kStages];
    const uint32_t par = ((g / kStages) & 1) ^ 1;
    int ready = 1;
    if (lane == 0) ready = mbar_wait(eb, par, P, &m->abort, op, t) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ready, 0)) return false;
    if (lane == 0) {
      if (tr_first) {
        *tr_first = globaltimer();
        tr_first = nullptr;
      }
      uint8_t* dst = S.ring + (g % kStages) * kStageBytes;
      uint64_t* fb = &m->full[g % kStages];
      mbar_arrive_expect_tx(fb, bytes + bytes2);
      if (bytes && src) bulk_g2s(dst, src, bytes, fb, pol);  // src null: the caller copies it later
      if (bytes2) bulk_g2s(dst + off2, src2, bytes2, fb, pol);
    }
    __syncwarp();
    ++g;
    return true;
  };
  bool ok = true;
  int pos = pos0;
  unsigned epoch = epoch0;
  for (int step = 0; step < P.n_steps && ok; ++step) {
  if (step > 0) {
    // A launch of several steps: the previous step's final op (the last op) wrote this
    // step's state; take it once that op is published, and end if it asked to.
    int r = 0, npos = 0, nep = 0, stop = 0;
    if (lane == 0) {
      r = wait_counter(P, P.nops - 1, epoch, &m->abort, P.nops - 1, 0) ? 1 : 0;
      if (r) {
        npos = __ldcg(&P.state->pos);
        nep = __ldcg(&P.state->epoch);
        stop = __ldcg(&P.state->stop);
        m->prod_route_op = -1;
        m->prod_dep_op = -1;
      }
    }
    if (!__shfl_sync(0xffffffffu, r, 0) || __shfl_sync(0xffffffffu, stop, 0)) break;
    pos = __shfl_sync(0xffffffffu, npos, 0);
    epoch = (unsigned)__shfl_sync(0xffffffffu, nep, 0);
    __syncwarp();
    it.init(P);
  }
  while (ok && it.next(op, t)) {
    if (op != cur) {
      copy_od(S.pod, P.ops + op, lane, 32);
      __syncwarp();
      cur = op;
    }
    tr_first = nullptr;
    if (P.trace && lane == 0) {  // when the producer reached this task
      const int idx = P.persistent ? it.i - 1 : t;
      if (idx < P.trace_cap) {
        unsigned long long* rec = P.trace + 2 + 6 * (size_t)P.trace_cap + 3 * (size_t)idx;
        rec[0] = ((unsigned long long)blockIdx.x << 48) | ((unsigned long long)op << 32) | (unsigned)t;
        rec[1] = globaltimer();
        tr_first = rec + 2;  // the task's first issued stage stamps it
      }
    }
    if (od.kind == OP_GEMV) {
      const int tpt = od.tpt > 1 ? od.tpt : 1;
      const bool row_task = od.qc && t == od.ntasks - 1;  // absorb_q's latent-row task streams nothing
      for (int i = 0; i < tpt && ok && !row_task; ++i) {
      const TaskGeo geo = gemv_geo(od, t * tpt + i);
      const Seg& sg = od.seg[geo.si];
      const uint8_t* base = sg.w;
      if (sg.slot >= 0) {
        if (m->prod_route_op != od.pdep) {
          bool ready = true;
          if (P.persistent) {
            int r = 1;
            if (lane == 0) r = wait_counter(P, od.pdep, epoch, &m->abort, op, t) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, r, 0) != 0;
          }
          if (!ready) {
            ok = false;
            break;
          }
          if (lane < od.top_k) m->prod_idx[lane] = __ldcg(od.rt_ids + lane);  // written by the router's last task
          if (lane == 0) m->prod_route_op = od.pdep;
          __syncwarp();
        }
        base += (size_t)m->prod_idx[sg.slot] * sg.w_estride;
      }
      const uint32_t sb = (uint32_t)(od.R * od.kcb);
      const uint8_t* tile = base + (size_t)(geo.rt * od.S + geo.s) * od.nst * sb;
      for (int st = 0; st < od.nst && ok; ++st) ok = issue(tile + (size_t)st * sb, sb, nullptr, 0, 0, pol_w);
      }  // units
    } else if (od.kind == OP_ATTN) {
      const int kvh = t / od.nch, c = t % od.nch;
      const ChunkB b = chunk_bounds(c, od.nch, pos);
      const int rowb = od.hd * (od.cache_bf16 ? 2 : 4);
      for (int a = b.t0; a < b.tc && ok; a += od.np) {
        const int n = (b.tc - a) < od.np ? (b.tc - a) : od.np;
        const size_t off = ((size_t)kvh * od.max_seq + a) * rowb;
        ok = issue((const uint8_t*)od.kcache + off, n * rowb, (const uint8_t*)od.vcache + off, n * rowb,
                   od.np * rowb, pol_kv);
      }
    } else if (od.kind == OP_MLA) {
      // block cb: nine (Q chunk, C chunk) stages for S, then two C stages for O (one: the
      // task's half of O's columns when the op splits O)
      const int os = od.osplit > 1 ? od.osplit : 1, cb = t / os, part = t % os;
      if (cb * kMlaBlock <= pos) {
        const int rowe = od.kvl + od.rdim, nS = rowe / 64;
        const uint8_t* blk = (const uint8_t*)od.kcache + (size_t)cb * rowe * kMlaBlock * 2;
        const uint8_t* q = (const uint8_t*)od.qc;
        int early = 0;
        const uint32_t g0 = g;
        if (m->prod_dep_op != op) {
          // The cache chunks do not depend on this step's ops (except in the block that
          // absorb_q appends to): start them in the first free stages now; the query
          // chunks (written by absorb_q) join the same stages once absorb_q is done.
          if (pos >= (cb + 1) * kMlaBlock)
            for (; early < nS && early < kStages && ok; ++early)
              ok = issue(nullptr, 16384, blk + early * 8192, 8192, 16384, pol_kv);  // expects both parts
          int r = ok ? 1 : 0;
          if (lane == 0 && ok) {
            if (P.persistent) r = wait_counter(P, od.pdep, epoch, &m->abort, op, t) ? 1 : 0;
            fence_async_global();
          }
          if (!__shfl_sync(0xffffffffu, r, 0)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            m->prod_dep_op = op;
            for (int j = 0; j < early; ++j) {
              const uint32_t gj = g0 + j;
              bulk_g2s(S.ring + (gj % kStages) * kStageBytes, q + j * 16384, 16384, &m->full[gj % kStages], pol_kv);
            }
          }
          __syncwarp();
        }
        for (int j = early; j < nS && ok; ++j) ok = issue(q + j * 16384, 16384, blk + j * 8192, 8192, 16384, pol_kv);
        if (os == 4)  // a quarter of the columns: 16 contiguous 8-dim groups, 16 KB
          ok = issue(blk + part * 16384, 16384, nullptr, 0, 0, pol_kv);
        else
          for (int o = 0; o < od.kvl / 256 && ok; ++o)
            if (os == 1 || o == part) ok = issue(blk + o * 32768, 32768, nullptr, 0, 0, pol_kv);
      }
    }
  }
  }  // steps
  if (lane == 0) m->issued = (int)g;
}

// --------------------------------------------------------------- signaller
// Hands a finished task (or the end sentinel op = -1) to the signaller warp.
// Called by all consumer threads after the task's last barrier.
__device__ __forceinline__ void post_task(const KParams& P, Misc* m, uint32_t q, int op, int t, uint64_t t0) {
  const int slot = q % kMail;
  const uint32_t par = (q / kMail) & 1;
  if (threadIdx.x == 0) {
    const uint64_t t_done = P.trace ? globaltimer() : 0;
    mbar_wait(&m->sig_free[slot], par ^ 1, P, &m->abort, op, t);
    m->mail_op[slot] = op;
    m->mail_task[slot] = t;
    m->mail_t[slot][0] = t0;
    m->mail_t[slot][1] = m->tr_pro;
    m->mail_t[slot][2] = m->tr_data;
    m->mail_t[slot][3] = t_done;
  }
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&m->sig_done[slot]);
}

// Publishes finished tasks in batches: it waits for the oldest unpublished task,
// takes every later one that is already finished too, and releases the whole
// batch with one gpu-scope fence and one counter add per run of equal ops.
__device__ void signal_loop(const KParams& P, const Smem& S) {
  Misc* m = S.m;
  const int lane = threadIdx.x & 31;
  uint32_t q = 0;
  bool done = false;
  while (!done) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait(&m->sig_done[q % kMail], (q / kMail) & 1, P, &m->abort, -1, (int)q) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    if (lane == 0) {
      uint32_t end = q + 1;  // batch [q, end)
      // a probe of the later slots: test_wait, which never suspends the thread
      while (end - q < kMail && mbar_test_wait(&m->sig_done[end % kMail], (end / kMail) & 1)) ++end;
      // every consumer write of these tasks happened before their mailbox hand-off
      __threadfence();
      uint32_t i = q;
      while (i < end) {
        const int op = m->mail_op[i % kMail];
        if (op < 0) {
          done = true;
          end = i;
          break;
        }
        uint32_t j = i + 1;
        while (j < end && m->mail_op[j % kMail] == op) ++j;
        uint32_t cnt = j - i;
        if (P.test_stall && op == 0)  // failure-path test: task 0 of op 0 is never published
          for (uint32_t z = i; z < j; ++z)
            if (m->mail_task[z % kMail] == 0) --cnt;
        if (cnt) red_release_gpu_add(&P.counters[op], cnt);
        i = j;
      }
      if (P.trace) {
        const uint64_t now = globaltimer();
        const unsigned r0 = atomicAdd(reinterpret_cast<unsigned*>(P.trace), end - q);
        for (uint32_t k = q; k < end; ++k) {
          const unsigned r = r0 + (k - q);
          if ((int)r < P.trace_cap) {
            unsigned long long* rec = P.trace + 2 + (size_t)r * 6;
            rec[0] = ((unsigned long long)blockIdx.x << 48) | ((unsigned long long)m->mail_op[k % kMail] << 32) |
                     (unsigned)m->mail_task[k % kMail];
            rec[1] = m->mail_t[k % kMail][0];
            rec[2] = m->mail_t[k % kMail][1];
            rec[3] = m->mail_t[k % kMail][2];
            rec[4] = m->mail_t[k % kMail][3];
            rec[5] = now;
          }
        }
      }
      for (uint32_t k = q; k < end; ++k) mbar_arrive(&m->sig_free[k % kMail]);
      q = end;
    }
    done = __shfl_sync(0xffffffffu, done ? 1 : 0, 0) != 0;
    q = __shfl_sync(0xffffffffu, q, 0);
  }
}

// --------------------------------------------------------------- consumer
// WT: weight storage type of the model; MLA: whether attention is the MLA kind.
// Each model compiles only its own GEMV and attention paths.
template <int WT, bool MLA>
__device__ __forceinline__ void consumer_loop(const KParams& P, const Smem& S) {
  Misc* m = S.m;
  uint32_t g = 0, q = 0, nmma = 0;
  TaskIter it;
  it.init(P);
  int op, t, cur = -1;
  const OpDesc& od = *S.cod;
  bool stopped = false;
  for (int step = 0; step < P.n_steps && !stopped; ++step) {
  if (step > 0) {
    // the previous step's final op wrote this step's state (see the producer)
    if (threadIdx.x == 0) {
      if (wait_counter(P, P.nops - 1, (unsigned)m->st.epoch, &m->abort, P.nops - 1, 0)) {
        m->st.epoch = __ldcg(&P.state->epoch);
        m->st.pos = __ldcg(&P.state->pos);
        m->st.tok = __ldcg(&P.state->tok);
        m->st.stop = __ldcg(&P.state->stop);
        m->x_op = -1;
        if (!m->st.stop) atomicAdd(P.started, 1u);  // this CTA has read the step's state
      }
    }
    if (named_bar_or(1, kConsumers, m->abort)) break;
    if (m->st.stop) break;
    it.init(P);
    cur = -1;
  }
  const unsigned epoch = (unsigned)m->st.epoch;
  while (it.next(op, t)) {
    if (op != cur) {
      copy_od(S.cod, P.ops + op, threadIdx.x, kConsumers);
      if (P.persistent && threadIdx.x == 0) {
        const OpDesc* go = P.ops + op;
        if (wait_counter(P, __ldg(&go->dep[0]), epoch, &m->abort, op, t))
          wait_counter(P, __ldg(&go->dep[1]), epoch, &m->abort, op, t);
      }
      // uniform decision: every consumer thread sees the same value
      if (named_bar_or(1, kConsumers, m->abort)) {
        stopped = true;
        break;
      }
      cur = op;
    }
    const uint64_t t_start = P.trace ? globaltimer() : 0;
    if (P.trace && threadIdx.x == 0) m->tr_pro = m->tr_data = t_start;
    const int kind = od.kind;
    if (kind == OP_GEMV) {
      gemv_consume<WT>(P, od, op, t, S, g);
    } else if (kind == OP_FINAL) {
      final_consume(P, od, op, t, S);
    } else {
      if constexpr (MLA)
        mla_consume(P, od, op, t, S, g, nmma);
      else
        attn_consume(P, od, op, t, S, g);
      if (threadIdx.x == 0) m->x_op = -1;
    }
    // A failed wait anywhere in the task makes every thread stop here, after the
    // task's barriers, without publishing the task.
    if (named_bar_or(1, kConsumers, m->abort)) {
      stopped = true;
      break;
    }
    post_task(P, m, q++, op, t, t_start);
  }
  }  // steps
  post_task(P, m, q, -1, -1, 0);  // end sentinel for the signaller
  if (threadIdx.x == 0) m->consumed = (int)g;
}

template <int WT, bool MLA>
__global__ void __launch_bounds__(kThreads, 1) engine_kernel(KParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const Smem S = smem_layout(smem_raw);
  Misc* m = S.m;
  if (threadIdx.x == 0) {
    m->st = *P.state;
    if (P.tok_in >= 0) m->st.tok = P.tok_in;
    m->abort = 0;
    m->x_op = -1;
    m->x_group = -1;
    m->prod_route_op = -1;
    m->prod_dep_op = -1;
    // valid expert ids until the router's are read: a task that runs on stale data after
    // a failed wait (abort) still addresses weights and scales inside their arrays
    for (int i = 0; i < kMaxTopK; ++i) m->prod_idx[i] = 0;
    m->issued = 0;
    m->consumed = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&m->full[i], 1);
      mbar_init(&m->empty[i], kConsumerWarps);
    }
    for (int i = 0; i < kMail; ++i) {
      mbar_init(&m->sig_done[i], kConsumerWarps);
      mbar_init(&m->sig_free[i], 1);
    }
    mbar_init(&m->mma_bar, 1);
    mbar_init(&m->fin_bar, 1);
    fence_mbar_init();
    if (P.persistent) {
      __threadfence();
      atomicAdd(P.started, 1u);
    }
  }
  const int warp = threadIdx.x >> 5;
  if constexpr (MLA) {  // all 512 TMEM columns: one CTA per SM
    if (warp == 0) {
      __syncwarp();  // .sync.aligned: the whole warp, converged
      tmem_alloc(&m->tmem, 512);
      tmem_relinquish();
    }
    tc_fence_before();
  }
  __syncthreads();
  if constexpr (MLA) tc_fence_after();
  if (warp == kProducerWarp)
    producer_loop(P, S);
  else if (warp == kSignalWarp)
    signal_loop(P, S);
  else
    consumer_loop<WT, MLA>(P, S);
  __syncthreads();
  if constexpr (MLA) {
    // no MMA may still be running when the columns are freed (after a failure mid-task)
    if (warp == 0) {
      if (threadIdx.x == 0) {
        tc_commit(&m->fin_bar);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&m->fin_bar, 0) && globaltimer() - t0 < 1000000000ull) {
        }
      }
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(m->tmem, 512);
    }
  }
  // After a failure, let the copies still in flight land before the CTA exits.
  if (threadIdx.x == 0 && m->issued > m->consumed) {
    const uint64_t t0 = globaltimer();
    for (int g = m->consumed; g < m->issued; ++g) {
      while (!mbar_try_wait(&m->full[g % kStages], (g / kStages) & 1)) {
        if (globaltimer() - t0 > 2000000000ull) break;
      }
    }
  }
}

}  // namespace dec
