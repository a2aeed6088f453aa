// Device engine of the decode step: tile tasks and the persistent scheduler.
//
// A CTA = 8 consumer warps (compute) + 1 producer warp (weight / KV streaming).
// The producer walks the CTA's task list and streams every task's bytes from
// HBM into a kStages-deep shared-memory ring with 1-D TMA bulk copies; it never
// waits for activation dependencies (weights are static), so the next tasks'
// weights are in flight while the consumers wait for the previous layer.  Only
// routed-expert weights wait: their address comes from the router's top-k.
// Consumers wait on the dependency counters of the task's op, build the
// task's input vector in shared memory (norm / combine / SwiGLU prologue),
// consume the ring stages and publish fp32 partial outputs plus one counter
// increment.  Every wait is bounded by a global-timer deadline; on expiry the
// CTA records the failure in a status word and drains its in-flight copies.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "dec_types.h"
#include "ptx.cuh"

namespace dec {

struct Misc {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  StepState st;
  volatile int abort;
  int x_op, x_group;   // identity of the input vector currently in the work area
  int consumed;        // ring stages consumed (consumer thread 0)
  int issued;          // ring stages issued (producer lane 0)
  int prod_route_op;   // router op whose top-k is in prod_idx
  int prod_idx[kMaxTopK];
  float cons_w[kMaxTopK];
  float red[256];
  unsigned long long redk[8];
  float attn_M[128], attn_den[128];
};

constexpr int kRingBytes = kStages * kStageBytes;
constexpr int kSmemBytes = kRingBytes + kWorkBytes + (int)sizeof(Misc);

struct Smem {
  uint8_t* ring;
  uint8_t* work;
  Misc* m;
};

__device__ __forceinline__ Smem smem_layout(uint8_t* base) {
  Smem s;
  s.ring = base;
  s.work = base + kRingBytes;
  s.m = reinterpret_cast<Misc*>(base + kRingBytes + kWorkBytes);
  return s;
}

// ------------------------------------------------------------ error / waits
__device__ __forceinline__ void report_timeout(const KParams& P, int op, int task) {
  if (atomicCAS(&P.status->code, 0, 1) == 0) {
    P.status->cta = blockIdx.x;
    P.status->op = op;
    P.status->task = task;
  }
}

// Spin until ready(); false if this CTA or another one gave up.
template <class F>
__device__ __forceinline__ bool bounded_wait(F ready, const KParams& P, volatile int* abort, int op, int task,
                                             bool sleep) {
  if (ready()) return true;
  const uint64_t t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
    if (ready()) return true;
    if ((it & 31) == 0) {
      if (*abort) return false;
      if (ld_volatile_int(&P.status->code) != 0) {
        *abort = 1;
        return false;
      }
      if (globaltimer() - t0 > P.timeout_ns) {
        report_timeout(P, op, task);
        *abort = 1;
        return false;
      }
    }
    if (sleep) __nanosleep(64);
  }
}

__device__ __forceinline__ bool wait_counter(const KParams& P, int dop, unsigned epoch, volatile int* abort,
                                             int op, int task) {
  if (dop < 0) return true;
  const unsigned target = epoch * (unsigned)P.ops[dop].ntasks;
  const unsigned* c = &P.counters[dop];
  return bounded_wait([&] { return (int)(ld_acquire_gpu(c) - target) >= 0; }, P, abort, op, task, true);
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

__device__ __forceinline__ float rnd(float v, int bf16) { return bf16 ? bf16_round(v) : v; }

__device__ __forceinline__ void store_x(uint8_t* work, int in_bf16, int e, float v) {
  if (in_bf16)
    reinterpret_cast<__nv_bfloat16*>(work)[e] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(work)[e] = v;
}

// Softmax top-k router (one warp, all 32 lanes call): pick the k largest logits,
// ties to the lower expert id, weights renormalised over the chosen k:
// w_j = exp(r_j - r_max) / sum_i exp(r_i - r_max).
__device__ void warp_route(const PSet& logits, int E, int k, int* idx_out, float* w_out) {
  const int lane = threadIdx.x & 31;
  float v[8];
  int taken = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int e = lane + 32 * i;
    v[i] = e < E ? pset(logits, e) : -INFINITY;
  }
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
    if (bi >= E) {  // only reachable with NaN logits: fall back to the lowest free id
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
}

// ------------------------------------------------------------- prologues
// Build the input vector of (op, group) in the work area, all 256 consumer threads.
__device__ void prologue(const OpDesc& od, int group, int task, const Smem& S) {
  Misc* m = S.m;
  const int tid = threadIdx.x;
  uint8_t* x = S.work;
  const int n = od.n;
  const int bf = od.in_bf16;
  switch (od.pro) {
    case PRO_RESID_NORM: {
      if (od.routed.ptr) {
        if (tid < 32) warp_route(od.route_logits, od.n_experts, od.top_k, nullptr, m->cons_w);
        named_bar_sync(1, kConsumers);
      }
      constexpr int kPer = kMaxD / kConsumers;
      float v[kPer];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = tid + i * kConsumers;
        float h = 0.f;
        if (e < n) {
          if (od.base_embed) {
            const size_t row = (size_t)m->st.tok * n;
            h = od.embed_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(od.embed)[row + e])
                              : reinterpret_cast<const float*>(od.embed)[row + e];
          } else {
            h = ldcg(od.h_base + e);
          }
          if (od.add.ptr) h += pset(od.add, e);
          if (od.routed.ptr) {
            float r = 0.f;
            for (int j = 0; j < od.top_k; ++j) {
              PSet p = od.routed;
              p.off += j * od.routed_slot_stride;
              r += m->cons_w[j] * pset(p, e);
            }
            h += r;
          }
          if (od.add2.ptr) h += pset(od.add2, e);
          ss += h * h;
        }
        v[i] = h;
      }
      const float tot = consumer_sum(ss, m);
      const float inv = 1.0f / sqrtf(tot / (float)n + od.eps);
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = tid + i * kConsumers;
        if (e < n) {
          store_x(x, bf, e, rnd(v[i] * inv * od.gain[e], bf));
          if (od.h_out && task == 0) od.h_out[e] = v[i];
        }
      }
      break;
    }
    case PRO_NORM_SUM: {
      constexpr int kPer = kMaxD / kConsumers;
      float v[kPer];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = tid + i * kConsumers;
        v[i] = e < n ? pset(od.src, e) : 0.f;
        ss += v[i] * v[i];
      }
      const float tot = consumer_sum(ss, m);
      const float inv = 1.0f / sqrtf(tot / (float)n + od.eps);
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = tid + i * kConsumers;
        if (e < n) store_x(x, bf, e, rnd(v[i] * inv * od.gain[e], bf));
      }
      break;
    }
    case PRO_SUM: {
      PSet p = od.src;
      p.off += group * od.gstride;
      for (int e = tid; e < n; e += kConsumers) store_x(x, bf, e, rnd(pset(p, e), bf));
      break;
    }
    case PRO_SWIGLU: {
      PSet g = od.gate, u = od.up;
      g.off += group * od.slot_stride;
      u.off += group * od.slot_stride;
      for (int e = tid; e < n; e += kConsumers) {
        const float gv = pset(g, e), uv = pset(u, e);
        store_x(x, bf, e, rnd(gv / (1.0f + expf(-gv)) * uv, bf));
      }
      break;
    }
    case PRO_ATTN_COMBINE: {
      // per head: M = max over chunks with data, den = sum e^(m_c - M) l_c
      for (int h = tid; h < od.nheads; h += kConsumers) {
        float M = -INFINITY;
        for (int c = 0; c < od.nch; ++c)
          if (ldcg(od.al + h * od.nch + c) > 0.f) M = fmaxf(M, ldcg(od.am + h * od.nch + c));
        float den = 0.f;
        for (int c = 0; c < od.nch; ++c) {
          const float l = ldcg(od.al + h * od.nch + c);
          if (l > 0.f) den += expf(ldcg(od.am + h * od.nch + c) - M) * l;
        }
        m->attn_M[h] = M;
        m->attn_den[h] = den;
      }
      named_bar_sync(1, kConsumers);
      for (int e = tid; e < n; e += kConsumers) {
        const int h = e / od.hdim, d = e % od.hdim;
        const float M = m->attn_M[h];
        float num = 0.f;
        for (int c = 0; c < od.nch; ++c) {
          const float l = ldcg(od.al + h * od.nch + c);
          if (l > 0.f) num += expf(ldcg(od.am + h * od.nch + c) - M) * ldcg(od.ao + ((size_t)h * od.nch + c) * od.hdim + d);
        }
        store_x(x, bf, e, rnd(num / m->attn_den[h], bf));
      }
      break;
    }
    case PRO_MLA_COMBINE: {
      const int h = group;
      if (tid < 32) {
        float M = -INFINITY;
        for (int c = tid; c < od.nch; c += 32)
          if (ldcg(od.al + h * od.nch + c) > 0.f) M = fmaxf(M, ldcg(od.am + h * od.nch + c));
        M = warp_max(M);
        float den = 0.f;
        for (int c = tid; c < od.nch; c += 32) {
          const float l = ldcg(od.al + h * od.nch + c);
          if (l > 0.f) den += expf(ldcg(od.am + h * od.nch + c) - M) * l;
        }
        den = warp_sum(den);
        if (tid == 0) {
          m->attn_M[0] = M;
          m->attn_den[0] = den;
        }
      }
      named_bar_sync(1, kConsumers);
      const float M = m->attn_M[0], den = m->attn_den[0];
      for (int e = tid; e < n; e += kConsumers) {
        float num = 0.f;
        for (int c = 0; c < od.nch; ++c) {
          const float l = ldcg(od.al + h * od.nch + c);
          if (l > 0.f) num += expf(ldcg(od.am + h * od.nch + c) - M) * ldcg(od.ao + ((size_t)h * od.nch + c) * od.hdim + e);
        }
        store_x(x, bf, e, rnd(num / den, bf));
      }
      break;
    }
    default:
      break;
  }
  // zero padding up to Kpad
  for (int e = n + tid; e < od.Kpad; e += kConsumers) store_x(x, bf, e, 0.f);
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

__device__ __forceinline__ bool wait_full(const KParams& P, const Smem& S, uint32_t g, int op, int task) {
  uint64_t* bar = &S.m->full[g % kStages];
  const uint32_t par = (g / kStages) & 1;
  return bounded_wait([&] { return mbar_try_wait(bar, par); }, P, &S.m->abort, op, task, false);
}

__device__ __forceinline__ void release_stage(const Smem& S, uint32_t g) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&S.m->empty[g % kStages]);
}

__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

template <int WT>
__device__ __forceinline__ void gemv_stage(const uint8_t* stage, const uint8_t* x, int k0, const OpDesc& od,
                                           int c, int rg, float scale, float* acc) {
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
    for (int i = 0; i < 8; ++i) {
      if (i >= od.rpt) break;
      const int r = rg + od.G * i;
      const uint4 wv = *reinterpret_cast<const uint4*>(stage + r * od.kcb + c * 16);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
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
    for (int i = 0; i < 8; ++i) {
      if (i >= od.rpt) break;
      const int r = rg + od.G * i;
      const uint4 wv = *reinterpret_cast<const uint4*>(stage + r * od.kcb + c * 16);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
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
    for (int i = 0; i < 8; ++i) {
      if (i >= od.rpt) break;
      const int r = rg + od.G * i;
      const float4 wv = *reinterpret_cast<const float4*>(stage + r * od.kcb + c * 16);
      float a = acc[i];
      a = fmaf(wv.x, xa.x, a);
      a = fmaf(wv.y, xa.y, a);
      a = fmaf(wv.z, xa.z, a);
      a = fmaf(wv.w, xa.w, a);
      acc[i] = a;
    }
  }
}

template <int WT>
__device__ bool gemv_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S, uint32_t& g) {
  const TaskGeo geo = gemv_geo(od, t);
  const Seg& sg = od.seg[geo.si];
  Misc* m = S.m;
  if (m->x_op != op || m->x_group != geo.group) {
    prologue(od, geo.group, t, S);
    if (threadIdx.x == 0) {
      m->x_op = op;
      m->x_group = geo.group;
    }
  }
  const int tid = threadIdx.x;
  const int c = tid % od.cpr, rg = tid / od.cpr;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const float* sc = nullptr;
  const int nkb = (od.K + 127) / 128;
  for (int st = 0; st < od.nst; ++st) {
    wait_full(P, S, g, op, t);  // on failure the task runs to its end on stale data; the caller stops after it
    const uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    const int k0 = (geo.s * od.nst + st) * od.kc;
    float scale = 1.f;
    if constexpr (WT == WT_FP8) {
      if (st == 0) {
        sc = sg.sc + (size_t)((geo.rt * od.R) / 128) * nkb;
        if (sg.slot >= 0) sc += (size_t)m->prod_idx[sg.slot] * sg.s_estride;
      }
      const int cb = (k0 + c * 16) >> 7;
      scale = cb < nkb ? __ldg(sc + cb) : 0.f;
    }
    gemv_stage<WT>(stage, S.work, k0, od, c, rg, scale, acc);
    release_stage(S, g);
    ++g;
  }
  // reduce the cpr partials of every row
  const int lane = tid & 31, warp = tid >> 5;
  const int span = od.cpr < 32 ? od.cpr : 32;
  const int parts = od.cpr / span;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= od.rpt) break;
    float v = acc[i];
    for (int o = span >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    acc[i] = v;
  }
  if ((lane & (span - 1)) == 0) {
    const int part = od.cpr >= 32 ? (warp * 32 % od.cpr) / 32 : 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= od.rpt) break;
      m->red[(i * od.G + rg) * parts + part] = acc[i];
    }
  }
  named_bar_sync(1, kConsumers);
  unsigned long long key = 0ull;
  if (tid < od.R) {
    const int i = tid / od.G, rg2 = tid % od.G;
    float y = 0.f;
    for (int p = 0; p < parts; ++p) y += m->red[(i * od.G + rg2) * parts + p];
    const int row = geo.rt * od.R + tid;
    if (row < sg.N) {
      od.out[(size_t)geo.s * od.out_stride + sg.out_off + row] = y;
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
  return true;
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

__device__ __forceinline__ int attn_stages(const OpDesc& od, int t, int pos) {
  const int c = od.kind == OP_ATTN ? t % od.nch : t % od.nch;
  const ChunkB b = chunk_bounds(c, od.nch, pos);
  return (b.tc - b.t0 + od.np - 1) / od.np;
}

// Dense GQA split-KV attention: task = (kv head g, chunk c); all gs query heads of g.
// Each head keeps a running (max m, sum l, weighted values o) over the chunk
// (online softmax, Milakov & Gimelshein 2018) and publishes them for the
// log-sum-exp combine in the output projection's prologue.
__device__ bool attn_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S, uint32_t& g) {
  Misc* m = S.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = t / od.nch, c = t % od.nch;
  const int pos = m->st.pos;
  const ChunkB b = chunk_bounds(c, od.nch, pos);
  const int hd = od.hd, gs = od.gs, cb = od.cache_bf16 ? 2 : 4;
  const int rowb = hd * cb;
  float* q_s = reinterpret_cast<float*>(S.work);           // [gs][hd]
  uint8_t* new_s = S.work + gs * hd * 4;                    // K row then V row (cache dtype)
  float* sc = reinterpret_cast<float*>(new_s + 2 * rowb);   // [gs][np]
  const int half = hd / 2;
  const float* cosr = od.rope_cos + (size_t)pos * (od.rope_dim / 2);
  const float* sinr = od.rope_sin + (size_t)pos * (od.rope_dim / 2);
  // queries of the group (RoPE, rounded), and the new K/V row if this chunk holds position pos
  for (int e = tid; e < gs * half; e += kConsumers) {
    const int i = e / half, j = e % half;
    const int qh = kvh * gs + i;
    const float a = pset(od.qkv, qh * hd + j), bq = pset(od.qkv, qh * hd + j + half);
    q_s[i * hd + j] = rnd(a * cosr[j] - bq * sinr[j], od.cache_bf16);
    q_s[i * hd + j + half] = rnd(a * sinr[j] + bq * cosr[j], od.cache_bf16);
  }
  if (b.has_new) {
    const int koff = od.hq * hd + kvh * hd, voff = (od.hq + od.hkv) * hd + kvh * hd;
    for (int j = tid; j < half; j += kConsumers) {
      const float a = pset(od.qkv, koff + j), bk = pset(od.qkv, koff + j + half);
      const float k0 = rnd(a * cosr[j] - bk * sinr[j], od.cache_bf16);
      const float k1 = rnd(a * sinr[j] + bk * cosr[j], od.cache_bf16);
      const size_t crow = ((size_t)kvh * od.max_seq + pos) * hd;
      if (od.cache_bf16) {
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
      const float v = rnd(pset(od.qkv, voff + j), od.cache_bf16);
      const size_t crow = ((size_t)kvh * od.max_seq + pos) * hd;
      if (od.cache_bf16) {
        reinterpret_cast<__nv_bfloat16*>(new_s + rowb)[j] = __float2bfloat16_rn(v);
        reinterpret_cast<__nv_bfloat16*>(od.vcache)[crow + j] = __float2bfloat16_rn(v);
      } else {
        reinterpret_cast<float*>(new_s + rowb)[j] = v;
        reinterpret_cast<float*>(od.vcache)[crow + j] = v;
      }
    }
  }
  named_bar_sync(1, kConsumers);
  // per-head running state: warp i < gs owns head i; lane owns hd/32 dims
  const int dpl = hd / 32;
  float mrun = -INFINITY, lrun = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  const int nck = rowb / 16;
  auto block = [&](const uint8_t* Kp, const uint8_t* Vp, int n) {
    for (int p = tid; p < gs * n; p += kConsumers) {
      const int i = p / n, tt = p % n;
      const float* q = q_s + i * hd;
      const uint8_t* krow = Kp + (size_t)tt * rowb;
      float dot = 0.f;
      for (int j = 0; j < nck; ++j) {
        int jj = j + tt;
        jj = jj % nck;
        const uint4 kv = *reinterpret_cast<const uint4*>(krow + jj * 16);
        if (od.cache_bf16) {
          const float* qq = q + jj * 8;
          dot = fmaf(bf16lo(kv.x), qq[0], dot);
          dot = fmaf(bf16hi(kv.x), qq[1], dot);
          dot = fmaf(bf16lo(kv.y), qq[2], dot);
          dot = fmaf(bf16hi(kv.y), qq[3], dot);
          dot = fmaf(bf16lo(kv.z), qq[4], dot);
          dot = fmaf(bf16hi(kv.z), qq[5], dot);
          dot = fmaf(bf16lo(kv.w), qq[6], dot);
          dot = fmaf(bf16hi(kv.w), qq[7], dot);
        } else {
          const float* qq = q + jj * 4;
          dot = fmaf(__uint_as_float(kv.x), qq[0], dot);
          dot = fmaf(__uint_as_float(kv.y), qq[1], dot);
          dot = fmaf(__uint_as_float(kv.z), qq[2], dot);
          dot = fmaf(__uint_as_float(kv.w), qq[3], dot);
        }
      }
      sc[i * od.np + tt] = dot * od.attn_scale;
    }
    named_bar_sync(1, kConsumers);
    if (warp < gs) {
      float* s = sc + warp * od.np;
      float mx = -INFINITY;
      for (int tt = lane; tt < n; tt += 32) mx = fmaxf(mx, s[tt]);
      mx = warp_max(mx);
      const float mnew = fmaxf(mrun, mx);
      const float alpha = expf(mrun - mnew);
      float ls = 0.f;
      for (int tt = lane; tt < n; tt += 32) {
        const float pv = expf(s[tt] - mnew);
        s[tt] = pv;
        ls += pv;
      }
      ls = warp_sum(ls);
      __syncwarp();
      lrun = lrun * alpha + ls;
      mrun = mnew;
      for (int d = 0; d < dpl; ++d) o[d] *= alpha;
      for (int tt = 0; tt < n; ++tt) {
        const float pv = s[tt];
        const uint8_t* vrow = Vp + (size_t)tt * rowb;
        if (od.cache_bf16) {
          const __nv_bfloat16* vv = reinterpret_cast<const __nv_bfloat16*>(vrow) + lane * dpl;
          for (int d = 0; d < dpl; ++d) o[d] = fmaf(pv, __bfloat162float(vv[d]), o[d]);
        } else {
          const float* vv = reinterpret_cast<const float*>(vrow) + lane * dpl;
          for (int d = 0; d < dpl; ++d) o[d] = fmaf(pv, vv[d], o[d]);
        }
      }
    }
    named_bar_sync(1, kConsumers);
  };
  const int nst = (b.tc - b.t0 + od.np - 1) / od.np;
  for (int st = 0; st < nst; ++st) {
    wait_full(P, S, g, op, t);
    const uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    const int a = b.t0 + st * od.np;
    const int n = (b.tc - a) < od.np ? (b.tc - a) : od.np;
    block(stage, stage + (size_t)od.np * rowb, n);
    release_stage(S, g);
    ++g;
  }
  if (b.has_new) block(new_s, new_s + rowb, 1);
  if (warp < gs) {
    const int qh = kvh * gs + warp;
    const size_t pi = (size_t)qh * od.nch + c;
    if (lane == 0) {
      od.m_out[pi] = mrun;
      od.l_out[pi] = lrun;
    }
    for (int d = 0; d < dpl; ++d) od.o_out[pi * hd + lane * dpl + d] = o[d];
  }
  return true;
}

// MLA absorbed-latent attention (CUDA cores): task = (head group of HG heads, chunk c).
// s_h(t) = (q_lat^h . c_t + q_pe^h . kpe_t) * scale over the cached rows
// [c_t | kpe_t]; the chunk holding position pos also normalises, RoPEs and
// appends the new latent row (RMSNorm of the kv_a latent part, RoPE of its key part).
__device__ bool mla_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S, uint32_t& g) {
  Misc* m = S.m;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = t / od.nch, c = t % od.nch;
  const int HG = od.HG, kvl = od.kvl, rd = od.rdim, rowe = kvl + rd, rowb = rowe * 2;
  const int pos = m->st.pos;
  const ChunkB b = chunk_bounds(c, od.nch, pos);
  float* ql = reinterpret_cast<float*>(S.work);            // [HG][kvl]
  float* qp = ql + HG * kvl;                                // [HG][rd]
  __nv_bfloat16* newrow = reinterpret_cast<__nv_bfloat16*>(qp + HG * rd);  // [rowe]
  float* sc = reinterpret_cast<float*>(newrow + rowe);      // [HG][np]
  const float* cosr = od.rope_cos + (size_t)pos * (rd / 2);
  const float* sinr = od.rope_sin + (size_t)pos * (rd / 2);
  const int h0 = hg * HG;
  for (int e = tid; e < HG * kvl; e += kConsumers) {
    const int i = e / kvl, j = e % kvl;
    ql[e] = (h0 + i) < od.H ? bf16_round(pset(od.qlat, (h0 + i) * kvl + j)) : 0.f;
  }
  const int qstride = od.nope + rd;
  for (int e = tid; e < HG * (rd / 2); e += kConsumers) {
    const int i = e / (rd / 2), j = e % (rd / 2);
    float a = 0.f, bb = 0.f;
    if (h0 + i < od.H) {
      a = pset(od.qkv, (h0 + i) * qstride + od.nope + j);
      bb = pset(od.qkv, (h0 + i) * qstride + od.nope + j + rd / 2);
    }
    qp[i * rd + j] = bf16_round(a * cosr[j] - bb * sinr[j]);
    qp[i * rd + j + rd / 2] = bf16_round(a * sinr[j] + bb * cosr[j]);
  }
  if (b.has_new) {
    float ss = 0.f;
    for (int j = tid; j < kvl; j += kConsumers) {
      const float v = pset(od.ckv, j);
      ss += v * v;
    }
    const float tot = consumer_sum(ss, m);
    const float inv = 1.0f / sqrtf(tot / (float)kvl + od.eps);
    __nv_bfloat16* crow = reinterpret_cast<__nv_bfloat16*>(od.kcache) + (size_t)pos * rowe;
    for (int j = tid; j < kvl; j += kConsumers) {
      const __nv_bfloat16 v = __float2bfloat16_rn(pset(od.ckv, j) * inv * od.kvnorm_g[j]);
      newrow[j] = v;
      if (hg == 0) crow[j] = v;
    }
    for (int j = tid; j < rd / 2; j += kConsumers) {
      const float a = pset(od.ckv, kvl + j), bb = pset(od.ckv, kvl + j + rd / 2);
      const __nv_bfloat16 v0 = __float2bfloat16_rn(a * cosr[j] - bb * sinr[j]);
      const __nv_bfloat16 v1 = __float2bfloat16_rn(a * sinr[j] + bb * cosr[j]);
      newrow[kvl + j] = v0;
      newrow[kvl + j + rd / 2] = v1;
      if (hg == 0) {
        crow[kvl + j] = v0;
        crow[kvl + j + rd / 2] = v1;
      }
    }
  }
  named_bar_sync(1, kConsumers);
  // warp w owns heads w*hpw .. ; lane owns latent dims [lane*dpl, +dpl)
  const int hpw = HG / kConsumerWarps;  // heads per warp (2)
  const int dpl = kvl / 32;             // 16
  float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
  float o[2][16];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int d = 0; d < 16; ++d) o[a][d] = 0.f;
  const int nck = rowb / 16;  // 72
  const int nql = kvl / 8;    // chunks of the latent part
  auto block = [&](const uint8_t* rows, int n) {
    for (int p = tid; p < HG * n; p += kConsumers) {
      const int i = p / n, tt = p % n;
      const uint8_t* row = rows + (size_t)tt * rowb;
      float dot = 0.f;
      for (int j = 0; j < nck; ++j) {
        int jj = j + tt;
        jj = jj % nck;
        const uint4 kv = *reinterpret_cast<const uint4*>(row + jj * 16);
        const float* qq = jj < nql ? ql + i * kvl + jj * 8 : qp + i * rd + (jj - nql) * 8;
        dot = fmaf(bf16lo(kv.x), qq[0], dot);
        dot = fmaf(bf16hi(kv.x), qq[1], dot);
        dot = fmaf(bf16lo(kv.y), qq[2], dot);
        dot = fmaf(bf16hi(kv.y), qq[3], dot);
        dot = fmaf(bf16lo(kv.z), qq[4], dot);
        dot = fmaf(bf16hi(kv.z), qq[5], dot);
        dot = fmaf(bf16lo(kv.w), qq[6], dot);
        dot = fmaf(bf16hi(kv.w), qq[7], dot);
      }
      sc[i * od.np + tt] = dot * od.attn_scale;
    }
    named_bar_sync(1, kConsumers);
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      if (a >= hpw) break;
      float* s = sc + (warp * hpw + a) * od.np;
      float mx = -INFINITY;
      for (int tt = lane; tt < n; tt += 32) mx = fmaxf(mx, s[tt]);
      mx = warp_max(mx);
      const float mnew = fmaxf(mrun[a], mx);
      const float alpha = expf(mrun[a] - mnew);
      float ls = 0.f;
      for (int tt = lane; tt < n; tt += 32) {
        const float pv = expf(s[tt] - mnew);
        s[tt] = pv;
        ls += pv;
      }
      ls = warp_sum(ls);
      __syncwarp();
      lrun[a] = lrun[a] * alpha + ls;
      mrun[a] = mnew;
#pragma unroll
      for (int d = 0; d < 16; ++d) o[a][d] *= alpha;
    }
    for (int tt = 0; tt < n; ++tt) {
      const uint4* cr = reinterpret_cast<const uint4*>(rows + (size_t)tt * rowb + lane * dpl * 2);
      const uint4 c0 = cr[0], c1 = cr[1];
      const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        if (a >= hpw) break;
        const float pv = sc[(warp * hpw + a) * od.np + tt];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          o[a][2 * q] = fmaf(pv, bf16lo(cw[q]), o[a][2 * q]);
          o[a][2 * q + 1] = fmaf(pv, bf16hi(cw[q]), o[a][2 * q + 1]);
        }
      }
    }
    named_bar_sync(1, kConsumers);
  };
  const int nst = (b.tc - b.t0 + od.np - 1) / od.np;
  for (int st = 0; st < nst; ++st) {
    wait_full(P, S, g, op, t);
    const uint8_t* stage = S.ring + (g % kStages) * kStageBytes;
    const int a = b.t0 + st * od.np;
    const int n = (b.tc - a) < od.np ? (b.tc - a) : od.np;
    block(stage, n);
    release_stage(S, g);
    ++g;
  }
  if (b.has_new) block(reinterpret_cast<const uint8_t*>(newrow), 1);
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    if (a >= hpw) break;
    const int h = h0 + warp * hpw + a;
    if (h < od.H) {
      const size_t pi = (size_t)h * od.nch + c;
      if (lane == 0) {
        od.m_out[pi] = mrun[a];
        od.l_out[pi] = lrun[a];
      }
#pragma unroll
      for (int d = 0; d < 16; ++d) od.o_out[pi * kvl + lane * dpl + d] = o[a][d];
    }
  }
  return true;
}

// Final op: greedy token = argmax over the LM-head tasks' best keys; advance the step state.
__device__ bool final_consume(const KParams& P, const OpDesc& od, int op, int t, const Smem& S) {
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
    if (next < 0 || next >= od.vocab) next = 0;  // NaN logits only
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
    *P.state = ns;
  }
  return true;
}

// ------------------------------------------------------------ task lists
struct TaskIter {
  const KParams* P;
  int i, end, op, stride;
  __device__ void init(const KParams& p) {
    P = &p;
    if (p.persistent) {
      i = p.task_off[blockIdx.x];
      end = p.task_off[blockIdx.x + 1];
      stride = 1;
    } else {
      op = p.op_only;
      i = blockIdx.x;
      end = p.ops[op].ntasks;
      stride = gridDim.x;
    }
  }
  __device__ bool next(int& o, int& t) {
    if (i >= end) return false;
    if (P->persistent) {
      const int2 v = P->tasks[i];
      o = v.x;
      t = v.y;
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
  const uint64_t pol_kv = policy_evict_last();  // caches: re-read every step
  uint32_t g = 0;
  TaskIter it;
  it.init(P);
  int op, t;
  const int pos = m->st.pos;
  const unsigned epoch = (unsigned)m->st.epoch;
  auto issue = [&](const void* src, uint32_t bytes, const void* src2, uint32_t bytes2, uint32_t off2,
                   uint64_t pol) -> bool {
    uint64_t* eb = &m->empty[g % kStages];
    const uint32_t par = ((g / kStages) & 1) ^ 1;
    int ready = 1;
    if (lane == 0) ready = bounded_wait([&] { return mbar_try_wait(eb, par); }, P, &m->abort, op, t, false) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ready, 0)) return false;
    if (lane == 0) {
      uint8_t* dst = S.ring + (g % kStages) * kStageBytes;
      uint64_t* fb = &m->full[g % kStages];
      mbar_arrive_expect_tx(fb, bytes + bytes2);
      if (bytes) bulk_g2s(dst, src, bytes, fb, pol);
      if (bytes2) bulk_g2s(dst + off2, src2, bytes2, fb, pol);
    }
    __syncwarp();
    ++g;
    return true;
  };
  bool ok = true;
  while (ok && it.next(op, t)) {
    const OpDesc& od = P.ops[op];
    if (od.kind == OP_GEMV) {
      const TaskGeo geo = gemv_geo(od, t);
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
          warp_route(od.route_logits, od.n_experts, od.top_k, m->prod_idx, nullptr);
          if (lane == 0) {
            m->prod_route_op = od.pdep;
            if (od.route_dump)
              for (int j = 0; j < od.top_k; ++j) od.route_dump[j] = m->prod_idx[j];
          }
          __syncwarp();
        }
        base += (size_t)m->prod_idx[sg.slot] * sg.w_estride;
      }
      const uint32_t sb = (uint32_t)(od.R * od.kcb);
      const uint8_t* tile = base + (size_t)(geo.rt * od.S + geo.s) * od.nst * sb;
      for (int st = 0; st < od.nst && ok; ++st) ok = issue(tile + (size_t)st * sb, sb, nullptr, 0, 0, pol_w);
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
      const int c = t % od.nch;
      const ChunkB b = chunk_bounds(c, od.nch, pos);
      const int rowb = (od.kvl + od.rdim) * 2;
      for (int a = b.t0; a < b.tc && ok; a += od.np) {
        const int n = (b.tc - a) < od.np ? (b.tc - a) : od.np;
        ok = issue((const uint8_t*)od.kcache + (size_t)a * rowb, n * rowb, nullptr, 0, 0, pol_kv);
      }
    }
  }
  if (lane == 0) m->issued = (int)g;
}

// --------------------------------------------------------------- consumer
__device__ void consumer_loop(const KParams& P, const Smem& S) {
  Misc* m = S.m;
  uint32_t g = 0;
  TaskIter it;
  it.init(P);
  int op, t, cur = -1;
  const unsigned epoch = (unsigned)m->st.epoch;
  while (it.next(op, t)) {
    const OpDesc& od = P.ops[op];
    if (op != cur) {
      if (P.persistent && threadIdx.x == 0) {
        if (wait_counter(P, od.dep[0], epoch, &m->abort, op, t)) wait_counter(P, od.dep[1], epoch, &m->abort, op, t);
      }
      // uniform decision: every consumer thread sees the same value
      if (named_bar_or(1, kConsumers, m->abort)) break;
      cur = op;
    }
    const uint64_t t_start = P.trace ? globaltimer() : 0;
    switch (od.kind) {
      case OP_GEMV:
        if (od.wtype == WT_FP8)
          gemv_consume<WT_FP8>(P, od, op, t, S, g);
        else if (od.wtype == WT_BF16)
          gemv_consume<WT_BF16>(P, od, op, t, S, g);
        else
          gemv_consume<WT_F32>(P, od, op, t, S, g);
        break;
      case OP_ATTN:
        attn_consume(P, od, op, t, S, g);
        if (threadIdx.x == 0) m->x_op = -1;
        break;
      case OP_MLA:
        mla_consume(P, od, op, t, S, g);
        if (threadIdx.x == 0) m->x_op = -1;
        break;
      case OP_FINAL:
        final_consume(P, od, op, t, S);
        break;
    }
    // A failed wait anywhere in the task makes every thread stop here, after the
    // task's barriers, without publishing the task.
    if (named_bar_or(1, kConsumers, m->abort)) break;
    if (threadIdx.x == 0) {
      __threadfence();
      red_release_gpu_add(&P.counters[op], 1u);
      if (P.trace) {
        const int slot = atomicAdd(reinterpret_cast<unsigned*>(P.trace), 1u);
        if (slot < P.trace_cap) {
          unsigned long long* r = P.trace + 2 + (size_t)slot * 3;
          r[0] = ((unsigned long long)blockIdx.x << 48) | ((unsigned long long)op << 32) | (unsigned)t;
          r[1] = t_start;
          r[2] = globaltimer();
        }
      }
    }
  }
  if (threadIdx.x == 0) m->consumed = (int)g;
}

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
    m->issued = 0;
    m->consumed = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&m->full[i], 1);
      mbar_init(&m->empty[i], kConsumerWarps);
    }
    fence_mbar_init();
    if (P.persistent) {
      __threadfence();
      atomicAdd(P.started, 1u);
    }
  }
  __syncthreads();
  if (threadIdx.x >= kConsumers)
    producer_loop(P, S);
  else
    consumer_loop(P, S);
  __syncthreads();
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
