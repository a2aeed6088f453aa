// Split-KV decode attention that allocates no device memory.
//
// Some callers cannot call cudaMalloc: code running while a CUDA graph is being
// captured, runtimes whose device memory is owned by an outside allocator that
// forbids allocations on the serving path, or embedders that must keep a fixed
// memory footprint after start-up.  dec_attention_noalloc gives them the split-KV
// attention of the decode step (the same split into position chunks, the same
// online softmax per chunk and log-sum-exp combine) with its per-chunk partials
// kept in a fixed array compiled into the library instead of a buffer allocated
// per call.  Every GPU that loads the library holds that array (2 MiB) until the
// process exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/dec.h"

namespace {

constexpr int kScratchFloats = 1 << 19;  // 2 MiB: heads * chunks * (head_dim + 2) floats at most
constexpr int kMaxDevices = 64;
constexpr int kTile = 32;                // positions staged in shared memory at a time
constexpr int kThreadsP = 256;

// Per-chunk partials of every call: max [H][C], sum [H][C], weighted values [H][C][D].
static __device__ __align__(256) float g_attn_scratch[kScratchFloats];

float* g_scratch_addr[kMaxDevices];
bool g_ready[kMaxDevices];
std::mutex g_mu;

__device__ __forceinline__ float warp_max_(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One block per (kv head, chunk): online softmax over the chunk's positions for the
// gs query heads that share the kv head; writes (m, l, o) per head to the scratch.
__global__ void __launch_bounds__(kThreadsP) attn_partial(const float* __restrict__ q, const __nv_bfloat16* kc,
                                                          const __nv_bfloat16* vc, int H, int Hkv, int D, int n_pos,
                                                          int stride, int nch, float scale, float* scratch) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int gs = H / Hkv;
  const int kvh = blockIdx.x / nch, c = blockIdx.x % nch;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* q_s = reinterpret_cast<float*>(sm);                                  // [gs][D]
  __nv_bfloat16* k_s = reinterpret_cast<__nv_bfloat16*>(q_s + gs * D);      // [kTile][D]
  __nv_bfloat16* v_s = k_s + kTile * D;                                       // [kTile][D]
  float* sc = reinterpret_cast<float*>(v_s + kTile * D);                      // [gs][kTile]
  const int t0 = (int)((long long)c * n_pos / nch), t1 = (int)((long long)(c + 1) * n_pos / nch);
  for (int e = tid; e < gs * D; e += kThreadsP) q_s[e] = q[(size_t)(kvh * gs) * D + e];
  const int dpl = D / 32;
  float mrun = -INFINITY, lrun = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  const __nv_bfloat16* kbase = kc + (size_t)kvh * stride * D;
  const __nv_bfloat16* vbase = vc + (size_t)kvh * stride * D;
  for (int a = t0; a < t1; a += kTile) {
    const int n = (t1 - a) < kTile ? (t1 - a) : kTile;
    __syncthreads();
    const int vec = n * D / 8;  // 16-byte pieces per tile
    for (int i = tid; i < vec; i += kThreadsP) {
      reinterpret_cast<uint4*>(k_s)[i] = reinterpret_cast<const uint4*>(kbase + (size_t)a * D)[i];
      reinterpret_cast<uint4*>(v_s)[i] = reinterpret_cast<const uint4*>(vbase + (size_t)a * D)[i];
    }
    __syncthreads();
    for (int p = tid; p < gs * n; p += kThreadsP) {
      const int i = p / n, tt = p % n;
      float dot = 0.f;
      for (int j = 0; j < D; ++j) dot = fmaf(__bfloat162float(k_s[tt * D + j]), q_s[i * D + j], dot);
      sc[i * kTile + tt] = dot * scale;
    }
    __syncthreads();
    if (warp < gs) {
      float* s = sc + warp * kTile;
      float mx = -INFINITY;
      for (int tt = lane; tt < n; tt += 32) mx = fmaxf(mx, s[tt]);
      mx = warp_max_(mx);
      const float mnew = fmaxf(mrun, mx);
      const float alpha = expf(mrun - mnew);
      float ls = 0.f;
      for (int tt = lane; tt < n; tt += 32) {
        const float pv = expf(s[tt] - mnew);
        s[tt] = pv;
        ls += pv;
      }
      ls = warp_sum_(ls);
      __syncwarp();
      lrun = lrun * alpha + ls;
      mrun = mnew;
      for (int d = 0; d < dpl; ++d) o[d] *= alpha;
      for (int tt = 0; tt < n; ++tt) {
        const float pv = s[tt];
        for (int d = 0; d < dpl; ++d) o[d] = fmaf(pv, __bfloat162float(v_s[tt * D + lane * dpl + d]), o[d]);
      }
    }
  }
  if (warp < gs) {
    const int h = kvh * gs + warp;
    float* m_out = scratch;
    float* l_out = scratch + (size_t)H * nch;
    float* o_out = scratch + (size_t)2 * H * nch;
    const size_t pi = (size_t)h * nch + c;
    if (lane == 0) {
      m_out[pi] = mrun;
      l_out[pi] = lrun;
    }
    for (int d = 0; d < dpl; ++d) o_out[pi * D + lane * dpl + d] = o[d];
  }
}

// One block per query head: out = sum_c e^(m_c - M) o_c / sum_c e^(m_c - M) l_c.
__global__ void attn_combine(int H, int D, int nch, const float* scratch, float* out) {
  __shared__ float w[64];
  const int h = blockIdx.x, tid = threadIdx.x;
  const float* m_in = scratch;
  const float* l_in = scratch + (size_t)H * nch;
  const float* o_in = scratch + (size_t)2 * H * nch;
  if (tid < 32) {
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    if (tid < nch) {
      m0 = m_in[h * nch + tid];
      l0 = l_in[h * nch + tid];
    }
    if (tid + 32 < nch) {
      m1 = m_in[h * nch + tid + 32];
      l1 = l_in[h * nch + tid + 32];
    }
    const float M = warp_max_(fmaxf(l0 > 0.f ? m0 : -INFINITY, l1 > 0.f ? m1 : -INFINITY));
    const float e0 = l0 > 0.f ? expf(m0 - M) : 0.f, e1 = l1 > 0.f ? expf(m1 - M) : 0.f;
    const float den = warp_sum_(e0 * l0 + e1 * l1);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (tid < nch) w[tid] = e0 * inv;
    if (tid + 32 < nch) w[tid + 32] = e1 * inv;
  }
  __syncthreads();
  for (int d = tid; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < nch; ++c) acc = fmaf(w[c], o_in[((size_t)h * nch + c) * D + d], acc);
    out[(size_t)h * D + d] = acc;
  }
}

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DEC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ready[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return DEC_ERR_CUDA;
    }
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_ready[dev] = true;
  }
  *out = g_scratch_addr[dev];
  return DEC_OK;
}

}  // namespace

extern "C" int dec_attention_noalloc(const float* q, const void* k_cache, const void* v_cache, int32_t n_heads,
                                     int32_t n_kv_heads, int32_t head_dim, int32_t n_pos, int32_t cache_stride,
                                     float* out, void* stream) {
  if (!q || !k_cache || !v_cache || !out) return DEC_ERR_INVALID_ARG;
  // K and V rows are read with 16-byte loads; q and out with 4-byte ones
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15) return DEC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 3) return DEC_ERR_INVALID_ARG;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads || n_heads / n_kv_heads > 8) return DEC_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return DEC_ERR_INVALID_ARG;
  if (n_pos < 1 || cache_stride < n_pos) return DEC_ERR_INVALID_ARG;
  // About one block per SM of a B200, at most 64 chunks (one warp combines them).  With
  // n_kv_heads <= 148 this keeps n_heads * nch <= 8 * 148 rows of partials, far inside the
  // scratch; only very many kv heads (nch = 1) can exceed it.
  int nch = 148 / n_kv_heads;
  if (nch < 1) nch = 1;
  if (nch > 64) nch = 64;
  if (nch > n_pos) nch = n_pos;
  if ((long long)n_heads * nch * (head_dim + 2) > kScratchFloats) return DEC_ERR_CAPACITY;
  // A launch error of this call must not be confused with one the caller left pending.
  if (cudaPeekAtLastError() != cudaSuccess) return DEC_ERR_CUDA;
  float* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc) return rc;
  const int gs = n_heads / n_kv_heads;
  const size_t smem = (size_t)gs * head_dim * 4 + 2 * (size_t)kTile * head_dim * 2 + (size_t)gs * kTile * 4;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  attn_partial<<<n_kv_heads * nch, kThreadsP, smem, s>>>(
      q, static_cast<const __nv_bfloat16*>(k_cache), static_cast<const __nv_bfloat16*>(v_cache), n_heads, n_kv_heads,
      head_dim, n_pos, cache_stride, nch, 1.0f / sqrtf((float)head_dim), scratch);
  if (cudaGetLastError() != cudaSuccess) return DEC_ERR_CUDA;
  attn_combine<<<n_heads, 128, 0, s>>>(n_heads, head_dim, nch, scratch, out);
  if (cudaGetLastError() != cudaSuccess) return DEC_ERR_CUDA;
  return DEC_OK;
}
