// Seeded synthetic inputs, GPU side.
//
// Draws the same values as synth.c (SplitMix64 counter streams, Irwin-Hall(4)
// of the four 16-bit fields, one fp32 multiply and one fp32 add; block-FP8
// quantisation per 128x128 block with E4M3 round-to-nearest-even and
// saturation).  It is an independent implementation of the published
// generator, used to fill device buffers for workloads whose weights do not
// fit in host memory.  It holds none of the decode arithmetic.
//
// All entry points are asynchronous on the given stream and return a
// cudaError_t value cast to int (0 = success).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float irwin_hall4(uint64_t s0, uint64_t i, float c, float offset) {
  uint64_t h = mix64(s0 + (i + 1) * kGamma);
  int n = (int)(h & 0xFFFF) + (int)((h >> 16) & 0xFFFF) + (int)((h >> 32) & 0xFFFF) + (int)((h >> 48) & 0xFFFF) -
          131070;
  // Separate roundings (no contraction) so the CPU side can reproduce them.
  return __fadd_rn(offset, __fmul_rn((float)n, c));
}

__global__ void k_normal_f32(uint64_t s0, uint64_t start, uint64_t n, float c, float offset, float* out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n; j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = irwin_hall4(s0, start + j, c, offset);
}

__device__ __forceinline__ uint16_t bf16_rne(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__global__ void k_normal_bf16(uint64_t s0, uint64_t start, uint64_t n, float c, float offset, uint16_t* out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n; j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = bf16_rne(irwin_hall4(s0, start + j, c, offset));
}

__device__ __forceinline__ uint8_t e4m3_rne_sat(float x) {
  uint16_t r;
  // Hardware conversion: round to nearest even, saturate to the largest finite value.
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return (uint8_t)(r & 0xFF);
}

// One CTA of 256 threads per 128x128 block.
__global__ void __launch_bounds__(256) k_fp8_b128(uint64_t s0, int64_t rows, int64_t cols, float c, uint8_t* q,
                                                  float* scales) {
  const int64_t nbc = (cols + 127) / 128;
  const int64_t br = blockIdx.x / nbc, bc = blockIdx.x % nbc;
  const int64_t r0 = br * 128, c0 = bc * 128;
  const int nr = (int)(rows - r0 < 128 ? rows - r0 : 128), nc = (int)(cols - c0 < 128 ? cols - c0 : 128);
  float v[64];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    int idx = threadIdx.x + 256 * j;
    int r = idx >> 7, cc = idx & 127;
    v[j] = 0.f;
    if (r < nr && cc < nc) {
      v[j] = irwin_hall4(s0, (uint64_t)((r0 + r) * cols + c0 + cc), c, 0.0f);
      amax = fmaxf(amax, fabsf(v[j]));
    }
  }
  __shared__ float red[8];
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
  const float s = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
  if (threadIdx.x == 0) scales[blockIdx.x] = s;
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    int idx = threadIdx.x + 256 * j;
    int r = idx >> 7, cc = idx & 127;
    if (r < nr && cc < nc) q[(r0 + r) * cols + c0 + cc] = e4m3_rne_sat(__fdiv_rn(v[j], s));
  }
}

__global__ void k_tokens(uint64_t s0, uint64_t start, uint64_t n, uint32_t vocab, int32_t* out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n; j += (uint64_t)gridDim.x * blockDim.x)
    out[j] = (int32_t)(mix64(s0 + (start + j + 1) * kGamma) % vocab);
}

inline unsigned grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  return (unsigned)(g < 148 * 32 ? (g == 0 ? 1 : g) : 148 * 32);
}

}  // namespace

extern "C" {

uint64_t synthc_stream(uint64_t seed, uint64_t tid) { return mix64((seed << 32) + tid); }

int synthc_normal_f32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, float c, float offset, float* out,
                      void* stream) {
  if (n == 0) return 0;
  k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(synthc_stream(seed, tid), start, n, c, offset, out);
  return (int)cudaGetLastError();
}

int synthc_normal_bf16(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, float c, float offset, uint16_t* out,
                       void* stream) {
  if (n == 0) return 0;
  k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(synthc_stream(seed, tid), start, n, c, offset, out);
  return (int)cudaGetLastError();
}

int synthc_fp8_b128(uint64_t seed, uint64_t tid, int64_t rows, int64_t cols, float c, uint8_t* q, float* scales,
                    void* stream) {
  int64_t nb = ((rows + 127) / 128) * ((cols + 127) / 128);
  if (nb == 0) return 0;
  k_fp8_b128<<<(unsigned)nb, 256, 0, (cudaStream_t)stream>>>(synthc_stream(seed, tid), rows, cols, c, q, scales);
  return (int)cudaGetLastError();
}

int synthc_tokens(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, uint32_t vocab, int32_t* out,
                  void* stream) {
  if (n == 0) return 0;
  k_tokens<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(synthc_stream(seed, tid), start, n, vocab, out);
  return (int)cudaGetLastError();
}

}  // extern "C"
