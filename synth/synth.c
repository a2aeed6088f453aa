/*
 * Seeded synthetic inputs, CPU side.
 *
 * This file draws the weights, norm gains, token ids and prefilled caches of
 * the synthetic decode workloads.  It holds none of the decode arithmetic:
 * it only makes inputs.  The GPU side (synth_cuda.cu) implements the same
 * published generator independently; tests check that both produce the same
 * bytes.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-style:
 *   mix64(z)       = the SplitMix64 output finaliser
 *   s0(seed, tid)  = mix64(seed * 2^32 + tid)       one stream per tensor
 *   draw(s0, i)    = mix64(s0 + (i + 1) * GAMMA)    i-th output of the stream
 * A value is Irwin-Hall(4) of the four 16-bit fields of draw(s0, i):
 *   n = u0 + u1 + u2 + u3 - 131070   (integer, exact in fp32)
 *   v = offset + (float)n * c        (one fp32 multiply, one fp32 add)
 * with c chosen by the caller (std / sqrt((65536^2 - 1) / 3), rounded once to
 * fp32), so v is approximately N(offset, std^2).
 *
 * Block-FP8 weights are quantised once, here, per 128x128 block of the
 * row-major [rows][cols] matrix (edge blocks clipped):
 *   amax = max |v|,  s = amax / 448 (s = 1 when amax == 0),
 *   q    = E4M3 round-to-nearest-even, saturated to +-448, of v / s.
 * The decoders (GPU path and oracle) only ever see q and s.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t synth_stream(uint64_t seed, uint64_t tid) { return synth_mix64((seed << 32) + tid); }

uint64_t synth_draw(uint64_t s0, uint64_t i) { return synth_mix64(s0 + (i + 1) * GAMMA); }

static inline float irwin_hall4(uint64_t h, float c, float offset) {
  int32_t n = (int32_t)(h & 0xFFFF) + (int32_t)((h >> 16) & 0xFFFF) + (int32_t)((h >> 32) & 0xFFFF) +
              (int32_t)((h >> 48) & 0xFFFF) - 131070;
  float v = (float)n * c;
  return offset + v;
}

void synth_normal_f32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, float c, float offset,
                      float* out) {
  uint64_t s0 = synth_stream(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)n; ++j) out[j] = irwin_hall4(synth_draw(s0, start + (uint64_t)j), c, offset);
}

/* fp32 -> bf16, round to nearest even (finite inputs). */
uint16_t synth_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void synth_normal_bf16(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, float c, float offset,
                       uint16_t* out) {
  uint64_t s0 = synth_stream(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)n; ++j)
    out[j] = synth_bf16_rne(irwin_hall4(synth_draw(s0, start + (uint64_t)j), c, offset));
}

/* fp32 -> E4M3 ("fn" variant: bias 7, no infinities, 0x7F/0xFF = NaN),
 * round to nearest even, magnitudes above 448 saturate to 448. */
uint8_t synth_e4m3_rne(float x) {
  uint8_t sign = (uint8_t)(signbit(x) ? 0x80 : 0x00);
  float a = fabsf(x);
  if (isnan(x)) return 0x7F;
  if (a > 448.0f) return sign | 0x7E;
  if (a < 0.015625f) { /* below 2^-6: subnormal grid of 2^-9 */
    float m = nearbyintf(a * 512.0f); /* exact scaling; ties to even in the default mode */
    return sign | (uint8_t)m;         /* m == 8 encodes the smallest normal */
  }
  int e;
  float fr = frexpf(a, &e); /* a = fr * 2^e, fr in [0.5, 1) */
  float mant = fr * 2.0f;   /* [1, 2), exponent e - 1 */
  int ex = e - 1;
  float m = nearbyintf((mant - 1.0f) * 8.0f);
  if (m == 8.0f) {
    m = 0.0f;
    ex += 1;
  }
  int code = ((ex + 7) << 3) | (int)m;
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

void synth_fp8_b128(uint64_t seed, uint64_t tid, int64_t rows, int64_t cols, float c, uint8_t* q,
                    float* scales) {
  uint64_t s0 = synth_stream(seed, tid);
  int64_t nbr = (rows + 127) / 128, nbc = (cols + 127) / 128;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < nbr * nbc; ++b) {
    int64_t br = b / nbc, bc = b % nbc;
    int64_t r0 = br * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
    int64_t c0 = bc * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
    float vals[128 * 128];
    float amax = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t cc = c0; cc < c1; ++cc) {
        float v = irwin_hall4(synth_draw(s0, (uint64_t)(r * cols + cc)), c, 0.0f);
        vals[(r - r0) * 128 + (cc - c0)] = v;
        float av = fabsf(v);
        if (av > amax) amax = av;
      }
    float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scales[br * nbc + bc] = s;
    for (int64_t r = r0; r < r1; ++r)
      for (int64_t cc = c0; cc < c1; ++cc) q[r * cols + cc] = synth_e4m3_rne(vals[(r - r0) * 128 + (cc - c0)] / s);
  }
}

void synth_tokens(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, uint32_t vocab, int32_t* out) {
  uint64_t s0 = synth_stream(seed, tid);
  for (uint64_t j = 0; j < n; ++j) out[j] = (int32_t)(synth_draw(s0, start + j) % vocab);
}
