/*
 * Seeded synthetic inputs for the MoE FFN layer.
 *
 * This file is the ONE module that both the CUDA path (through the tests and
 * the benchmark) and the f64 oracle draw their inputs from.  It holds no step
 * of the MoE method: it only turns (seed, stream, index) into numbers and
 * rounds them to the storage formats the layer consumes (f32, bf16, fp16
 * scales and GGML-style Q8_0 blocks).
 *
 * Generator (counter based, so any element can be produced independently and
 * in parallel):
 *   mix64(z)        = the splitmix64 finaliser (Steele, Lea, Flood, "Fast
 *                     splittable pseudorandom number generators", OOPSLA 2014)
 *   key(seed, s)    = mix64(seed + (s + 1) * GAMMA)
 *   bits(key, n)    = mix64(key + (n + 1) * GAMMA)
 *   uniform01(a)    = ((a >> 11) + 0.5) * 2^-53            in (0, 1)
 *   normal(2j)      = sqrt(-2 ln u1) * cos(2 pi u2)        (Box-Muller: both
 *   normal(2j + 1)  = sqrt(-2 ln u1) * sin(2 pi u2)         outputs of pair j),
 *                     u1 = uniform01(bits(key, 2j)), u2 = uniform01(bits(key, 2j + 1))
 * Samples are computed in double and rounded once to f32; bf16 and fp16 values
 * are then rounded to nearest-even from that f32 sample.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(seed + (stream + 1) * GAMMA);
}

static inline double uniform01(uint64_t key, uint64_t n) {
  uint64_t a = mix64(key + (n + 1) * GAMMA);
  return ((double)(a >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Both Box-Muller outputs of pair j: z[0] = element 2j, z[1] = element 2j + 1. */
static inline void normal_pair(uint64_t key, uint64_t j, double* z) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = uniform01(key, 2 * j);
  double u2 = uniform01(key, 2 * j + 1);
  double r = sqrt(-2.0 * log(u1));
  double s, c;
  sincos(two_pi * u2, &s, &c);
  z[0] = r * c;
  z[1] = r * s;
}

/* f32 -> bf16, round to nearest even (finite inputs only; NaN kept quiet). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline uint16_t f32_to_f16_rne(float f) {
  _Float16 h = (_Float16)f; /* IEEE conversion, round to nearest even */
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

/* n samples of N(mean, std) as f32. */
void gen_normal_f32(uint64_t seed, uint64_t stream, double mean, double std, int64_t n, float* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (n + 1) / 2; ++j) {
    double z[2];
    normal_pair(key, (uint64_t)j, z);
    out[2 * j] = (float)(mean + std * z[0]);
    if (2 * j + 1 < n) out[2 * j + 1] = (float)(mean + std * z[1]);
  }
}

/* n samples of N(mean, std): f32 sample, then bf16 (RNE) bit patterns. */
void gen_normal_bf16(uint64_t seed, uint64_t stream, double mean, double std, int64_t n, uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (n + 1) / 2; ++j) {
    double z[2];
    normal_pair(key, (uint64_t)j, z);
    out[2 * j] = f32_to_bf16_rne((float)(mean + std * z[0]));
    if (2 * j + 1 < n) out[2 * j + 1] = f32_to_bf16_rne((float)(mean + std * z[1]));
  }
}

/* n samples of U[lo, hi) as f32. */
void gen_uniform_f32(uint64_t seed, uint64_t stream, double lo, double hi, int64_t n, float* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(lo + (hi - lo) * uniform01(key, (uint64_t)i));
}

/*
 * GGML-style Q8_0 blocks for a [rows, cols] matrix (cols % 32 == 0), row-major
 * along the input dimension: each block is 34 bytes, {fp16 d; int8 q[32]}.
 * q ~ U{q_lo..q_hi} (integers, inclusive), d ~ U[d_lo, d_hi) rounded to fp16.
 */
void gen_q8_0_blocks(uint64_t seed, uint64_t stream, int64_t rows, int64_t cols, int q_lo, int q_hi,
                     double d_lo, double d_hi, uint8_t* out) {
  uint64_t kq = stream_key(seed, 2 * stream);
  uint64_t kd = stream_key(seed, 2 * stream + 1);
  int64_t nb = cols / 32;
  uint64_t span = (uint64_t)(q_hi - q_lo + 1);
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < rows * nb; ++b) {
    uint8_t* blk = out + b * 34;
    uint16_t d = f32_to_f16_rne((float)(d_lo + (d_hi - d_lo) * uniform01(kd, (uint64_t)b)));
    memcpy(blk, &d, 2);
    for (int j = 0; j < 32; ++j) {
      uint64_t a = mix64(kq + ((uint64_t)(b * 32 + j) + 1) * GAMMA);
      int q = q_lo + (int)(a % span);
      blk[2 + j] = (uint8_t)(int8_t)q;
    }
  }
}

/* Round an f32 array to bf16 bit patterns (RNE). */
void round_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}
