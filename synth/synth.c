/*
 * Seeded synthetic inputs for the MXFP4 W4A4 linear layer.
 *
 * This module only draws numbers. It holds none of the layer's arithmetic
 * (no rotation, no scale choice, no rounding to E2M1, no contraction), so the
 * CPU oracle and the CUDA path can both be fed from it without sharing any of
 * the method.
 *
 * Generator: counter-based splitmix64. Draw number `c` of stream
 * (seed, tensor_id) is mix64(origin(seed, tensor_id) + (c + 1) * golden),
 * which is exactly the c-th output of a splitmix64 sequence started at
 * `origin`. Any element can be drawn independently of every other one, so the
 * result does not depend on thread count or iteration order.
 *
 * Normal variates: Box-Muller in double, element i uses draws 2i and 2i+1.
 * Activations: N(0,1) with a chosen set of "outlier" channels multiplied by a
 * factor, rounded to fp32 then to bf16 (round to nearest even), matching the
 * DiT/LLM activation recipe (a small fraction of K-channels carrying large
 * values, the situation the block rotations are meant to handle).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_origin(uint64_t seed, uint64_t tensor_id) {
  return mix64(seed * GOLDEN + tensor_id * 0xD1B54A32D192ED03ULL + 0x2545F4914F6CDD1DULL);
}

static inline uint64_t draw_at(uint64_t origin, uint64_t counter) {
  return mix64(origin + (counter + 1) * GOLDEN);
}

/* 53-bit uniform in [0, 1). */
static inline double unit_uniform(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

static inline double normal_at(uint64_t origin, uint64_t i) {
  double u1 = 1.0 - unit_uniform(draw_at(origin, 2 * i)); /* (0, 1] */
  double u2 = unit_uniform(draw_at(origin, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* fp32 -> bf16 bits, round to nearest even (NaN kept quiet). */
static inline uint16_t bf16_bits_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws (for tests of the generator itself). */
void synth_raw_u64(uint64_t seed, uint64_t tensor_id, int64_t n, uint64_t* out) {
  uint64_t o = stream_origin(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = draw_at(o, (uint64_t)i);
}

/* out[i] = scale * N(0,1)_i, as fp32. */
void synth_normal_f32(uint64_t seed, uint64_t tensor_id, int64_t n, double scale, float* out) {
  uint64_t o = stream_origin(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(scale * normal_at(o, (uint64_t)i));
}

/* out[i] = scale * N(0,1)_i, as double. */
void synth_normal_f64(uint64_t seed, uint64_t tensor_id, int64_t n, double scale, double* out) {
  uint64_t o = stream_origin(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = scale * normal_at(o, (uint64_t)i);
}

/*
 * The first `count` entries of a Fisher-Yates shuffle of 0..K-1, drawn from
 * stream (seed, tensor_id): step i swaps position i with i + floor(u_i * (K - i)).
 */
void synth_outlier_channels(uint64_t seed, uint64_t tensor_id, int64_t K, int64_t count,
                            int32_t* perm_scratch /* K entries */, int32_t* out /* count */) {
  uint64_t o = stream_origin(seed, tensor_id);
  for (int64_t i = 0; i < K; ++i) perm_scratch[i] = (int32_t)i;
  for (int64_t i = 0; i < count && i < K; ++i) {
    int64_t j = i + (int64_t)(unit_uniform(draw_at(o, (uint64_t)i)) * (double)(K - i));
    if (j >= K) j = K - 1;
    int32_t t = perm_scratch[i];
    perm_scratch[i] = perm_scratch[j];
    perm_scratch[j] = t;
    out[i] = perm_scratch[i];
  }
}

/*
 * Activation matrix X[M, K] (row-major, bf16 bits): N(0,1) draws from stream
 * (seed, tensor_id), channels flagged in `is_outlier` (K bytes) multiplied by
 * `factor`, rounded to fp32 then to bf16.
 */
void synth_activation_bf16(uint64_t seed, uint64_t tensor_id, int64_t M, int64_t K,
                           const uint8_t* is_outlier, double factor, uint16_t* out) {
  uint64_t o = stream_origin(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      double v = normal_at(o, (uint64_t)(m * K + k));
      if (is_outlier[k]) v *= factor;
      out[m * K + k] = bf16_bits_rne((float)v);
    }
  }
}

/* fp32 -> bf16 bits for an arbitrary array (round to nearest even). */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_rne(in[i]);
}

/* Uniform integers in [lo, hi] as bytes (random codes / scale bytes). */
void synth_uniform_u8(uint64_t seed, uint64_t tensor_id, int64_t n, int lo, int hi, uint8_t* out) {
  uint64_t o = stream_origin(seed, tensor_id);
  double span = (double)(hi - lo + 1);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    int v = lo + (int)(unit_uniform(draw_at(o, (uint64_t)i)) * span);
    if (v > hi) v = hi;
    out[i] = (uint8_t)v;
  }
}
