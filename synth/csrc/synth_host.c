/*
 * synth_host.c -- host twin of the synthetic input generator (definition in
 * synth.h).  Must stay bit-identical to synth_dev.cu; the test suite checks
 * that on the GPU.  Compiled with -ffp-contract=off so that no multiply-add is
 * fused: every fp32 operation here is one correctly rounded IEEE operation.
 */
#include <stdint.h>
#include <string.h>
#include "synth.h"

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30; z *= SYNTH_M1;
  z ^= z >> 27; z *= SYNTH_M2;
  return z ^ (z >> 31);
}

static inline uint64_t tensor_key(uint64_t seed, uint32_t tensor_id) {
  return mix64(mix64(seed + SYNTH_GAMMA) + ((uint64_t)tensor_id + 1ULL) * SYNTH_GAMMA);
}

static inline uint64_t draw(uint64_t key, uint64_t i, uint64_t j) {
  return mix64(key + (2ULL * i + j + 1ULL) * SYNTH_GAMMA);
}

static inline int32_t ih8_sum(uint64_t a, uint64_t b) {
  int32_t s = 0;
  for (int q = 0; q < 4; ++q) {
    s += (int32_t)((a >> (16 * q)) & 0xFFFFu);
    s += (int32_t)((b >> (16 * q)) & 0xFFFFu);
  }
  return s - SYNTH_IH8_CENTER;
}

static inline float normal_at(uint64_t key, uint64_t i, float sigma) {
  float z = (float)ih8_sum(draw(key, i, 0), draw(key, i, 1));
  float t = z * SYNTH_IH8_SCALE;
  return t * sigma;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void synth_host_normal_f32(uint64_t seed, uint32_t tensor_id, uint64_t start,
                           int64_t count, float sigma, float* out) {
  const uint64_t key = tensor_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < count; ++n) out[n] = normal_at(key, start + (uint64_t)n, sigma);
}

void synth_host_normal_bf16(uint64_t seed, uint32_t tensor_id, uint64_t start,
                            int64_t count, float sigma, uint16_t* out) {
  const uint64_t key = tensor_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < count; ++n)
    out[n] = f32_to_bf16_rne(normal_at(key, start + (uint64_t)n, sigma));
}

void synth_host_uniform_f32(uint64_t seed, uint32_t tensor_id, uint64_t start,
                            int64_t count, float lo, float hi, float* out) {
  const uint64_t key = tensor_key(seed, tensor_id);
  float span = hi - lo;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < count; ++n) {
    float t = (float)(draw(key, start + (uint64_t)n, 0) >> 40) * 0x1p-24f;
    float p = span * t;
    out[n] = lo + p;
  }
}

/* Raw 64-bit draws, exported so that tests can check the stream itself. */
void synth_host_raw(uint64_t seed, uint32_t tensor_id, uint64_t start, int64_t count,
                    uint64_t* out) {
  const uint64_t key = tensor_key(seed, tensor_id);
  for (int64_t n = 0; n < count; ++n) out[n] = draw(key, start + (uint64_t)n, 0);
}
