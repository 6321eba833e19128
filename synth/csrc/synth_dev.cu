// synth_dev.cu -- device twin of the synthetic input generator (definition in
// synth.h).  Every fp32 operation is an explicit round-to-nearest intrinsic so
// that the compiler cannot fuse a multiply into an add; the result is
// bit-identical to synth_host.c.  Grid-stride kernels sized to the SM count.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "synth.h"

namespace {

__host__ __device__ __forceinline__ uint64_t mix64_hd(uint64_t z) {
  z ^= z >> 30; z *= SYNTH_M1;
  z ^= z >> 27; z *= SYNTH_M2;
  return z ^ (z >> 31);
}

uint64_t tensor_key(uint64_t seed, uint32_t tensor_id) {
  return mix64_hd(mix64_hd(seed + SYNTH_GAMMA) + ((uint64_t)tensor_id + 1ULL) * SYNTH_GAMMA);
}

__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t i, uint64_t j) {
  return mix64_hd(key + (2ULL * i + j + 1ULL) * SYNTH_GAMMA);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i, float sigma) {
  const uint64_t a = draw(key, i, 0), b = draw(key, i, 1);
  int32_t s = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    s += (int32_t)((a >> (16 * q)) & 0xFFFFu);
    s += (int32_t)((b >> (16 * q)) & 0xFFFFu);
  }
  const float z = __int2float_rn(s - SYNTH_IH8_CENTER);
  return __fmul_rn(__fmul_rn(z, SYNTH_IH8_SCALE), sigma);
}

template <typename T>
__global__ void k_normal(uint64_t key, uint64_t start, int64_t count, float sigma, T* out) {
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < count;
       n += (int64_t)gridDim.x * blockDim.x) {
    const float v = normal_at(key, start + (uint64_t)n, sigma);
    if constexpr (sizeof(T) == 2) out[n] = __float2bfloat16_rn(v);
    else out[n] = v;
  }
}

__global__ void k_uniform(uint64_t key, uint64_t start, int64_t count, float lo, float hi,
                          float* out) {
  const float span = __fsub_rn(hi, lo);
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < count;
       n += (int64_t)gridDim.x * blockDim.x) {
    const float t = __fmul_rn(__ull2float_rn(draw(key, start + (uint64_t)n, 0) >> 40), 0x1p-24f);
    out[n] = __fadd_rn(lo, __fmul_rn(span, t));
  }
}

int grid_for(int64_t count) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (count + 255) / 256;
  int64_t cap = (int64_t)sms * 8;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

extern "C" {

int synth_dev_normal_bf16(uint64_t seed, uint32_t tensor_id, uint64_t start, int64_t count,
                          float sigma, void* out, void* stream) {
  if (count <= 0) return 0;
  k_normal<__nv_bfloat16><<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      tensor_key(seed, tensor_id), start, count, sigma, (__nv_bfloat16*)out);
  return (int)cudaGetLastError();
}

int synth_dev_normal_f32(uint64_t seed, uint32_t tensor_id, uint64_t start, int64_t count,
                         float sigma, void* out, void* stream) {
  if (count <= 0) return 0;
  k_normal<float><<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      tensor_key(seed, tensor_id), start, count, sigma, (float*)out);
  return (int)cudaGetLastError();
}

int synth_dev_uniform_f32(uint64_t seed, uint32_t tensor_id, uint64_t start, int64_t count,
                          float lo, float hi, void* out, void* stream) {
  if (count <= 0) return 0;
  k_uniform<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      tensor_key(seed, tensor_id), start, count, lo, hi, (float*)out);
  return (int)cudaGetLastError();
}

}  // extern "C"
