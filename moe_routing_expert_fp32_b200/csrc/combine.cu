// combine.cu -- unpermute and weighted combine of the expert outputs.
//
// Follows "Kimi K3 · Add shared output", moe-forward excerpt (moe_infer):
// new_x[idxs] = outs, then new_x.view(N, K, d).type(fp32).mul_(w).sum(dim=1)
// .type(bf16).  The scatter into new_x is not materialised: token t reads its
// K rows straight from y through pos[t*K + k].  Products are rounded to fp32
// (__fmul_rn) and summed in k order (__fadd_rn), then rounded once to bf16.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

// One warp per (token, chunk of 256 columns): lane l handles the 8 columns of
// 16-byte vector c*32 + l, so even a decode batch of 128 tokens spreads over
// thousands of warps.
__global__ void __launch_bounds__(32 * kWarps) k_combine(const __nv_bfloat16* __restrict__ y,
                                                         const int32_t* __restrict__ pos,
                                                         const float* __restrict__ w, int64_t N,
                                                         int K, int d, int64_t S,
                                                         __nv_bfloat16* __restrict__ out,
                                                         DeviceStatus* st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  const int nch = (nv + 31) / 32;
  const int64_t items = N * nch;
  for (int64_t it = (int64_t)blockIdx.x * kWarps + warp; it < items;
       it += (int64_t)gridDim.x * kWarps) {
    const int64_t t = it / nch;
    const int v = (int)(it - t * nch) * 32 + lane;
    int my_p = -1;
    float my_w = 0.f;
    if (lane < K) {
      my_p = pos[t * K + lane];
      my_w = w[t * K + lane];
      if (my_p < 0 || my_p >= S) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 40);
        my_p = -1;
      }
    }
    float acc[8];
    bool have = false;
    for (int k = 0; k < K; ++k) {
      const int p = __shfl_sync(0xffffffffu, my_p, k);
      const float wk = __shfl_sync(0xffffffffu, my_w, k);
      if (p < 0 || v >= nv) continue;
      const uint4 raw = reinterpret_cast<const uint4*>(y + (int64_t)p * d)[v];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        const float p0 = __fmul_rn(f.x, wk), p1 = __fmul_rn(f.y, wk);
        if (have) {
          acc[2 * j] = __fadd_rn(acc[2 * j], p0);
          acc[2 * j + 1] = __fadd_rn(acc[2 * j + 1], p1);
        } else {
          acc[2 * j] = p0;
          acc[2 * j + 1] = p1;
        }
      }
      have = true;
    }
    if (v >= nv) continue;
    if (!have) {
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    }
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) o2[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    reinterpret_cast<uint4*>(out + t * d)[v] = o;
  }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* pos, const float* w, int64_t N,
                           int K, int d_e, int64_t S, __nv_bfloat16* out, DeviceStatus* st,
                           cudaStream_t s) {
  const int64_t items = N * ((d_e / 8 + 31) / 32);
  int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  if (blocks > cap) blocks = cap;
  k_combine<<<(unsigned)blocks, 32 * kWarps, 0, s>>>(y, pos, w, N, K, d_e, S, out, st);
  return cudaGetLastError();
}

}  // namespace moe
