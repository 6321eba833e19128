// combine.cu -- unpermute and weighted combine of the expert outputs.
//
// Follows "Kimi K3 · Add shared output", moe-forward excerpt (moe_infer):
// new_x[idxs] = outs, then new_x.view(N, K, d).type(fp32).mul_(w).sum(dim=1)
// .type(bf16).  Token t's K rows come either straight from the sorted y
// through pos[t*K + k] (the scatter into new_x is not materialised), or, when
// the expert MLP's last GEMM has already written y in slot order (new_x
// itself), from rows t*K .. t*K+K-1 (pos == nullptr).  Products are rounded
// to fp32 (__fmul_rn) and summed in k order (__fadd_rn), then rounded once to
// bf16.
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
                                                         const __nv_bfloat16* __restrict__ res,
                                                         DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
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
      my_p = pos ? pos[t * K + lane] : (int)(t * K + lane);
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
    if (res) {
      // the combined row is a bf16 tensor before the residual add
      const uint4 rr = reinterpret_cast<const uint4*>(res + t * d)[v];
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(r2[j]);
        acc[2 * j] = __fadd_rn(__bfloat162float(__float2bfloat16_rn(acc[2 * j])), f.x);
        acc[2 * j + 1] = __fadd_rn(__bfloat162float(__float2bfloat16_rn(acc[2 * j + 1])), f.y);
      }
    }
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) o2[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    reinterpret_cast<uint4*>(out + t * d)[v] = o;
  }
}

// The same combine with every lane issuing the loads of all KK = K rows of
// its 16-byte column before it sums any of them, so each warp has K loads in
// flight instead of one.  Row k of token t is pos[t*K + k] (the sorted y), or
// t*K + k when pos is NULL (y in slot order, as moe_expert_ffn_to_slots
// writes it).  Rows are skipped and reported exactly as in k_combine, and the
// arithmetic is k_combine's (products rounded to fp32, summed in k order), so
// the result is the same bits.  KK is 4, 8 or 16.
template <int KK>
__global__ void __launch_bounds__(32 * kWarps) k_combine_rows(
    const __nv_bfloat16* __restrict__ y, const int32_t* __restrict__ pos,
    const float* __restrict__ w, int64_t N, int d, int64_t S, __nv_bfloat16* __restrict__ out,
    const __nv_bfloat16* __restrict__ res, DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  const int nch = (nv + 31) / 32;
  const int64_t items = N * nch;
  for (int64_t it = (int64_t)blockIdx.x * kWarps + warp; it < items;
       it += (int64_t)gridDim.x * kWarps) {
    const int64_t t = it / nch;
    const int v = (int)(it - t * nch) * 32 + lane;
    // the K rows and weights go to every lane before any lane leaves the item
    int my_p = -1;
    float my_w = 0.f;
    if (lane < KK) {
      my_p = pos ? pos[t * KK + lane] : (int)(t * KK + lane);
      my_w = w[t * KK + lane];
      if (my_p < 0 || my_p >= S) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 41);
        my_p = -1;
      }
    }
    int rk[KK];
    float wks[KK];
#pragma unroll
    for (int k = 0; k < KK; ++k) {
      rk[k] = __shfl_sync(0xffffffffu, my_p, k);
      wks[k] = __shfl_sync(0xffffffffu, my_w, k);
    }
    if (v >= nv) continue;
    uint4 raw[KK];
#pragma unroll
    for (int k = 0; k < KK; ++k)
      raw[k] = rk[k] >= 0 ? reinterpret_cast<const uint4*>(y + (int64_t)rk[k] * d)[v]
                          : make_uint4(0, 0, 0, 0);
    float acc[8];
    bool have = false;
#pragma unroll
    for (int k = 0; k < KK; ++k) {
      if (rk[k] < 0) continue;
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[k]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        const float p0 = __fmul_rn(f.x, wks[k]), p1 = __fmul_rn(f.y, wks[k]);
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
    if (!have) {
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    }
    if (res) {
      const uint4 rr = reinterpret_cast<const uint4*>(res + t * d)[v];
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(r2[j]);
        acc[2 * j] = __fadd_rn(__bfloat162float(__float2bfloat16_rn(acc[2 * j])), f.x);
        acc[2 * j + 1] = __fadd_rn(__bfloat162float(__float2bfloat16_rn(acc[2 * j + 1])), f.y);
      }
    }
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) o2[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    reinterpret_cast<uint4*>(out + t * d)[v] = o;
  }
}

// ------------------------------------------------------------------ RMSNorm
// routed_expert_norm of the latent block, read as an RMSNorm: per row
// r = 1/sqrt(mean(x^2) + eps) in double, n = bf16(x*r) (one rounding from
// double), out = bf16(w*n) (the product of two bf16 values is exact in fp32).
// One warp per row; lane l owns the 16-byte vectors l, l+32, ...
constexpr int kMaxNormVecs = 32;  // d <= 32 * 8 * 32 = 8192 held in registers

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ uint4 norm_vec(const uint4 xv, const uint4 wv, double r) {
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv);
  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(&wv);
  uint4 o;
  __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float n = __bfloat162float(__double2bfloat16((double)__bfloat162float(xb[j]) * r));
    ob[j] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(wb[j]), n));
  }
  return o;
}

__device__ __forceinline__ double sumsq_vec(const uint4 xv) {
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv);
  double a = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const double v = (double)__bfloat162float(xb[j]);
    a += v * v;
  }
  return a;
}

template <int NV>
__global__ void __launch_bounds__(32 * kWarps) k_rms_norm(const __nv_bfloat16* __restrict__ x,
                                                          int64_t N, int d,
                                                          const __nv_bfloat16* __restrict__ w,
                                                          float eps,
                                                          __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int64_t t = (int64_t)blockIdx.x * kWarps + warp; t < N; t += (int64_t)gridDim.x * kWarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
    uint4 xv[NV];
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = i * 32 + lane;
      xv[i] = v < nv ? xr[v] : make_uint4(0, 0, 0, 0);
      ss += sumsq_vec(xv[i]);
    }
    ss = warp_sum_d(ss);
    const double r = 1.0 / sqrt(ss / (double)d + (double)eps);
    uint4* orow = reinterpret_cast<uint4*>(out + t * d);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = i * 32 + lane;
      if (v < nv) orow[v] = norm_vec(xv[i], reinterpret_cast<const uint4*>(w)[v], r);
    }
  }
}

// Combine (as k_combine) and RMSNorm of the combined bf16 row in one pass:
// one warp per token, the combined row kept in registers.
template <int NV>
__global__ void __launch_bounds__(32 * kWarps) k_combine_rms_norm(
    const __nv_bfloat16* __restrict__ y, const int32_t* __restrict__ pos,
    const float* __restrict__ w, int64_t N, int K, int d, int64_t S,
    const __nv_bfloat16* __restrict__ norm_w, float eps, __nv_bfloat16* __restrict__ out,
    DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  for (int64_t t = (int64_t)blockIdx.x * kWarps + warp; t < N; t += (int64_t)gridDim.x * kWarps) {
    int my_p = -1;
    float my_w = 0.f;
    if (lane < K) {
      my_p = pos ? pos[t * K + lane] : (int)(t * K + lane);
      my_w = w[t * K + lane];
      if (my_p < 0 || my_p >= S) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 41);
        my_p = -1;
      }
    }
    float acc[NV][8];
    bool have = false;
    for (int k = 0; k < K; ++k) {
      const int p = __shfl_sync(0xffffffffu, my_p, k);
      const float wk = __shfl_sync(0xffffffffu, my_w, k);
      if (p < 0) continue;
      const uint4* yr = reinterpret_cast<const uint4*>(y + (int64_t)p * d);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int v = i * 32 + lane;
        const uint4 raw = v < nv ? yr[v] : make_uint4(0, 0, 0, 0);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h2[j]);
          const float p0 = __fmul_rn(f.x, wk), p1 = __fmul_rn(f.y, wk);
          acc[i][2 * j] = have ? __fadd_rn(acc[i][2 * j], p0) : p0;
          acc[i][2 * j + 1] = have ? __fadd_rn(acc[i][2 * j + 1], p1) : p1;
        }
      }
      have = true;
    }
    uint4 cv[NV];
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      __nv_bfloat162* c2 = reinterpret_cast<__nv_bfloat162*>(&cv[i]);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        c2[j] = have ? __floats2bfloat162_rn(acc[i][2 * j], acc[i][2 * j + 1])
                     : __floats2bfloat162_rn(0.f, 0.f);
      if (i * 32 + lane >= nv) cv[i] = make_uint4(0, 0, 0, 0);
      ss += sumsq_vec(cv[i]);
    }
    ss = warp_sum_d(ss);
    const double r = 1.0 / sqrt(ss / (double)d + (double)eps);
    uint4* orow = reinterpret_cast<uint4*>(out + t * d);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int v = i * 32 + lane;
      if (v < nv) orow[v] = norm_vec(cv[i], reinterpret_cast<const uint4*>(norm_w)[v], r);
    }
  }
}

int64_t row_blocks(int64_t N) {
  int64_t blocks = (N + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  return blocks > cap ? cap : blocks;
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* pos, const float* w, int64_t N,
                           int K, int d_e, int64_t S, __nv_bfloat16* out, DeviceStatus* st,
                           cudaStream_t s, const __nv_bfloat16* residual) {
  const int64_t items = N * ((d_e / 8 + 31) / 32);
  int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  if (blocks > cap) blocks = cap;
  if (K == 4 || K == 8 || K == 16) {  // all K loads of a column in flight together
    const dim3 g((unsigned)blocks), b(32 * kWarps);
    if (K == 4)
      return launch_pdl(k_combine_rows<4>, g, b, 0, s, y, pos, w, N, d_e, S, out, residual, st);
    if (K == 8)
      return launch_pdl(k_combine_rows<8>, g, b, 0, s, y, pos, w, N, d_e, S, out, residual, st);
    return launch_pdl(k_combine_rows<16>, g, b, 0, s, y, pos, w, N, d_e, S, out, residual, st);
  }
  return launch_pdl(k_combine, dim3((unsigned)blocks), dim3(32 * kWarps), 0, s, y, pos, w, N, K,
                    d_e, S, out, residual, st);
}

// d <= 256 * NV columns; the smallest register footprint that holds the row
#define MOE_NORM_DISPATCH(KERNEL, ...)                                          \
  do {                                                                          \
    const int nvl = (d + 255) / 256;                                            \
    const unsigned g = (unsigned)row_blocks(N);                                 \
    if (nvl <= 4) e = launch_pdl(KERNEL<4>, dim3(g), dim3(32 * kWarps), 0, s, __VA_ARGS__);  \
    else if (nvl <= 8) e = launch_pdl(KERNEL<8>, dim3(g), dim3(32 * kWarps), 0, s, __VA_ARGS__); \
    else if (nvl <= 16)                                                          \
      e = launch_pdl(KERNEL<16>, dim3(g), dim3(32 * kWarps), 0, s, __VA_ARGS__);  \
    else e = launch_pdl(KERNEL<kMaxNormVecs>, dim3(g), dim3(32 * kWarps), 0, s, __VA_ARGS__); \
  } while (0)

cudaError_t launch_rms_norm(const __nv_bfloat16* x, int64_t N, int d, const __nv_bfloat16* w,
                            float eps, __nv_bfloat16* out, cudaStream_t s) {
  if (d > kMaxNormVecs * 256) return cudaErrorInvalidValue;
  cudaError_t e;
  MOE_NORM_DISPATCH(k_rms_norm, x, N, d, w, eps, out);
  return e;
}

cudaError_t launch_combine_rms_norm(const __nv_bfloat16* y, const int32_t* pos, const float* w,
                                    int64_t N, int K, int d_e, int64_t S,
                                    const __nv_bfloat16* norm_w, float eps,
                                    __nv_bfloat16* out, DeviceStatus* st, cudaStream_t s) {
  const int d = d_e;
  if (d > kMaxNormVecs * 256) return cudaErrorInvalidValue;
  cudaError_t e;
  MOE_NORM_DISPATCH(k_combine_rms_norm, y, pos, w, N, K, d, S, norm_w, eps, out, st);
  return e;
}

}  // namespace moe
