// ep_rows.cu -- the expert-parallel exchange over peer memory.
//
// "Kimi K3 · Add shared output", moe-forward excerpt: with expert
// parallelism a rank runs only self.experts[i + ep_rank * experts_per_rank],
// so the rows routed to another rank's experts travel there and their
// outputs travel back before the weighted sum.  Here no collective library
// moves them:
//   k_ep_dispatch_rows  reads every token row once and stores it to the K
//                       receiving ranks' row buffers (peer addresses), at the
//                       row its sorted position maps to;
//   k_ep_combine_rows   loads each slot's expert output from the rank that
//                       computed it and takes moe_combine's weighted sum
//                       (products rounded to fp32, summed in k order).
// Sorted position j of this rank goes to the rank q whose expert range holds
// it, offsets[q*E_local] <= j < offsets[(q+1)*E_local], at row
// first[q] + j - offsets[q*E_local] of q's buffer.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kRowBatch = 8;  // a token's rows loaded together by the combine (K <= 16)

// The rank and row that sorted position j maps to; -1 when j or the row is out
// of range.  P <= 64 boundaries, read through L1.
__device__ __forceinline__ int peer_of(const PeerTable& pt, const int32_t* __restrict__ offsets,
                                       int j, int64_t& row) {
  if (j < 0) return -1;
  for (int q = 0; q < pt.P; ++q) {
    const int hi = offsets[(q + 1) * pt.E_local];
    if (j < hi) {
      const int lo = offsets[q * pt.E_local];
      if (j < lo) return -1;
      row = pt.first[q] + (int64_t)(j - lo);
      return row < pt.cap[q] ? q : -1;
    }
  }
  return -1;
}

// One warp per (token, chunk of 256 columns), as the local gather: the row
// vector is loaded once and stored to each of the token's K destinations.
__global__ void __launch_bounds__(32 * kWarps) k_ep_dispatch_rows(
    const __nv_bfloat16* __restrict__ x, int64_t N, int K, int d,
    const int32_t* __restrict__ pos, const int32_t* __restrict__ offsets, int64_t S,
    const __grid_constant__ PeerTable pt, DeviceStatus* st) {
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
    int my_q = -1;
    int64_t my_row = 0;
    if (lane < K) {
      const int j = pos[t * K + lane];
      if (j >= S) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 50);
      } else if (j >= 0) {
        my_q = peer_of(pt, offsets, j, my_row);
        if (my_q < 0) record_error(st, MOE_ERR_DEVICE_BOUNDS, 51);
      }
    }
    const uint4 val =
        v < nv ? reinterpret_cast<const uint4*>(x + t * d)[v] : make_uint4(0, 0, 0, 0);
    for (int k = 0; k < K; ++k) {
      const int q = __shfl_sync(0xffffffffu, my_q, k);
      const long long row = __shfl_sync(0xffffffffu, (long long)my_row, k);
      if (q >= 0 && v < nv) reinterpret_cast<uint4*>(pt.rows[q] + row * d)[v] = val;
    }
  }
}

// One warp per (token, chunk of 256 columns).  The token's rows are loaded
// kRowBatch at a time before any is summed (loads from another GPU have a
// long latency); the sum starts from -0 (-0 + x == x, so the first product
// enters unchanged) and runs in k order, as moe_combine.
__global__ void __launch_bounds__(32 * kWarps) k_ep_combine_rows(
    const __grid_constant__ PeerTable pt, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ offsets, int64_t S, const float* __restrict__ w, int64_t N,
    int K, int d, __nv_bfloat16* __restrict__ out, DeviceStatus* st) {
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
    int my_q = -1;
    int64_t my_row = 0;
    float my_w = 0.f;
    if (lane < K) {
      const int j = pos[t * K + lane];
      my_w = w[t * K + lane];
      if (j >= S) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 52);
      } else if (j >= 0) {
        my_q = peer_of(pt, offsets, j, my_row);
        if (my_q < 0) record_error(st, MOE_ERR_DEVICE_BOUNDS, 53);
      }
    }
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = -0.f;
    bool have = false;
    for (int k0 = 0; k0 < K; k0 += kRowBatch) {
      uint4 raw[kRowBatch];
      float wk[kRowBatch];
      bool ok[kRowBatch];
#pragma unroll
      for (int b = 0; b < kRowBatch; ++b) {
        const int k = k0 + b;
        const int q = __shfl_sync(0xffffffffu, my_q, k & 31);
        const long long row = __shfl_sync(0xffffffffu, (long long)my_row, k & 31);
        wk[b] = __shfl_sync(0xffffffffu, my_w, k & 31);
        ok[b] = k < K && q >= 0 && v < nv;
        raw[b] = ok[b] ? reinterpret_cast<const uint4*>(pt.rows[q] + row * d)[v]
                       : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int b = 0; b < kRowBatch; ++b) {
        if (!ok[b]) continue;
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw[b]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h2[i]);
          acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(f.x, wk[b]));
          acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(f.y, wk[b]));
        }
        have = true;
      }
    }
    if (v >= nv) continue;
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o2[i] = have ? __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1])
                   : __floats2bfloat162_rn(0.f, 0.f);
    reinterpret_cast<uint4*>(out + t * d)[v] = o;
  }
}

unsigned row_item_blocks(int64_t N, int d) {
  const int64_t items = N * ((d / 8 + 31) / 32);
  int64_t blocks = (items + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  return (unsigned)(blocks > cap ? cap : blocks);
}

}  // namespace

cudaError_t launch_ep_dispatch_rows(const __nv_bfloat16* x, int64_t N, int K, int d,
                                    const int32_t* pos, const int32_t* offsets, int64_t S,
                                    const PeerTable& pt, DeviceStatus* st, cudaStream_t s) {
  return launch_pdl(k_ep_dispatch_rows, dim3(row_item_blocks(N, d)), dim3(32 * kWarps), 0, s, x,
                    N, K, d, pos, offsets, S, pt, st);
}

cudaError_t launch_ep_combine_rows(const PeerTable& pt, const int32_t* pos,
                                   const int32_t* offsets, int64_t S, const float* w, int64_t N,
                                   int K, int d, __nv_bfloat16* out, DeviceStatus* st,
                                   cudaStream_t s) {
  return launch_pdl(k_ep_combine_rows, dim3(row_item_blocks(N, d)), dim3(32 * kWarps), 0, s, pt,
                    pos, offsets, S, w, N, K, d, out, st);
}

}  // namespace moe
