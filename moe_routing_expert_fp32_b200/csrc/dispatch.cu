// dispatch.cu -- moe_infer's dispatch without a host round trip.
//
// Follows "Kimi K3 · Add shared output", moe-forward excerpt (moe_infer):
// per-expert counts (cnts.scatter_ + sum), argsort of the flat slots, and
// sorted_tokens = x[idxs // K].  The page copies the counts to the host
// (.cpu()) to drive a Python loop over experts; here the counts, offsets and
// the grouped GEMM's tile list stay on the device.
//
// The slot sort is a stable counting sort in three passes:
//   k_hist    one warp per chunk of CH consecutive slots: per-chunk expert
//             counts (warp-aggregated with __match_any_sync);
//   k_scan    one block per 32 experts: counts[e] and, per chunk, the number
//             of expert-e slots in the chunks before it;
//   k_scatter one warp per chunk again: every block takes the exclusive scan
//             of counts (block 0 stores it as offsets), then the slots are
//             ranked in slot order within the chunk -> pos[slot], perm[pos].
// Small sorts (at most 4096 slots, at most 1024 experts: decode batches) run
// the same three passes in one block instead: k_sort_small, 32 warps, warp w
// the w-th of 32 contiguous chunks, its counts in shared memory.
// Then k_gather copies every token row once from HBM and writes it to its K
// sorted positions (token-major, so x_e is read once, not K times).  Without
// xs (the expert MLP gathering its rows itself) k_gather is skipped.
// The chunk passes load kIdxBatch slot indices per lane before using any, so
// a warp has that many loads in flight instead of one.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 4;
constexpr int kIdxBatch = 8;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(32 * kWarps) k_hist(const int32_t* __restrict__ idx, int64_t S,
                                                      int E, int CH, int nchunks,
                                                      int32_t* __restrict__ cc, DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t cnt_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kWarps + warp;
  if (c >= nchunks) return;
  int32_t* cnt = cnt_all + warp * E;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const int64_t beg = (int64_t)c * CH;
  const int64_t end = beg + CH < S ? beg + CH : S;
  for (int64_t b0 = beg; b0 < end; b0 += 32 * kIdxBatch) {
    int ev[kIdxBatch];
#pragma unroll
    for (int i = 0; i < kIdxBatch; ++i) {
      const int64_t slot = b0 + 32 * i + lane;
      ev[i] = slot < end ? idx[slot] : -1;
    }
#pragma unroll
    for (int i = 0; i < kIdxBatch; ++i) {
      int e = ev[i];
      if (b0 + 32 * i + lane < end && (e < 0 || e >= E)) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 10);
        e = -1;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
      __syncwarp();
    }
  }
  int32_t* out = cc + (int64_t)c * E;
  for (int e = lane; e < E; e += 32) out[e] = cnt[e];
}

// One block per 32 experts, 32 warps: lane l owns expert 32*blockIdx.x + l,
// warp w the chunks [w*per, (w+1)*per).  cc[c][e] becomes the number of
// expert-e slots in chunks 0..c-1; counts[e] the total.
constexpr int kScanHeld = 8;  // chunks per warp kept in registers (per <= 8)

__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ cc, int nchunks, int E,
                                               int32_t* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t part[32][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const int per = (nchunks + 31) / 32;
  const int c0 = w * per;
  const int c1 = c0 + per < nchunks ? c0 + per : nchunks;
  const bool live = e < E;
  int32_t held[kScanHeld];
  int32_t sum = 0;
  if (per <= kScanHeld) {
#pragma unroll
    for (int i = 0; i < kScanHeld; ++i) {
      held[i] = (live && c0 + i < c1) ? cc[(int64_t)(c0 + i) * E + e] : 0;
      sum += held[i];
    }
  } else if (live) {
    for (int c = c0; c < c1; ++c) sum += cc[(int64_t)c * E + e];
  }
  part[w][lane] = sum;
  __syncthreads();
  int32_t run = 0;
  for (int i = 0; i < w; ++i) run += part[i][lane];
  if (w == 0 && live) {
    int32_t tot = 0;
    for (int i = 0; i < 32; ++i) tot += part[i][lane];
    counts[e] = tot;
  }
  if (!live) return;
  if (per <= kScanHeld) {
#pragma unroll
    for (int i = 0; i < kScanHeld; ++i)
      if (c0 + i < c1) {
        cc[(int64_t)(c0 + i) * E + e] = run;
        run += held[i];
      }
  } else {
    for (int c = c0; c < c1; ++c) {
      const int32_t n = cc[(int64_t)c * E + e];
      cc[(int64_t)c * E + e] = run;
      run += n;
    }
  }
}

__global__ void __launch_bounds__(32 * kWarps) k_scatter(const int32_t* __restrict__ idx,
                                                         int64_t S, int E, int CH, int nchunks,
                                                         const int32_t* __restrict__ cc,
                                                         const int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ perm,
                                                         int32_t* __restrict__ pos) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm_all[];  // [E] expert offsets, then kWarps x [E] chunk bases
  __shared__ int32_t warp_tot[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* off = sm_all;
  const int c = blockIdx.x * kWarps + warp;
  int32_t* base = sm_all + (1 + warp) * E;
  // this chunk's counts first: their loads overlap the scan below
  if (c < nchunks) {
    const int32_t* in = cc + (int64_t)c * E;
    for (int e = lane; e < E; e += 32) base[e] = in[e];
  }
  // exclusive scan of counts: thread i owns experts i*per .. i*per+per-1
  const int per = (E + 32 * kWarps - 1) / (32 * kWarps);
  const int e0 = threadIdx.x * per;
  int32_t mine = 0;
  for (int j = 0; j < per; ++j)
    if (e0 + j < E) mine += counts[e0 + j];
  int32_t v = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  int32_t run = v - mine;
  for (int i = 0; i < warp; ++i) run += warp_tot[i];
  for (int j = 0; j < per; ++j) {
    const int e = e0 + j;
    if (e < E) {
      off[e] = run;
      if (blockIdx.x == 0) offsets[e] = run;
      run += counts[e];
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 32 * kWarps - 1) offsets[E] = run;
  __syncthreads();
  if (c >= nchunks) return;
  for (int e = lane; e < E; e += 32) base[e] += off[e];
  __syncwarp();
  const unsigned lt = lanemask_lt();
  const int64_t beg = (int64_t)c * CH;
  const int64_t end = beg + CH < S ? beg + CH : S;
  for (int64_t b0 = beg; b0 < end; b0 += 32 * kIdxBatch) {
    int ev[kIdxBatch];
#pragma unroll
    for (int i = 0; i < kIdxBatch; ++i) {
      const int64_t slot = b0 + 32 * i + lane;
      ev[i] = slot < end ? idx[slot] : -1;
    }
#pragma unroll
    for (int i = 0; i < kIdxBatch; ++i) {
      const int64_t slot = b0 + 32 * i + lane;
      const int e = (ev[i] < 0 || ev[i] >= E) ? -1 : ev[i];
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (slot < end) {
        if (e >= 0) {
          const int32_t p = base[e] + __popc(peers & lt);
          pos[slot] = p;
          perm[p] = (int32_t)slot;
        } else {
          pos[slot] = -1;
        }
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) base[e] += __popc(peers);
      __syncwarp();
    }
  }
}

// The stable counting sort of k_hist + k_scan + k_scatter in one block of 32
// warps for S <= kSmallSortMaxS slots and E <= kSmallSortMaxE experts: warp w
// takes the w-th of 32 contiguous chunks of slots, counts them per expert
// (pass 1), every expert's thread turns the warps' counts into their
// exclusive prefix and the expert totals into offsets (pass 2), and each warp
// ranks its slots in slot order (pass 3).  The ranks are those of the
// three-kernel sort: pos and perm are unique for a stable sort.  The counts
// are 16-bit (at most 4096 slots), 32 x E of them in dynamic shared memory.
constexpr int kSmallSortMaxS = 4096;
constexpr int kSmallSortMaxE = 1024;
constexpr int kSmallSortRounds = kSmallSortMaxS / (32 * 32);  // slots per lane

__global__ void __launch_bounds__(1024) k_sort_small(const int32_t* __restrict__ idx, int S, int E,
                                                     int32_t* __restrict__ counts,
                                                     int32_t* __restrict__ offsets,
                                                     int32_t* __restrict__ perm,
                                                     int32_t* __restrict__ pos,
                                                     DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int16_t cnt_raw[];  // [32][E]
  __shared__ int32_t warp_tot[32];
  auto cnt = [&](int w, int e) -> int16_t& { return cnt_raw[w * E + e]; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CH = (S + 31) / 32;
  const int beg = warp * CH;
  const int end = beg + CH < S ? beg + CH : S;
  for (int e = lane; e < E; e += 32) cnt(warp, e) = 0;
  __syncwarp();
  // pass 1: this warp's counts; the slot indices stay in registers
  int ev[kSmallSortRounds];
#pragma unroll
  for (int i = 0; i < kSmallSortRounds; ++i) {
    const int slot = beg + 32 * i + lane;
    int e = slot < end ? idx[slot] : -1;
    if (slot < end && (e < 0 || e >= E)) {
      record_error(st, MOE_ERR_DEVICE_BOUNDS, 10);
      e = -1;
    }
    ev[i] = e;
  }
#pragma unroll
  for (int i = 0; i < kSmallSortRounds; ++i) {
    const unsigned peers = __match_any_sync(0xffffffffu, ev[i]);
    if (ev[i] >= 0 && lane == __ffs(peers) - 1)
      cnt(warp, ev[i]) = (int16_t)(cnt(warp, ev[i]) + __popc(peers));
    __syncwarp();
  }
  __syncthreads();
  // pass 2: thread e, expert e: the warps' exclusive prefix, the total, then
  // the exclusive scan of the totals over the experts
  const int e = threadIdx.x;
  int32_t tot = 0;
  if (e < E) {
    for (int w = 0; w < 32; ++w) {
      const int32_t t = cnt(w, e);
      cnt(w, e) = (int16_t)tot;
      tot += t;
    }
    counts[e] = tot;
  }
  int32_t v = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  int32_t off = v - tot;
  for (int i = 0; i < warp; ++i) off += warp_tot[i];
  if (e < E) {
    offsets[e] = off;
    for (int w = 0; w < 32; ++w) cnt(w, e) = (int16_t)(cnt(w, e) + off);
    if (e == E - 1) offsets[E] = off + tot;
  }
  __syncthreads();
  // pass 3: ranks in slot order, as k_scatter
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int i = 0; i < kSmallSortRounds; ++i) {
    const int slot = beg + 32 * i + lane;
    const int ee = ev[i];
    const unsigned peers = __match_any_sync(0xffffffffu, ee);
    if (slot < end) {
      if (ee >= 0) {
        const int32_t p = cnt(warp, ee) + __popc(peers & lt);
        pos[slot] = p;
        perm[p] = slot;
      } else {
        pos[slot] = -1;
      }
    }
    __syncwarp();
    if (ee >= 0 && lane == __ffs(peers) - 1)
      cnt(warp, ee) = (int16_t)(cnt(warp, ee) + __popc(peers));
    __syncwarp();
  }
}

// One warp per (token, chunk of 256 columns): each lane reads one 16-byte
// vector of the token's row once and writes it to the K sorted positions
// pos[t*K + k] (token-major, so x_e is read once, not K times).  The next
// item's row and positions are loaded before this item's K stores issue.
__device__ __forceinline__ void gather_load(const __nv_bfloat16* __restrict__ x, int K, int d,
                                            int nv, int nch, int lane, int64_t it,
                                            const int32_t* __restrict__ pos, uint4& val,
                                            int& my_p) {
  const int64_t t = it / nch;
  const int v = (int)(it - t * nch) * 32 + lane;
  my_p = lane < K ? pos[t * K + lane] : -1;
  val = v < nv ? reinterpret_cast<const uint4*>(x + t * d)[v] : make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(256) k_gather(const __nv_bfloat16* __restrict__ x, int64_t N,
                                                int K, int d, const int32_t* __restrict__ pos,
                                                __nv_bfloat16* __restrict__ xs) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = d / 8;
  const int nch = (nv + 31) / 32;
  const int64_t items = N * nch;
  const int64_t stride = (int64_t)gridDim.x * 8;
  int64_t it = (int64_t)blockIdx.x * 8 + warp;
  if (it >= items) return;
  uint4 val;
  int my_p;
  gather_load(x, K, d, nv, nch, lane, it, pos, val, my_p);
  for (; it < items; it += stride) {
    uint4 nval = make_uint4(0, 0, 0, 0);
    int n_p = -1;
    if (it + stride < items) gather_load(x, K, d, nv, nch, lane, it + stride, pos, nval, n_p);
    const int64_t t = it / nch;
    const int v = (int)(it - t * nch) * 32 + lane;
    for (int k = 0; k < K; ++k) {
      const int p = __shfl_sync(0xffffffffu, my_p, k);
      if (p >= 0 && v < nv) reinterpret_cast<uint4*>(xs + (int64_t)p * d)[v] = val;
    }
    val = nval;
    my_p = n_p;
  }
}

// offsets[i] = sum_{j<i} counts[j] for i <= n (n <= 1024), one block.
__global__ void __launch_bounds__(1024) k_counts_offsets(const int32_t* __restrict__ counts, int n,
                                                         int32_t* __restrict__ offsets,
                                                         DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t warp_tot[32];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  int32_t c = 0;
  if (i < n) {
    c = counts[i];
    if (c < 0) {
      record_error(st, MOE_ERR_DEVICE_BOUNDS, 12);
      c = 0;
    }
  }
  int32_t v = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  const int32_t excl = v - c + (warp > 0 ? warp_tot[warp - 1] : 0);
  if (i < n) offsets[i] = excl;
  if (i == n - 1) offsets[n] = excl + c;
}

}  // namespace

cudaError_t launch_counts_offsets(const int32_t* counts, int n, int32_t* offsets,
                                  DeviceStatus* st, cudaStream_t s) {
  return launch_pdl(k_counts_offsets, dim3(1), dim3(1024), 0, s, counts, n, offsets, st);
}

int dispatch_chunks(int64_t S) {
  int64_t ch = S / 256;
  if (ch < 64) ch = 64;
  if (ch > 1024) ch = 1024;
  ch = (ch + 31) / 32 * 32;
  return (int)((S + ch - 1) / ch);
}

static int dispatch_chunk_len(int64_t S) {
  int64_t ch = S / 256;
  if (ch < 64) ch = 64;
  if (ch > 1024) ch = 1024;
  return (int)((ch + 31) / 32 * 32);
}

size_t dispatch_scratch_bytes(int64_t S, int E) {
  return align_up(sizeof(int32_t) * (size_t)dispatch_chunks(S) * (size_t)E, 256);
}

cudaError_t launch_dispatch(const int32_t* idx, int64_t N, int K, int E, const __nv_bfloat16* x_e,
                            int d_e, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* pos, __nv_bfloat16* xs, int32_t* scratch, DeviceStatus* st,
                            cudaStream_t s) {
  const int64_t S = N * K;
  cudaError_t e;
  if (S >= 1 && S <= kSmallSortMaxS && E <= kSmallSortMaxE) {
    static std::once_flag once[kMaxDevices];
    static cudaError_t set_up[kMaxDevices];
    if ((e = once_per_device(once, set_up, [](int) {
           return cudaFuncSetAttribute(k_sort_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(sizeof(int16_t) * 32 * kSmallSortMaxE));
         })) != cudaSuccess)
      return e;
    const size_t smem = sizeof(int16_t) * 32 * (size_t)E;
    if ((e = launch_pdl(k_sort_small, dim3(1), dim3(1024), smem, s, idx, (int)S, E, counts,
                        offsets, perm, pos, st)) != cudaSuccess)
      return e;
  } else {
    const int CH = dispatch_chunk_len(S);
    const int nchunks = dispatch_chunks(S);
    const size_t smem = sizeof(int32_t) * (size_t)E * kWarps;
    const unsigned blocks = (unsigned)((nchunks + kWarps - 1) / kWarps);
    if ((e = launch_pdl(k_hist, dim3(blocks), dim3(32 * kWarps), smem, s, idx, S, E, CH, nchunks,
                        scratch, st)) != cudaSuccess ||
        (e = launch_pdl(k_scan, dim3((unsigned)((E + 31) / 32)), dim3(1024), 0, s, scratch,
                        nchunks, E, counts)) != cudaSuccess ||
        (e = launch_pdl(k_scatter, dim3(blocks), dim3(32 * kWarps), smem + sizeof(int32_t) * E, s,
                        idx, S, E, CH, nchunks, scratch, counts, offsets, perm, pos)) != cudaSuccess)
      return e;
  }
  if (!xs) return cudaSuccess;
  int64_t gb = (N * ((d_e / 8 + 31) / 32) + 7) / 8;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  if (gb > cap) gb = cap;
  return launch_pdl(k_gather, dim3((unsigned)gb), dim3(256), 0, s, x_e, N, K, d_e, pos, xs);
}

}  // namespace moe
