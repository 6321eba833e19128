// expert_gemm.cu -- grouped expert MLP on the 5th-generation tensor cores.
//
// Follows "Kimi K3 · Gate features", expert excerpt (KimiBlockSparseMLP:
// w1 = gate, w3 = up, w2 = down, all bias-free nn.Linear) and situ excerpt
// (SituAndMul), and the per-expert loop of moe_infer ("Kimi K3 · Add shared
// output", moe-forward excerpt), which is replaced by one persistent launch
// over a device-built tile list per projection.
//
// Design (sm_100a):
//   * swap-AB: the MMA's M = 128 side is weight rows, the N side is up to NTMAX
//     token rows of one expert (N rounded up to 16).  Decode batches put 1-8
//     rows on an expert, so the kernel is a weight stream whatever the count.
//   * gate_up unit = 64 rows of d_ff: its 128-row A tile is w1 rows f0..f0+63
//     over w3 rows f0..f0+63 (two 64-row TMA boxes), so one MMA per k-step
//     yields g (TMEM lanes 0-63) and u (lanes 64-127); the epilogue warps that
//     hold g and u of the same 32 rows swap half of each 16-column chunk
//     through shared memory, so all four warps apply the activation.
//   * down unit = 128 rows of d.
//   * TMA (cp.async.bulk.tensor, 128-byte swizzle) fills a STAGES-deep ring of
//     (A 128x64, B NTMAX x64) bf16 tiles guarded by mbarriers; one elected
//     thread issues tcgen05.mma kind::f16 (bf16 in, fp32 accumulate) into
//     TMEM; two accumulator buffers let the epilogue of one unit overlap the
//     MMAs of the next; 4 epilogue warps drain TMEM with tcgen05.ld and
//     write bf16 rows with 16-byte stores (an 8 x 8 / 8 x 16 shuffle
//     transpose per 8-lane group turns one feature per lane into 8
//     consecutive features per token);
//   * decode and mid variants can gather their token rows themselves: row i of
//     a tile is x_e[perm[row0 + i] / K], fetched with tile::gather4 TMA loads
//     (4 rows of 64 columns each, the same 128-byte swizzle), so no gathered
//     copy xs of the tokens is needed (a memory saving: 32 small loads per
//     128-row tile make it slower than a separate gather plus tiled loads);
//   * dense layers (one expert, every row) split K over units when the row
//     blocks alone would leave SMs idle, and k_splitk_reduce finishes them;
//   * three variants by average rows per expert: decode (NTMAX 32, 5 stages
//     of two 64-column sub-tiles: ~160 KB of weights in flight per SM, so each
//     weight row is read 256 contiguous bytes at a time, loaded with an L2
//     evict-first hint since each is read once), mid (NTMAX 128, two A blocks
//     and accumulators per unit, 4 stages) and large (a CTA pair running
//     256x256x16 cta_group::2 MMAs on two weight blocks per token tile, 4
//     stages; see k_expert_gemm_pair).
//   * the page's rounding points: g, u rounded to bf16; SiLU output rounded to
//     bf16 before the product; SiTU evaluated in fp32; h and y rounded to bf16.
//   * unit u -> (token tile, weight-row block), row block fastest: CTAs that
//     run together share one token tile from L2 and stream disjoint weights.
//   * every wait is bounded (2 s of %globaltimer); a wait that runs out records
//     MOE_ERR_DEVICE_TIMEOUT, tells the other roles to stop, frees TMEM and the
//     kernel returns.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BM = 128;        // A rows per tile (MMA M)
constexpr int BK = 64;         // K elements per stage: one 128-byte swizzle row
constexpr int UK = 16;         // K per tcgen05.mma for 16-bit inputs
constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kBoxRows = 16;   // token rows per small TMA box
constexpr int kBigBoxRows = 64;  // token rows per large TMA box (prefill variant)
constexpr int kGateUpRows = 64;  // d_ff rows per gate_up unit (w1 + w3 = 128 A rows)
constexpr int kXchgBytes = 8192;  // gate_up epilogue exchange: 2 pairs x 2 bufs x 2 x 32x8 fp32

enum Mode { kGateUp = 0, kDown = 1 };

// UM = A blocks (of 128 rows) per unit, each with its own accumulator;
// KSUB = 64-column sub-tiles per stage (a stage covers 64*KSUB of K, so each
// weight row is read KSUB*128 contiguous bytes at a time).
template <int NTMAX, int STAGES, int UM, int KSUB>
struct Cfg {
  static constexpr int kABlockBytes = BM * BK * 2;
  static constexpr int kABytes = UM * KSUB * kABlockBytes;
  static constexpr int kBSubBytes = NTMAX * BK * 2;
  static constexpr int kBBytes = KSUB * kBSubBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBufCols = UM * NTMAX;  // TMEM columns per accumulator buffer
  static constexpr int kTmemCols = (2 * kBufCols < 32) ? 32 : 2 * kBufCols;
  static constexpr size_t kSmem = (size_t)STAGES * kStageBytes + 1024 + 256 + kXchgBytes;
  static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// ------------------------------------------------------------ PTX wrappers
// (the shared ones are in sm100.cuh)
using sm100::gtimer;
using sm100::l2_evict_first_policy;
using sm100::mbar_arrive;
using sm100::mbar_arrive_expect_tx;
using sm100::mbar_init;
using sm100::mbar_try_wait;
using sm100::mbar_wait;
using sm100::smem_u32;
using sm100::tc_fence_after;
using sm100::tc_fence_before;
using sm100::tma_load_2d;
using sm100::tma_load_3d;
using sm100::tma_load_3d_hint;
using sm100::umma_commit;

// Four rows r0..r3 (any order, any rows) of a 2-D map whose box is 64 columns
// x 1 row, written to dst as consecutive 128-byte rows with the map's swizzle.
__device__ __forceinline__ void tma_gather4(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1),
      "r"(r2), "r"(r3)
      : "memory");
}

// Programmatic dependent launch: the dependent kernel waits here until the
// preceding kernel's memory is visible; a primary lets dependents launch.
__device__ __forceinline__ void grid_dep_wait() { pdl_wait(); }
__device__ __forceinline__ void grid_dep_launch() { pdl_trigger(); }

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// 32 lanes x 16 consecutive fp32 columns; waits for the load before returning.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  sm100::tmem_ld16(taddr, r);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (tile base 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return sm100::smem_desc(saddr, 1024, 2);
}
// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

// Diagnostics hook (moe_set_wait_probe): with `probe` set, the producer first
// waits on a barrier that nothing arrives on, with a 1 ms limit, before it
// issues any copy; the wait runs out and the kernel takes its abort path (the
// error recorded, the other roles stopped, TMEM freed).  Returns true when the
// kernel must stop.
constexpr uint64_t kProbeLimitNs = 1000000ull;
__device__ __forceinline__ bool probe_abort(int probe, uint64_t* never, volatile int* abort_flag,
                                            DeviceStatus* st, int detail) {
  if (!probe) return false;
  if (mbar_wait(never, 0, abort_flag, kProbeLimitNs)) return false;  // nothing arrives on it
  record_error(st, MOE_ERR_DEVICE_TIMEOUT, detail);
  *abort_flag = 1;
  return true;
}

__device__ __forceinline__ float bf16r(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// Down-projection output element (row, m): bf16 of the accumulator, or with a
// residual bf16( bf16(acc) + res ) -- the Linear output is a bf16 tensor
// before the add, and the add of two bf16 values is rounded once.
__device__ __forceinline__ __nv_bfloat16 down_out(float acc, const __nv_bfloat16* res, int row,
                                                  int M_rows, int m) {
  if (!res) return __float2bfloat16_rn(acc);
  return __float2bfloat16_rn(
      __fadd_rn(bf16r(acc), __bfloat162float(res[(int64_t)row * M_rows + m])));
}

// SiLU-and-mul with the page's rounding points: g and u are bf16 Linear
// outputs; silu(g) is evaluated in fp32 and rounded to bf16; the product of two
// bf16 values is exact in fp32 and rounded to bf16 by the store.
__device__ __forceinline__ float silu_mul(float g, float u) {
  g = bf16r(g);
  u = bf16r(u);
  const float a = bf16r(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))));
  return __fmul_rn(a, u);
}
// SiTU: beta*tanh(g/beta)*sigmoid(g) * (lbeta*tanh(u/lbeta) or u), in fp32.
__device__ __forceinline__ float situ_mul(float g, float u, float beta, float lbeta, bool has_lb) {
  g = bf16r(g);
  u = bf16r(u);
  const float t = __fmul_rn(beta, tanhf(__fdiv_rn(g, beta)));
  const float sg = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-g)));
  const float up = has_lb ? __fmul_rn(lbeta, tanhf(__fdiv_rn(u, lbeta))) : u;
  return __fmul_rn(__fmul_rn(t, sg), up);
}

// e: the weight index of the unit's segment.  Segment s (rows offsets[s] ..
// offsets[s+1]) uses weights s % emod: emod = E for the layer, E_local for
// rows received from several ranks, grouped by (source rank, local expert).

// bf16 of (lo, hi) in one word, lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t p) { return __uint_as_float(p & 0xffff0000u); }

// Stores one 16-token chunk of a down-projection accumulator (lane l holds
// feature m = m8 + (l & 7) of its 8-lane group, v[j] = token c0 + j) as
// out[token][feature] with 16-byte stores: the 8 x 16 block of each 8-lane
// group is transposed by shuffles so that lane i holds tokens 2i and 2i+1 of
// the group's 8 features.  Every lane of the warp must call it.
// (store_down_t8_packed takes the chunk already rounded: p[t] = bf16 of
// tokens 2t, 2t+1.)
__device__ __forceinline__ void store_down_t8_packed(const uint32_t* p, __nv_bfloat16* out,
                                                     int64_t tok0, int ntok, int M_rows, int m8,
                                                     bool live, int lane,
                                                     const int32_t* rowmap = nullptr,
                                                     int64_t map_rows = 0,
                                                     DeviceStatus* st = nullptr) {
  uint32_t a[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) a[t] = p[t];
  const int i = lane & 7;
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if ((j & s) == 0) {
        const bool upper = (i & s) != 0;
        const uint32_t send = upper ? a[j] : a[j | s];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, s);
        if (upper) a[j] = recv;
        else a[j | s] = recv;
      }
    }
  }
  // a[j] = feature m8 + j, tokens (2i, 2i+1)
  uint4 lo, hi;
  lo.x = __byte_perm(a[0], a[1], 0x5410); hi.x = __byte_perm(a[0], a[1], 0x7632);
  lo.y = __byte_perm(a[2], a[3], 0x5410); hi.y = __byte_perm(a[2], a[3], 0x7632);
  lo.z = __byte_perm(a[4], a[5], 0x5410); hi.z = __byte_perm(a[4], a[5], 0x7632);
  lo.w = __byte_perm(a[6], a[7], 0x5410); hi.w = __byte_perm(a[6], a[7], 0x7632);
  if (live) {
    // row r of the token tile goes to output row r, or to rowmap[r] (the
    // slot-order scatter: sorted row j is written where slot perm[j] lives)
    int64_t r0 = tok0 + 2 * i, r1 = r0 + 1;
    if (rowmap) {
      r0 = 2 * i < ntok ? rowmap[r0] : -1;
      r1 = 2 * i + 1 < ntok ? rowmap[r1] : -1;
      if ((2 * i < ntok && (r0 < 0 || r0 >= map_rows)) ||
          (2 * i + 1 < ntok && (r1 < 0 || r1 >= map_rows))) {
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 140);
        if (r0 >= map_rows) r0 = -1;
        if (r1 >= map_rows) r1 = -1;
      }
    }
    if (2 * i < ntok && r0 >= 0) *reinterpret_cast<uint4*>(out + r0 * M_rows + m8) = lo;
    if (2 * i + 1 < ntok && r1 >= 0) *reinterpret_cast<uint4*>(out + r1 * M_rows + m8) = hi;
  }
}
__device__ __forceinline__ void store_down_t8(const float* v, __nv_bfloat16* out, int64_t tok0,
                                              int ntok, int M_rows, int m8, bool live, int lane,
                                              const int32_t* rowmap = nullptr,
                                              int64_t map_rows = 0,
                                              DeviceStatus* st = nullptr) {
  uint32_t p[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) p[t] = pack_bf16x2(v[2 * t], v[2 * t + 1]);
  store_down_t8_packed(p, out, tok0, ntok, M_rows, m8, live, lane, rowmap, map_rows, st);
}


// The gate_up epilogue's 8 h values of one feature (lane l: feature f8 +
// (l & 7), tokens tok0 .. tok0 + 7) stored as out[token][feature] with one
// 16-byte store per lane: the 8 x 8 block of each 8-lane group is
// transposed by shuffles so that lane i holds token tok0 + i of the group's
// 8 features.  Every lane of the warp must call it.
__device__ __forceinline__ void store_h_t8(const float* h, __nv_bfloat16* out, int64_t tok0,
                                           int ntok, int M_rows, int f8, bool live, int lane) {
  uint32_t a[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const __nv_bfloat16 b = __float2bfloat16_rn(h[t]);
    a[t] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&b));
  }
  const int i = lane & 7;
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if ((j & s) == 0) {
        const bool upper = (i & s) != 0;
        const uint32_t send = upper ? a[j] : a[j | s];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, s);
        if (upper) a[j] = recv;
        else a[j | s] = recv;
      }
    }
  }
  // a[j] = feature f8 + j at token tok0 + i
  uint4 o;
  o.x = a[0] | (a[1] << 16);
  o.y = a[2] | (a[3] << 16);
  o.z = a[4] | (a[5] << 16);
  o.w = a[6] | (a[7] << 16);
  if (live && i < ntok) *reinterpret_cast<uint4*>(out + (tok0 + i) * M_rows + f8) = o;
}

struct Unit {
  int e, row0, nrows, rb;
};

// Unit u is weight block u % RB of the tile at position u / RB of the tile
// list; order (may be null) maps that position to a tile index.
__device__ __forceinline__ Unit decode_unit(int64_t u, int RB, int nt, const int32_t* tile_start,
                                            const int32_t* offsets, int E, int emod,
                                            const int32_t* order = nullptr) {
  Unit r;
  const int tp = (int)(u / RB);
  r.rb = (int)(u - (int64_t)tp * RB);
  const int tt = order ? order[tp] : tp;
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // largest e with tile_start[e] <= tt
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tt) lo = mid;
    else hi = mid - 1;
  }
  r.e = lo % emod;
  r.row0 = offsets[lo] + (tt - tile_start[lo]) * nt;
  const int rem = offsets[lo + 1] - r.row0;
  r.nrows = rem < nt ? rem : nt;
  return r;
}

template <int MODE, int NTMAX, int STAGES, int UM, int KSUB>
__global__ void __launch_bounds__(kThreads, 1)
    k_expert_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                  const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB64,
                  const int32_t* __restrict__ offsets,
                  const int32_t* __restrict__ tile_start, int E, int M_rows, int Kdim,
                  __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ res,
                  int act_kind, float beta, float lbeta, DeviceStatus* st, int pdl,
                  const int32_t* __restrict__ gperm, int gk, int gn, int ksplit,
                  float* __restrict__ part, int emod, int probe,
                  const int32_t* __restrict__ yrow) {
  using C = Cfg<NTMAX, STAGES, UM, KSUB>;
  constexpr int KS = BK * KSUB;  // K columns per stage
  constexpr bool kDecode = NTMAX <= 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* never = tempty + 2;  // the diagnostics hook's barrier (nothing arrives on it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xchg = reinterpret_cast<float*>(smem + STAGES * C::kStageBytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // rows of the output per A block: 64 d_ff rows (gate_up) or 128 d rows (down)
  const int blk_rows = (MODE == kGateUp) ? kGateUpRows : BM;
  const int unit_rows = UM * blk_rows;
  const int RB = (M_rows + unit_rows - 1) / unit_rows;
  const int KB = Kdim / KS;
  // split-K (dense layers with few units): unit u covers k-blocks
  // [ks*KB/ksplit, (ks+1)*KB/ksplit) of (token tile, row block) u / ksplit,
  // and its epilogue writes fp32 partial sums to `part` for k_splitk_reduce
  const int64_t total_units = (int64_t)tile_start[E] * RB * ksplit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(never, 1);
    *abort_flag = 0;
    sm100::mbar_init_fence();
  }
  if (warp == 1) sm100::tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  bool gathered = false;
  if constexpr (MODE == kGateUp) {
    if (warp == 0 && gperm != nullptr) {
      // ---------------------------------------- TMA producer, gathered rows
      // Row i of a unit's token tile is x_e[perm[row0 + i] / K] (sorted slot
      // -> token): the warp reads the tile's token ids, lane 0 fetches the
      // rows 4 at a time with tile::gather4 loads of tmB (box 64 x 1, same
      // swizzle as a tiled box).  Rows past the segment up to the next
      // multiple of 16 repeat its last row; their accumulator columns are
      // never stored.
      __shared__ int32_t tok_s[NTMAX];
      gathered = true;
      const uint64_t wpol = kDecode ? l2_evict_first_policy() : 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      if (lane == 0) ok = !probe_abort(probe, never, abort_flag, st, 190 + MODE);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      for (int64_t u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const Unit w = decode_unit(u / ksplit, RB, NTMAX, tile_start, offsets, E, emod);
        const int ks = (int)(u % ksplit);
        const int kb0 = (int)((int64_t)ks * KB / ksplit), kb1 = (int)((int64_t)(ks + 1) * KB / ksplit);
        const int rows = (w.nrows + 15) & ~15;
        __syncwarp();
        for (int i = lane; i < rows; i += 32) {
          int32_t t = gperm[w.row0 + (i < w.nrows ? i : w.nrows - 1)] / gk;
          if (t < 0 || t >= gn) {  // a slot outside the batch: recorded, row 0 read
            record_error(st, MOE_ERR_DEVICE_BOUNDS, 31);
            t = 0;
          }
          tok_s[i] = t;
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t bytes = C::kABytes + KSUB * rows * BK * 2;
          const int r0 = w.rb * unit_rows;
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
            uint8_t* sA = smem + stage * C::kStageBytes;
            uint8_t* sB = sA + C::kABytes;
            mbar_arrive_expect_tx(&full[stage], bytes);
#pragma unroll
            for (int sub = 0; sub < KSUB; ++sub) {
              const int kc = kb * KS + sub * BK;
#pragma unroll
              for (int a = 0; a < UM; ++a) {
                uint8_t* dA = sA + (a * KSUB + sub) * C::kABlockBytes;
                const int ra = r0 + a * blk_rows;
                void* d3 = dA + kGateUpRows * BK * 2;
                if (kDecode) {
                  tma_load_3d_hint(&tmA0, &full[stage], dA, kc, ra, w.e, wpol);
                  tma_load_3d_hint(&tmA1, &full[stage], d3, kc, ra, w.e, wpol);
                } else {
                  tma_load_3d(&tmA0, &full[stage], dA, kc, ra, w.e);
                  tma_load_3d(&tmA1, &full[stage], d3, kc, ra, w.e);
                }
              }
              for (int g = 0; g < rows; g += 4)
                tma_gather4(&tmB, &full[stage], sB + sub * C::kBSubBytes + g * BK * 2, kc,
                            tok_s[g], tok_s[g + 1], tok_s[g + 2], tok_s[g + 3]);
            }
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0) {
        grid_dep_launch();
        if (!ok) {
          record_error(st, MOE_ERR_DEVICE_TIMEOUT, 105);
          *abort_flag = 1;
        }
      }
    }
  }
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // (warp 0 is the producer in both forms; with gathered rows it ran above,
    // and it must not fall through to the MMA or epilogue roles)
    if (lane == 0 && !gathered) {
      const uint64_t wpol = kDecode ? l2_evict_first_policy() : 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = !probe_abort(probe, never, abort_flag, st, 190 + MODE);
      // With programmatic dependent launch the token rows (written by the
      // preceding kernel) may be read only after grid_dep_wait(); the weight
      // tiles of the first ring of stages are fetched before it.
      bool dep_pending = pdl != 0;
      for (int64_t u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const Unit w = decode_unit(u / ksplit, RB, NTMAX, tile_start, offsets, E, emod);
        const int ks = (int)(u % ksplit);
        const int kb0 = (int)((int64_t)ks * KB / ksplit), kb1 = (int)((int64_t)(ks + 1) * KB / ksplit);
        // token rows: 16-row boxes for short tiles, 64-row boxes otherwise
        const bool big = !kDecode && w.nrows > 2 * kBoxRows;
        const int brows = big ? kBigBoxRows : kBoxRows;
        const int nb = (w.nrows + brows - 1) / brows;
        const uint32_t bytes = C::kABytes + KSUB * nb * brows * BK * 2;
        const int r0 = w.rb * unit_rows;
        auto load_a = [&](int kb, uint8_t* sA) {
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub) {
            const int kc = kb * KS + sub * BK;
#pragma unroll
            for (int a = 0; a < UM; ++a) {
              uint8_t* dA = sA + (a * KSUB + sub) * C::kABlockBytes;
              const int ra = r0 + a * blk_rows;
              if (MODE == kGateUp) {
                // w1 rows ra..ra+63 over w3 rows ra..ra+63
                void* d3 = dA + kGateUpRows * BK * 2;
                if (kDecode) {
                  tma_load_3d_hint(&tmA0, &full[stage], dA, kc, ra, w.e, wpol);
                  tma_load_3d_hint(&tmA1, &full[stage], d3, kc, ra, w.e, wpol);
                } else {
                  tma_load_3d(&tmA0, &full[stage], dA, kc, ra, w.e);
                  tma_load_3d(&tmA1, &full[stage], d3, kc, ra, w.e);
                }
              } else {
                if (kDecode) tma_load_3d_hint(&tmA0, &full[stage], dA, kc, ra, w.e, wpol);
                else tma_load_3d(&tmA0, &full[stage], dA, kc, ra, w.e);
              }
            }
          }
        };
        auto load_b = [&](int kb, uint8_t* sB, int st_idx) {
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub)
            for (int i = 0; i < nb; ++i)
              tma_load_2d(big ? &tmB64 : &tmB, &full[st_idx],
                          sB + sub * C::kBSubBytes + i * brows * BK * 2, kb * KS + sub * BK,
                          w.row0 + i * brows);
        };
        int kb = kb0;
        if (dep_pending) {
          // weights of up to STAGES k-blocks first, then wait, then their tokens
          const int pre = kb0 + (kb1 - kb0 < STAGES ? kb1 - kb0 : STAGES);
          for (; kb < pre; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], bytes);
            load_a(kb, smem + stage * C::kStageBytes);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          grid_dep_wait();
          dep_pending = false;
          int st_idx = 0;  // the first unit started at stage 0
          for (int j = kb0; j < kb; ++j) {
            load_b(j, smem + st_idx * C::kStageBytes + C::kABytes, st_idx);
            if (++st_idx == STAGES) st_idx = 0;
          }
          if (!ok) break;
        }
        for (; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          load_a(kb, sA);
          load_b(kb, sA + C::kABytes, stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (dep_pending) grid_dep_wait();
      // every load of this CTA is issued: let the dependent kernel launch
      grid_dep_launch();
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 100 + MODE);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++local) {
        const Unit w = decode_unit(u / ksplit, RB, NTMAX, tile_start, offsets, E, emod);
        const int ks = (int)(u % ksplit);
        const int kb0 = (int)((int64_t)ks * KB / ksplit), kb1 = (int)((int64_t)(ks + 1) * KB / ksplit);
        const int n = ((w.nrows + 15) / 16) * 16;
        const uint32_t idesc = idesc_bf16(n);
        const int buf = local & 1;
        const uint32_t tphase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tphase ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + buf * C::kBufCols;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b0 = a0 + C::kABytes;
#pragma unroll
          for (int sub = 0; sub < KSUB; ++sub)
#pragma unroll
            for (int k = 0; k < BK / UK; ++k)
#pragma unroll
              for (int a = 0; a < UM; ++a)
                umma_bf16(d0 + a * NTMAX,
                          sw128_desc(a0 + (a * KSUB + sub) * C::kABlockBytes + k * UK * 2),
                          sw128_desc(b0 + sub * C::kBSubBytes + k * UK * 2), idesc,
                          (kb != kb0 || sub != 0 || k != 0));
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) umma_commit(&tfull[buf]);
      }
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 110 + MODE);
        *abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 belong to this warp
    const bool has_lb = !(lbeta == 0.0f || lbeta != lbeta);
    const float b_eff = (beta == 0.0f || beta != beta) ? 1.0f : beta;
    int local = 0;
    uint32_t xbuf = 0;  // exchange buffer parity (gate_up)
    for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x, ++local) {
      const Unit w = decode_unit(u / ksplit, RB, NTMAX, tile_start, offsets, E, emod);
      const int ks = (int)(u % ksplit);
      const int buf = local & 1;
      const uint32_t tphase = (local >> 1) & 1;
      if (!mbar_wait(&tfull[buf], tphase, abort_flag)) {
        if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 120 + MODE);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      for (int a = 0; a < UM; ++a) {
      const uint32_t taddr =
          tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * C::kBufCols + a * NTMAX;
      const int r0 = w.rb * unit_rows + a * blk_rows;
      if (part) {
        // fp32 partial sums: down -> part[ks][row][m]; gate_up -> g at
        // part[ks][row][f], u at part[ks][row][F + f]
        const int64_t S_rows = offsets[E];
        int m, ld, moff;
        if (MODE == kGateUp) {
          m = r0 + (quarter & 1) * 32 + lane;
          ld = 2 * M_rows;
          moff = quarter < 2 ? 0 : M_rows;
        } else {
          m = r0 + quarter * 32 + lane;
          ld = M_rows;
          moff = 0;
        }
        float* pcol = part + (int64_t)ks * S_rows * ld + moff + m;
        const int lim_m = m < M_rows ? 16 : 0;
        for (int c0 = 0; c0 < w.nrows; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
          int lim = w.nrows - c0 < 16 ? w.nrows - c0 : 16;
          lim = lim < lim_m ? lim : lim_m;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < lim) pcol[(int64_t)(w.row0 + c0 + j) * ld] = v[j];
        }
      } else if (MODE == kGateUp) {
        // quarters 0/1 hold g of rows 0-31 / 32-63, quarters 2/3 hold u of the
        // same rows; pair p = quarter & 1.  Per 16-column chunk the g warp keeps
        // columns 0-7 and hands g of columns 8-15 to the u warp, which keeps
        // columns 8-15 and hands u of columns 0-7 back.
        const int pair = quarter & 1;
        const bool is_g = quarter < 2;
        const int f = r0 + pair * 32 + lane;
        const bool live = f < M_rows;
        for (int c0 = 0; c0 < w.nrows; c0 += 16, ++xbuf) {
          float v[16];
          tmem_ld16(taddr + c0, v);
          float* xg = xchg + ((pair * 2 + (xbuf & 1)) * 2 + 0) * 256;  // g cols 8-15
          float* xu = xchg + ((pair * 2 + (xbuf & 1)) * 2 + 1) * 256;  // u cols 0-7
          float4* mine = reinterpret_cast<float4*>((is_g ? xg : xu) + lane * 8);
          const float* give = is_g ? v + 8 : v;
          mine[0] = make_float4(give[0], give[1], give[2], give[3]);
          mine[1] = make_float4(give[4], give[5], give[6], give[7]);
          asm volatile("bar.sync %0, 64;" ::"r"(1 + pair) : "memory");
          const float4* theirs = reinterpret_cast<const float4*>((is_g ? xu : xg) + lane * 8);
          const float4 t0 = theirs[0], t1 = theirs[1];
          const float other[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
          const int cbase = c0 + (is_g ? 0 : 8);
          float hv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float g = is_g ? v[j] : other[j];
            const float uu = is_g ? other[j] : v[8 + j];
            hv[j] = act_kind == MOE_ACT_SITU ? situ_mul(g, uu, b_eff, lbeta, has_lb)
                                             : silu_mul(g, uu);
          }
          store_h_t8(hv, out, w.row0 + cbase, w.nrows - cbase, M_rows, f & ~7, live, lane);
        }
      } else {
        const int m = r0 + quarter * 32 + lane;
        __nv_bfloat16* col = out + m;
        const int lim_m = m < M_rows ? 16 : 0;
        for (int c0 = 0; c0 < w.nrows; c0 += 16) {
          float v[16];
          tmem_ld16(taddr + c0, v);
          int lim = w.nrows - c0 < 16 ? w.nrows - c0 : 16;
          if (!res) {
            store_down_t8(v, out, w.row0 + c0, lim, M_rows, m & ~7, lim_m != 0, lane, yrow,
                          yrow ? (int64_t)offsets[E] : 0, st);
            continue;
          }
          lim = lim < lim_m ? lim : lim_m;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < lim) col[(int64_t)(w.row0 + c0 + j) * M_rows] = down_out(v[j], res, w.row0 + c0 + j, M_rows, m);
        }
      }
      }  // accumulators
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    sm100::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------ CTA-pair variant
// Large variant on a CTA pair (cluster of 2, tcgen05 cta_group::2): one MMA is
// M = 256 weight rows (128 per CTA, each from its own shared memory) x N = up
// to 256 token rows (N/2 rows held by each CTA), accumulating into each CTA's
// own TMEM (its 128 rows x N).  Each CTA therefore fetches half of the token
// tile it multiplies with, which halves the operand bytes per FLOP that every
// SM pulls from L2.  No TMA multicast: each CTA loads its own operands.
// Protocol:
//   full[s]   (even CTA only) one arrive.expect_tx by the even CTA's producer
//             for both CTAs' bytes; both CTAs' TMA loads credit it;
//   empty[s]  (both CTAs) the MMA commit is multicast to both;
//   tfull[b]  (both CTAs) the MMA commit is multicast to both;
//   tempty[b] (even CTA) one arrival per epilogue warp of both CTAs, by an
//             elected lane after the warp's TMEM loads and a warp sync.
// Cluster barriers after set-up and before freeing TMEM; every mbarrier wait
// is bounded as in the single-CTA kernel.
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;  // clears the pair-rank bit of a cluster address

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint64_t* bar, void* dst,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap* map, uint64_t* bar, void* dst,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1),
      "r"(c2)
      : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ uint32_t idesc_bf16_m256(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(256 >> 4) << 24);
}

constexpr int kPairNt = 256;     // token rows per tile (N, split 128 + 128)
// Tile order of the CTA-pair kernels: 1 spreads the one-tile experts among
// the tiles of larger ones (k_tiles' order), 0 keeps expert order.
#ifndef MOE_PAIR_INTERLEAVE
#define MOE_PAIR_INTERLEAVE 1
#endif
constexpr bool kPairInterleave = MOE_PAIR_INTERLEAVE != 0;
// Epilogue warps of the CTA-pair kernel: kPairSlices warps per TMEM lane
// quarter, each copying kPairNt / kPairSlices columns of an accumulator to
// registers.  With two weight blocks per unit the accumulators fill TMEM and
// the next unit's MMAs wait for this copy, so it is split over 16 warps; with
// the 64 TMA / MMA threads that is 576 per CTA (96 registers a thread).
#ifndef MOE_PAIR_SLICES
#define MOE_PAIR_SLICES 4
#endif
constexpr int kPairSlices = MOE_PAIR_SLICES;
constexpr int kPairThreads = 64 + 4 * 32 * kPairSlices;  // TMA, MMA, 4 x kPairSlices epilogue
static_assert(kPairNt % (32 * kPairSlices) == 0, "whole 32-column TMEM loads per slice");
// gate_up exchange through shared memory: per slice, quarter pair, parity and
// g/u, one 16-byte word per lane
constexpr int kPairXchgWords = 32 * 4;  // 32-bit words per entry

// PUM weight blocks of 256 rows (128 per CTA) per unit, all against the same
// token tile.  PUM = 1: 6 stages of (A 16 KB + B half 16 KB) per CTA, two
// TMEM accumulator buffers (the epilogue of one unit overlaps the MMAs of the
// next).  PUM = 2: 4 stages of (A 2 x 16 KB + B half 16 KB): each token byte
// brought from L2 feeds twice the MMAs, a quarter fewer bytes per MMA, which
// is what bounds the one-block form (its TMA issue runs flat out while the
// MMAs wait for data).  The two 256-column accumulators fill TMEM, so there
// is one buffer: the epilogue copies each accumulator to registers and hands
// it back before it computes and stores, and the next unit's first-block MMAs
// run on held stages while the second accumulator is copied.
template <int PUM>
struct PairCfg {
  static constexpr int kStages = PUM == 1 ? 6 : 4;
  static constexpr int kABlockBytes = BM * BK * 2;
  static constexpr int kABytes = PUM * kABlockBytes;
  static constexpr int kBBytes = (kPairNt / 2) * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBufCols = kPairNt;
  static constexpr int kTmemCols = 2 * kPairNt;
  static constexpr int kXchg = kPairSlices * 2 * 2 * 2 * kPairXchgWords * 4;
  static constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024 + 256 + kXchg;
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(PUM == 1 || PUM == 2, "one or two weight blocks per unit");
};

template <int MODE, int PUM>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_expert_gemm_pair(const __grid_constant__ CUtensorMap tmA0,
                       const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmB64,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ tile_start,
                       int E, int M_rows, int Kdim, __nv_bfloat16* __restrict__ out,
                       const __nv_bfloat16* __restrict__ res, int act_kind, float beta,
                       float lbeta, DeviceStatus* st, int pdl, int emod, int probe,
                       const int32_t* __restrict__ yrow, const int32_t* __restrict__ order) {
  using C = PairCfg<PUM>;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* never = tempty + 2;  // the diagnostics hook's barrier (nothing arrives on it)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xchg = reinterpret_cast<float*>(smem + STAGES * C::kStageBytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0: issues the MMAs for the pair
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // rows of the output per CTA and weight block: 64 d_ff rows (gate_up) or
  // 128 d rows (down); a block is 2 * blk_rows rows of the pair, a unit PUM
  // blocks
  const int blk_rows = (MODE == kGateUp) ? kGateUpRows : BM;
  const int unit_rows = PUM * 2 * blk_rows;
  const int RB = (M_rows + unit_rows - 1) / unit_rows;
  const int KB = Kdim / BK;
  const int64_t total_units = (int64_t)tile_start[E] * RB;
  // TMEM accumulators: PUM = 1, tfull/tempty[i] guard buffer i (units
  // alternate); PUM = 2, they guard the accumulator of block i (one buffer)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * (kPairThreads - 64) / 32);  // every epilogue warp of the pair
    }
    mbar_init(never, 1);
    *abort_flag = 0;
    sm100::mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive / credit
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = !probe_abort(probe, never, abort_flag, st, 290 + MODE);
      bool dep_pending = pdl != 0;  // see the single-CTA kernel
      for (int64_t u = pair_id; u < total_units && ok; u += npairs) {
        const Unit w = decode_unit(u, RB, kPairNt, tile_start, offsets, E, emod, order);
        const int n = ((w.nrows + 15) / 16) * 16;
        const int half = n / 2;  // token rows this CTA contributes
        const bool big = half > 2 * kBoxRows;
        const int brows = big ? kBigBoxRows : kBoxRows;
        const int nb = (half + brows - 1) / brows;
        const uint32_t cta_bytes = C::kABytes + nb * brows * BK * 2;
        const int tb = w.row0 + rank * half;
        auto load_a = [&](int kb, uint8_t* sA, int st_idx) {
#pragma unroll
          for (int a = 0; a < PUM; ++a) {
            const int ra = w.rb * unit_rows + a * 2 * blk_rows + rank * blk_rows;
            uint8_t* dA = sA + a * C::kABlockBytes;
            if (MODE == kGateUp) {
              tma_load_3d_pair(&tmA0, &full[st_idx], dA, kb * BK, ra, w.e);
              tma_load_3d_pair(&tmA1, &full[st_idx], dA + kGateUpRows * BK * 2, kb * BK, ra, w.e);
            } else {
              tma_load_3d_pair(&tmA0, &full[st_idx], dA, kb * BK, ra, w.e);
            }
          }
        };
        auto load_b = [&](int kb, uint8_t* sB, int st_idx) {
          for (int i = 0; i < nb; ++i)
            tma_load_2d_pair(big ? &tmB64 : &tmB, &full[st_idx], sB + i * brows * BK * 2, kb * BK,
                             tb + i * brows);
        };
        int kb = 0;
        if (dep_pending) {
          const int pre = KB < STAGES ? KB : STAGES;
          for (; kb < pre; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * cta_bytes);
            load_a(kb, smem + stage * C::kStageBytes, stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          grid_dep_wait();
          dep_pending = false;
          for (int j = 0; j < kb; ++j)
            load_b(j, smem + j * C::kStageBytes + C::kABytes, j);
          if (!ok) break;
        }
        for (; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * C::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * cta_bytes);
          load_a(kb, sA, stage);
          load_b(kb, sA + C::kABytes, stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (dep_pending) grid_dep_wait();
      grid_dep_launch();
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 200 + MODE);
        *abort_flag = 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint64_t desc_base = sw128_desc(smem_u32(smem));
      for (int64_t u = pair_id; u < total_units && ok; u += npairs, ++local) {
        const Unit w = decode_unit(u, RB, kPairNt, tile_start, offsets, E, emod, order);
        const int n = ((w.nrows + 15) / 16) * 16;
        const uint32_t idesc = idesc_bf16_m256(n);
        // the MMAs of weight block a on stage st (k-block kb)
        // descriptors: the shared-memory base's, plus each operand's byte
        // offset / 16 (the start-address field; no carry at these offsets)
        auto mma_block = [&](int a, int st, int kb, uint32_t d) {
          const uint64_t so = (uint64_t)(st * (C::kStageBytes >> 4));
          const uint64_t da = desc_base + so + (uint64_t)(a * (C::kABlockBytes >> 4));
          const uint64_t db = desc_base + so + (uint64_t)(C::kABytes >> 4);
          umma_bf16_pair(d, da, db, idesc, kb != 0);
#pragma unroll
          for (int k = 1; k < BK / UK; ++k)
            umma_bf16_pair(d, da + (uint64_t)(k * UK * 2 / 16), db + (uint64_t)(k * UK * 2 / 16),
                           idesc, 1u);
        };
        if constexpr (PUM == 1) {
          const int buf = local & 1;
          const uint32_t tphase = (local >> 1) & 1;
          if (!mbar_wait(&tempty[buf], tphase ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d0 = tmem_base + buf * C::kBufCols;
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            mma_block(0, stage, kb, d0);
            umma_commit_pair(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          if (ok) umma_commit_pair(&tfull[buf]);
        } else {
          // both accumulators must have been copied out by the epilogue
          // before the unit starts (block 1's copy follows block 0's by ~1 k
          // cycles); the loop then issues both blocks' MMAs on every stage
          const uint32_t tpar = (local & 1) ^ 1;
          if (!mbar_wait(&tempty[0], tpar, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&tempty[1], tpar, abort_flag)) { ok = false; break; }
          tc_fence_after();
          for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            mma_block(0, stage, kb, tmem_base);
            if (kb == KB - 1) umma_commit_pair(&tfull[0]);  // block 0 is complete
            mma_block(1, stage, kb, tmem_base + C::kBufCols);
            umma_commit_pair(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
          }
          if (ok) umma_commit_pair(&tfull[1]);
        }
      }
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 210 + MODE);
        *abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------ epilogue (both CTAs)
    // Each warp copies its share of an accumulator (the TMEM lanes of its
    // quarter, the columns of its slice) to registers, rounded to bf16 in
    // pairs as every output of the kernel is rounded first, and hands the
    // accumulator back at once: the MMAs of the next unit then wait only for
    // the copy, and the exchange, activation and stores overlap them.  (The
    // residual form keeps fp32 to the end and drains in place.)
    constexpr int kSliceCols = kPairNt / kPairSlices;
    constexpr int kChunks = kSliceCols / 16;
    const int quarter = warp & 3;       // TMEM lanes 32 * quarter .. + 31
    const int slice = (warp - 2) >> 2;  // TMEM columns col0 .. col0 + kSliceCols - 1
    const int col0 = slice * kSliceCols;
    const bool has_lb = !(lbeta == 0.0f || lbeta != lbeta);
    const float b_eff = (beta == 0.0f || beta != beta) ? 1.0f : beta;
    const uint32_t tempty_leader0 = peer_addr(smem_u32(&tempty[0]), 0);
    int local = 0;
    uint32_t xbuf = 0;
    bool stop = false;
    for (int64_t u = pair_id; u < total_units && !stop; u += npairs, ++local) {
      const Unit w = decode_unit(u, RB, kPairNt, tile_start, offsets, E, emod, order);
      if (MODE == kDown && res) {
        for (int a = 0; a < PUM; ++a) {
          const int buf = PUM == 1 ? (local & 1) : a;
          const uint32_t tphase = PUM == 1 ? ((local >> 1) & 1) : (local & 1);
          if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], tphase, abort_flag))) {
            if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 220 + MODE);
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * C::kBufCols;
          const int m = w.rb * unit_rows + a * 2 * blk_rows + rank * blk_rows + quarter * 32 + lane;
          __nv_bfloat16* col = out + m;
          const int lim_m = m < M_rows ? 16 : 0;
          for (int c0 = col0; c0 < w.nrows && c0 < col0 + kSliceCols; c0 += 16) {
            float v[16];
            tmem_ld16(taddr + c0, v);
            int lim = w.nrows - c0 < 16 ? w.nrows - c0 : 16;
            lim = lim < lim_m ? lim : lim_m;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (j < lim)
                col[(int64_t)(w.row0 + c0 + j) * M_rows] =
                    down_out(v[j], res, w.row0 + c0 + j, M_rows, m);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(tempty_leader0 + buf * (uint32_t)sizeof(uint64_t));
        }
        continue;
      }
      // pk[a][8 * ci + t]: block a, chunk ci (columns col0 + 16 ci ..), tokens
      // 2t and 2t + 1 of the chunk
      uint32_t pk[PUM][kSliceCols / 2];
#pragma unroll
      for (int a = 0; a < PUM; ++a) {
        const int buf = PUM == 1 ? (local & 1) : a;
        const uint32_t tphase = PUM == 1 ? ((local >> 1) & 1) : (local & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], tphase, abort_flag))) {
          if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 220 + MODE);
          *abort_flag = 1;
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * C::kBufCols + col0;
        if (col0 < w.nrows) {
#pragma unroll
          for (int q = 0; q < kSliceCols / 32; ++q) {
            uint32_t r[32];
            sm100::tmem_ld32(taddr + 32 * q, r);
#pragma unroll
            for (int t = 0; t < 16; ++t)
              pk[a][16 * q + t] =
                  pack_bf16x2(__uint_as_float(r[2 * t]), __uint_as_float(r[2 * t + 1]));
          }
        }
        tc_fence_before();
        __syncwarp();
        // the accumulator (buffer, or block) goes back to the even CTA's MMA
        // issuer: one arrival per warp, after the warp's loads and a warp sync
        if (lane == 0) mbar_arrive_remote(tempty_leader0 + buf * (uint32_t)sizeof(uint64_t));
      }
      if (stop) break;
#pragma unroll
      for (int a = 0; a < PUM; ++a) {
        const int r0 = w.rb * unit_rows + a * 2 * blk_rows + rank * blk_rows;
        if (MODE == kGateUp) {
          // lanes 0-63 of the block hold g (w1 rows), 64-127 u (w3 rows) of the
          // same 64 features: quarters q and q + 2 swap half of each chunk, so
          // the g quarter forms h for the chunk's first 8 tokens, the u quarter
          // for the last 8
          const int pair = quarter & 1;
          const bool is_g = quarter < 2;
          const int f = r0 + pair * 32 + lane;
          const bool live = f < M_rows;
#pragma unroll
          for (int ci = 0; ci < kChunks; ++ci) {
            const int c0 = col0 + 16 * ci;
            if (c0 >= w.nrows) break;
            const uint32_t* p = &pk[a][8 * ci];
            const int xe = ((slice * 2 + pair) * 2 + (xbuf & 1)) * 2;
            uint4* xg = reinterpret_cast<uint4*>(xchg + (xe + 0) * kPairXchgWords);
            uint4* xu = reinterpret_cast<uint4*>(xchg + (xe + 1) * kPairXchgWords);
            (is_g ? xg : xu)[lane] =
                is_g ? make_uint4(p[4], p[5], p[6], p[7]) : make_uint4(p[0], p[1], p[2], p[3]);
            asm volatile("bar.sync %0, 64;" ::"r"(1 + pair + 2 * slice) : "memory");
            const uint4 th = (is_g ? xu : xg)[lane];
            const uint32_t other[4] = {th.x, th.y, th.z, th.w};
            const int cbase = c0 + (is_g ? 0 : 8);
            float hv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t own = is_g ? p[j >> 1] : p[4 + (j >> 1)];
              const float mv = (j & 1) ? bf16_hi(own) : bf16_lo(own);
              const float ov = (j & 1) ? bf16_hi(other[j >> 1]) : bf16_lo(other[j >> 1]);
              const float g = is_g ? mv : ov;
              const float uu = is_g ? ov : mv;
              hv[j] = act_kind == MOE_ACT_SITU ? situ_mul(g, uu, b_eff, lbeta, has_lb)
                                               : silu_mul(g, uu);
            }
            store_h_t8(hv, out, w.row0 + cbase, w.nrows - cbase, M_rows, f & ~7, live, lane);
            ++xbuf;
          }
        } else {
          const int m = r0 + quarter * 32 + lane;
#pragma unroll
          for (int ci = 0; ci < kChunks; ++ci) {
            const int c0 = col0 + 16 * ci;
            if (c0 >= w.nrows) break;
            const int lim = w.nrows - c0 < 16 ? w.nrows - c0 : 16;
            store_down_t8_packed(&pk[a][8 * ci], out, w.row0 + c0, lim, M_rows, m & ~7,
                                 m < M_rows, lane, yrow, yrow ? (int64_t)offsets[E] : 0, st);
          }
        }
      }
    }
  }
  __syncthreads();
  cluster_sync_all();  // no MMA of the pair is still writing either CTA's TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C::kTmemCols));
  }
}

// Exclusive prefix of v over the block (<= 1024 threads); *total gets the sum.
__device__ __forceinline__ int32_t block_excl_scan(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t o = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += o;
  }
  __syncthreads();  // warp_tot is free (an earlier scan has read it)
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int32_t w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  *total = warp_tot[31];
  return x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
}

// Token tiles per expert and their prefix: tile_start[e] = sum_{e'<e}
// ceil(n_e'/nt), tile_start[E] = total.  Inconsistent offsets are recorded
// and give the expert no tile, so the GEMM never reads outside xs.
//
// order (may be null) receives the order in which the CTA-pair kernels take
// the tiles.  An expert with one tile streams its weights from HBM for that
// tile alone; the weights of an expert with several are read from HBM once and
// reused from L2.  In expert order the one-tile experts come in runs: while
// the pairs work on such a run the kernel waits on HBM, and in a run of a
// large expert's tiles on the tensor cores.  The order spreads the P one-tile
// tiles evenly among the R others, each group keeping its own order (the two
// are merged by the keys (2j+1)/2P and (2i+1)/2R, a tie going to the reused
// tile), so that at any time a share of the pairs streams weights while the
// rest compute.
constexpr int kMaxTileExperts = 1024;  // k_tiles: one thread per expert

__global__ void __launch_bounds__(1024) k_tiles(const int32_t* __restrict__ offsets, int E,
                                                int64_t S, int nt, int32_t* __restrict__ tile_start,
                                                int32_t* __restrict__ order, DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t warp_tot[32];
  const int e = threadIdx.x;
  int32_t n = 0;
  if (e < E) {
    const int32_t a = offsets[e], b = offsets[e + 1];
    const bool bad = a < 0 || b < a || b > S || (e == 0 && a != 0) || (e == E - 1 && b != S);
    if (bad) record_error(st, MOE_ERR_DEVICE_BOUNDS, 30);
    else n = (b - a + nt - 1) / nt;
  }
  int32_t T = 0, P = 0;
  const int32_t excl = block_excl_scan(n, warp_tot, &T);
  if (e < E) {
    tile_start[e] = excl;
    if (e == E - 1) tile_start[E] = excl + n;
  }
  if (!order) return;
  const int32_t j = block_excl_scan(n == 1 ? 1 : 0, warp_tot, &P);  // one-tile rank
  const int64_t R = (int64_t)T - P;
  // Each tile is placed by one thread: the tile's expert by binary search of
  // the tile prefix, then its rank in its group and the count of the other
  // group's tiles before it under the merge.
  __shared__ int32_t s_start[kMaxTileExperts + 1], s_one[kMaxTileExperts + 1];
  if (e < E) {
    s_start[e] = excl;
    s_one[e] = (n == 1) ? -1 - j : j;  // one-tile experts: -1 - rank; others: one-tile count before
  }
  if (e == 0) s_start[E] = T;
  __syncthreads();
  for (int32_t t = e; t < T; t += blockDim.x) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // largest expert whose tiles start at or before t
      const int mid = (lo + hi + 1) >> 1;
      if (s_start[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int32_t q = s_one[lo];
    int64_t pos;
    if (q < 0) {
      // one-tile rank jj: jj + #{i < R : (2i+1) P <= (2jj+1) R}
      const int64_t jj = -1 - q;
      const int64_t num = (2 * jj + 1) * R - P;
      int64_t c = num < 0 ? 0 : num / (2 * (int64_t)P) + 1;
      pos = jj + (c < R ? c : R);
    } else {
      // reused rank i: i + #{jj < P : (2jj+1) R < (2i+1) P}
      const int64_t i = t - q;
      const int64_t num = (2 * i + 1) * P - 1 - R;
      int64_t c = num < 0 ? 0 : num / (2 * R) + 1;
      pos = i + (c < P ? c : P);
    }
    order[pos] = t;
  }
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {  // looked up once (thread-safe static)
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// [batch, rows, cols] bf16, box cols=64 x rows=box_rows x 1
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t batch,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The diagnostics hook's switch (moe_set_wait_probe), read at every launch.
std::atomic<int> g_wait_probe{0};
int wait_probe() { return g_wait_probe.load(std::memory_order_relaxed); }

template <int MODE, int NTMAX, int STAGES, int UM, int KSUB>
cudaError_t launch_gemm(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                        const CUtensorMap& b64, const int32_t* offsets, const int32_t* tile_start,
                        int E, int M_rows, int Kdim, __nv_bfloat16* out,
                        const __nv_bfloat16* res, const moe_act_cfg& act, DeviceStatus* st,
                        cudaStream_t s, bool pdl_ok, const int32_t* gperm = nullptr,
                        int gk = 1, int gn = 0, int ksplit = 1, float* part = nullptr,
                        int emod = 0, const int32_t* yrow = nullptr) {
  using C = Cfg<NTMAX, STAGES, UM, KSUB>;
  static std::once_flag once[kMaxDevices];
  static cudaError_t set_up[kMaxDevices];
  const cudaError_t e0 = once_per_device(once, set_up, [](int) {
    return cudaFuncSetAttribute(k_expert_gemm<MODE, NTMAX, STAGES, UM, KSUB>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  });
  if (e0 != cudaSuccess) return e0;
  // The down projection is launched as a programmatic dependent of the kernel
  // before it (the gate_up kernel in the expert MLP): its CTAs start as those
  // CTAs retire and prefetch weight tiles.  Every role reads the tile list
  // before griddepcontrol.wait, so the caller allows this only when the list
  // was complete before the preceding kernel started.
  const int pdl = (MODE == kDown && pdl_ok) ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(dev_info()->sm_count, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return counted(cudaLaunchKernelEx(&cfg, k_expert_gemm<MODE, NTMAX, STAGES, UM, KSUB>, a0, a1, b, b64,
                            offsets, tile_start, E, M_rows, Kdim, out, res, (int)act.kind,
                            act.beta, act.linear_beta, st, pdl, gperm, gk, gn, ksplit, part,
                            emod > 0 ? emod : E, wait_probe(), yrow));
}

// Weight blocks per CTA-pair unit (1 or 2; see PairCfg).
#ifndef MOE_PAIR_BLOCKS
#define MOE_PAIR_BLOCKS 2
#endif
constexpr int kPairBlocks = MOE_PAIR_BLOCKS;

// Launches the CTA-pair kernel on as many pairs as can be resident at once.
template <int MODE>
cudaError_t launch_gemm_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                             const CUtensorMap& b64, const int32_t* offsets,
                             const int32_t* tile_start, int E, int M_rows, int Kdim,
                             __nv_bfloat16* out, const __nv_bfloat16* res,
                             const moe_act_cfg& act, DeviceStatus* st, cudaStream_t s,
                             bool pdl_ok, int emod = 0, const int32_t* yrow = nullptr,
                             const int32_t* order = nullptr) {
  using C = PairCfg<kPairBlocks>;
  constexpr auto kernel = k_expert_gemm_pair<MODE, kPairBlocks>;
  static_assert(kPairSlices >= 1 && 1 + 2 * kPairSlices <= 15, "named barriers 1 .. 2 * slices");
  static std::once_flag once[kMaxDevices];
  static cudaError_t set_up[kMaxDevices];
  static int grid_of[kMaxDevices] = {0};
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int pdl = (MODE == kDown && pdl_ok) ? 1 : 0;
  // kernel attribute and the number of resident pairs, once per device
  const cudaError_t e0 = once_per_device(once, set_up, [&](int dev) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmem);
    if (e != cudaSuccess) return e;
    int pairs = 0;
    cudaLaunchConfig_t q = cfg;
    q.gridDim = dim3(dev_info()->sm_count & ~1, 1, 1);
    e = cudaOccupancyMaxActiveClusters(&pairs, kernel, &q);
    if (e != cudaSuccess || pairs < 1) pairs = dev_info()->sm_count / 2;
    if (pairs > dev_info()->sm_count / 2) pairs = dev_info()->sm_count / 2;
    grid_of[dev] = 2 * pairs;
    return cudaSuccess;
  });
  if (e0 != cudaSuccess) return e0;
  int dev = 0;
  cudaGetDevice(&dev);
  cfg.gridDim = dim3(grid_of[dev], 1, 1);
  cfg.numAttrs = pdl ? 2 : 1;
  return counted(cudaLaunchKernelEx(&cfg, kernel, a0, a1, b, b64, offsets, tile_start,
                            E, M_rows, Kdim, out, res, (int)act.kind, act.beta, act.linear_beta,
                            st, pdl, emod > 0 ? emod : E, wait_probe(), yrow, order));
}

// Variant choice from shapes only (no host round trip), by the average rows
// per expert S / E: decode (<= 16: weight stream, deep ring of small stages),
// mid (<= 128: weight-bound; two 128-row A blocks per unit halve the token
// tile traffic per weight byte), large (tensor-bound: the CTA-pair kernel,
// 256x256 MMAs).
constexpr int kNtDecode = 32, kStagesDecode = 5, kUmDecode = 1, kKsubDecode = 2;
constexpr int kNtMid = 128, kStagesMid = 4, kUmMid = 2, kKsubMid = 1;

enum Variant { kVarDecode = 0, kVarMid = 1, kVarLarge = 2 };

Variant pick_variant(int64_t S, int E) {
  if (S <= 16 * (int64_t)E) return kVarDecode;
  if (S <= 128 * (int64_t)E) return kVarMid;
  return kVarLarge;
}

template <int MODE>
cudaError_t launch_variant(Variant v, const CUtensorMap& a0, const CUtensorMap& a1,
                           const CUtensorMap& b, const CUtensorMap& b64, const int32_t* offsets,
                           const int32_t* tile_start, int E, int M_rows, int Kdim,
                           __nv_bfloat16* out, const __nv_bfloat16* res, const moe_act_cfg& act,
                           DeviceStatus* st, cudaStream_t s, bool pdl_ok = true,
                           int emod = 0, const int32_t* yrow = nullptr,
                           const int32_t* order = nullptr) {
  switch (v) {
    case kVarDecode:
      return launch_gemm<MODE, kNtDecode, kStagesDecode, kUmDecode, kKsubDecode>(
          a0, a1, b, b64, offsets, tile_start, E, M_rows, Kdim, out, res, act, st, s, pdl_ok,
          nullptr, 1, 0, 1, nullptr, emod, yrow);
    case kVarMid:
      return launch_gemm<MODE, kNtMid, kStagesMid, kUmMid, kKsubMid>(
          a0, a1, b, b64, offsets, tile_start, E, M_rows, Kdim, out, res, act, st, s, pdl_ok,
          nullptr, 1, 0, 1, nullptr, emod, yrow);
    default:
      return launch_gemm_pair<MODE>(a0, a1, b, b64, offsets, tile_start, E, M_rows, Kdim, out,
                                    res, act, st, s, pdl_ok, emod, yrow, order);
  }
}

}  // namespace

// Scratch of the expert MLP: tile_start (E + 1), the CTA-pair tile order (one
// entry per tile: at most S / 256 + E), then h [S, F] bf16.
static size_t order_entries(int64_t S, int E) { return (size_t)(S / kPairNt) + (size_t)E + 1; }

size_t expert_scratch_bytes(int64_t S, int E, int F) {
  return align_up(sizeof(int32_t) * (size_t)(E + 1), 256) +
         align_up(sizeof(int32_t) * order_entries(S, E), 256) +
         align_up(sizeof(__nv_bfloat16) * (size_t)S * (size_t)F, 256);
}

bool expert_gather_fusable(int64_t S, int E) { return pick_variant(S, E) != kVarLarge; }

int expert_ffn_run(const __nv_bfloat16* xs, const int32_t* offsets, int E, int64_t S, int d_e,
                   int F, const __nv_bfloat16* w1, const __nv_bfloat16* w3,
                   const __nv_bfloat16* w2, const moe_act_cfg& act, __nv_bfloat16* y,
                   void* scratch, DeviceStatus* st, cudaStream_t s, cudaEvent_t after_gate_up,
                   const __nv_bfloat16* residual, const GatherSrc* gather, int n_weights,
                   const int32_t* y_rows) {
  // segments s use weights s % n_weights (n_weights = E for the layer)
  const int emod = n_weights > 0 ? n_weights : E;
  int32_t* tile_start = static_cast<int32_t*>(scratch);
  uint8_t* p = static_cast<uint8_t*>(scratch) + align_up(sizeof(int32_t) * (size_t)(E + 1), 256);
  int32_t* order = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * order_entries(S, E), 256);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p);
  CUtensorMap mw1, mw3, mw2, mxs, mh, mxs64, mh64;
  if (!make_map_3d(&mw1, w1, d_e, F, emod, kGateUpRows) ||
      !make_map_3d(&mw3, w3, d_e, F, emod, kGateUpRows) ||
      !make_map_3d(&mw2, w2, F, d_e, emod, BM) || !make_map_2d(&mh, h, F, S, kBoxRows) ||
      !make_map_2d(&mh64, h, F, S, kBigBoxRows))
    return MOE_ERR_CUDA;
  if (!gather && (!make_map_2d(&mxs, xs, d_e, S, kBoxRows) ||
                  !make_map_2d(&mxs64, xs, d_e, S, kBigBoxRows)))
    return MOE_ERR_CUDA;
  const Variant var = pick_variant(S, E);
  const int nt = var == kVarDecode ? kNtDecode : (var == kVarMid ? kNtMid : kPairNt);
  if (var != kVarLarge || !kPairInterleave) order = nullptr;
  if (launch_pdl(k_tiles, dim3(1), dim3(1024), 0, s, offsets, E, S, nt, tile_start, order, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  cudaError_t rc;
  if (gather) {
    // token rows straight from x_e (no xs): decode and mid variants only
    if (var == kVarLarge) return MOE_ERR_INVALID_ARG;
    CUtensorMap mxg;
    if (!make_map_2d(&mxg, gather->x_e, d_e, gather->N, 1)) return MOE_ERR_CUDA;
    rc = var == kVarDecode
             ? launch_gemm<kGateUp, kNtDecode, kStagesDecode, kUmDecode, kKsubDecode>(
                   mw1, mw3, mxg, mxg, offsets, tile_start, E, F, d_e, h, nullptr, act, st, s,
                   false, gather->perm, gather->K, (int)gather->N, 1, nullptr, emod)
             : launch_gemm<kGateUp, kNtMid, kStagesMid, kUmMid, kKsubMid>(
                   mw1, mw3, mxg, mxg, offsets, tile_start, E, F, d_e, h, nullptr, act, st, s,
                   false, gather->perm, gather->K, (int)gather->N, 1, nullptr, emod);
  } else {
    rc = launch_variant<kGateUp>(var, mw1, mw3, mxs, mxs64, offsets, tile_start, E, F, d_e, h,
                                 nullptr, act, st, s, true, emod, nullptr, order);
  }
  if (rc != cudaSuccess) return MOE_ERR_CUDA;
  if (after_gate_up && cudaEventRecord(after_gate_up, s) != cudaSuccess) return MOE_ERR_CUDA;
  rc = launch_variant<kDown>(var, mw2, mw2, mh, mh64, offsets, tile_start, E, d_e, F, y, residual,
                             act, st, s, true, emod, y_rows, order);
  return rc == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ------------------------------------------------------------ dense layers
// A dense bias-free Linear (or a shared-expert MLP) is the grouped GEMM with
// one expert whose segment is every row: offsets = {0, M}, one tile list.
// At decode sizes that is only a few units of 128-256 weight rows, so the
// weight stream is split over K as well (split-K): each unit writes fp32
// partial sums and k_splitk_reduce adds them in split order, then applies
// the bf16 rounding, the residual or the activation exactly as the GEMM's own
// epilogue does.
namespace {
template <int MODE>
__global__ void __launch_bounds__(256) k_splitk_reduce(const float* __restrict__ part, int ksplit,
                                                       int64_t M, int cols,
                                                       const __nv_bfloat16* __restrict__ res,
                                                       __nv_bfloat16* __restrict__ out,
                                                       int act_kind, float beta, float lbeta) {
  pdl_wait();
  pdl_trigger();
  const bool has_lb = !(lbeta == 0.0f || lbeta != lbeta);
  const float b_eff = (beta == 0.0f || beta != beta) ? 1.0f : beta;
  const int64_t ld = MODE == kGateUp ? 2 * (int64_t)cols : cols;
  const int64_t n4 = M * cols / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = (i * 4) / cols;
    const int m = (int)(i * 4 - t * cols);
    float a[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ks = 0; ks < ksplit; ++ks) {
      const float* row = part + ((int64_t)ks * M + t) * ld;
      const float4 v = *reinterpret_cast<const float4*>(row + m);
      if (ks == 0) { a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w; }
      else {
        a[0] = __fadd_rn(a[0], v.x); a[1] = __fadd_rn(a[1], v.y);
        a[2] = __fadd_rn(a[2], v.z); a[3] = __fadd_rn(a[3], v.w);
      }
      if (MODE == kGateUp) {
        const float4 u = *reinterpret_cast<const float4*>(row + cols + m);
        if (ks == 0) { g[0] = u.x; g[1] = u.y; g[2] = u.z; g[3] = u.w; }
        else {
          g[0] = __fadd_rn(g[0], u.x); g[1] = __fadd_rn(g[1], u.y);
          g[2] = __fadd_rn(g[2], u.z); g[3] = __fadd_rn(g[3], u.w);
        }
      }
    }
    __nv_bfloat16 o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (MODE == kGateUp) {
        // a = the w1 (gate) sum, g = the w3 (up) sum
        const float h = act_kind == MOE_ACT_SITU ? situ_mul(a[j], g[j], b_eff, lbeta, has_lb)
                                                 : silu_mul(a[j], g[j]);
        o[j] = __float2bfloat16_rn(h);
      } else {
        o[j] = down_out(a[j], res, (int)t, cols, m + j);
      }
    }
    __nv_bfloat16* dst = out + t * cols + m;
    *reinterpret_cast<__nv_bfloat162*>(dst) = __halves2bfloat162(o[0], o[1]);
    *reinterpret_cast<__nv_bfloat162*>(dst + 2) = __halves2bfloat162(o[2], o[3]);
  }
}

// Split factor of a dense layer (one expert, M rows): enough units for the
// 148 SMs of a B200, at least two k-blocks per split; 1 when the layer already
// fills the GPU.  A function of the shapes only, so workspace sizes can be
// computed before a device is chosen.
constexpr int kSplitTargetUnits = 148;
int dense_ksplit(Variant v, int mode, int64_t M, int M_rows, int Kdim) {
  if (v == kVarLarge || M <= 0 || M_rows <= 0) return 1;
  const int nt = v == kVarDecode ? kNtDecode : kNtMid;
  const int um = v == kVarDecode ? kUmDecode : kUmMid;
  const int ks = BK * (v == kVarDecode ? kKsubDecode : kKsubMid);
  const int unit_rows = um * (mode == kGateUp ? kGateUpRows : BM);
  const int64_t units = ((M + nt - 1) / nt) * ((M_rows + unit_rows - 1) / unit_rows);
  const int sms = kSplitTargetUnits;
  if (units * 2 >= sms) return 1;
  int k = (int)((sms + units - 1) / units);
  const int kb = Kdim / ks;
  if (k > kb / 2) k = kb / 2;
  if (k > 32) k = 32;
  return k < 1 ? 1 : k;
}

template <int MODE>
cudaError_t launch_dense(Variant var, const CUtensorMap& a0, const CUtensorMap& a1,
                         const CUtensorMap& b, const CUtensorMap& b64, const int32_t* tiles,
                         int64_t M, int M_rows, int Kdim, __nv_bfloat16* out,
                         const __nv_bfloat16* res, const moe_act_cfg& act, DeviceStatus* st,
                         cudaStream_t s, bool pdl_ok, float* part) {
  const int32_t* ts = tiles + 2 + 2 * (int)var;
  const int ksplit = part ? dense_ksplit(var, MODE, M, M_rows, Kdim) : 1;
  if (ksplit <= 1)
    return launch_variant<MODE>(var, a0, a1, b, b64, tiles, ts, 1, M_rows, Kdim, out, res, act,
                                st, s, pdl_ok);
  cudaError_t e =
      var == kVarDecode
          ? launch_gemm<MODE, kNtDecode, kStagesDecode, kUmDecode, kKsubDecode>(
                a0, a1, b, b64, tiles, ts, 1, M_rows, Kdim, out, res, act, st, s, pdl_ok,
                nullptr, 1, 0, ksplit, part)
          : launch_gemm<MODE, kNtMid, kStagesMid, kUmMid, kKsubMid>(
                a0, a1, b, b64, tiles, ts, 1, M_rows, Kdim, out, res, act, st, s, pdl_ok,
                nullptr, 1, 0, ksplit, part);
  if (e != cudaSuccess) return e;
  const int64_t n4 = M * M_rows / 4;
  int64_t blocks = (n4 + 255) / 256;
  const int64_t cap = (int64_t)dev_info()->sm_count * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_splitk_reduce<MODE>, dim3((unsigned)blocks), dim3(256), 0, s,
                    (const float*)part, ksplit, M, M_rows, res, out, (int)act.kind, act.beta,
                    act.linear_beta);
}
}  // namespace

size_t dense_part_bytes(int64_t M, int K, int Nout, bool gate_up) {
  const Variant v = pick_variant(M, 1);
  const int k = dense_ksplit(v, gate_up ? kGateUp : kDown, M, Nout, K);
  if (k <= 1) return 0;
  return align_up(sizeof(float) * (size_t)k * (size_t)M * (size_t)Nout * (gate_up ? 2 : 1), 256);
}

__global__ void k_dense_tiles(int64_t M, int32_t* __restrict__ tiles) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    tiles[0] = 0;  // offsets
    tiles[1] = (int32_t)M;
    tiles[2] = 0;  // tile_start for each variant's token tile
    tiles[3] = (int32_t)((M + kNtDecode - 1) / kNtDecode);
    tiles[4] = 0;
    tiles[5] = (int32_t)((M + kNtMid - 1) / kNtMid);
    tiles[6] = 0;
    tiles[7] = (int32_t)((M + kPairNt - 1) / kPairNt);
  }
}

cudaError_t launch_dense_tiles(int64_t M, int32_t* tiles, cudaStream_t s) {
  return launch_pdl(k_dense_tiles, dim3(1), dim3(32), 0, s, M, tiles);
}

int linear_run(const __nv_bfloat16* x, int64_t M, int K, const __nv_bfloat16* W, int Nout,
               const __nv_bfloat16* residual, __nv_bfloat16* y, const int32_t* tiles,
               DeviceStatus* st, cudaStream_t s, bool pdl_ok, float* part) {
  CUtensorMap mw, mx, mx64;
  if (!make_map_3d(&mw, W, K, Nout, 1, BM) || !make_map_2d(&mx, x, K, M, kBoxRows) ||
      !make_map_2d(&mx64, x, K, M, kBigBoxRows))
    return MOE_ERR_CUDA;
  const Variant var = pick_variant(M, 1);
  const moe_act_cfg none = {MOE_ACT_SILU, 1.0f, 0.0f};
  return launch_dense<kDown>(var, mw, mw, mx, mx64, tiles, M, Nout, K, y, residual, none, st, s,
                             pdl_ok, part) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int shared_ffn_run(const __nv_bfloat16* x, int64_t M, int d, int F, const __nv_bfloat16* w1,
                   const __nv_bfloat16* w3, const __nv_bfloat16* w2, const moe_act_cfg& act,
                   const __nv_bfloat16* residual, __nv_bfloat16* y, __nv_bfloat16* h,
                   const int32_t* tiles, DeviceStatus* st, cudaStream_t s, float* part) {
  CUtensorMap mw1, mw3, mw2, mx, mh, mx64, mh64;
  if (!make_map_3d(&mw1, w1, d, F, 1, kGateUpRows) || !make_map_3d(&mw3, w3, d, F, 1, kGateUpRows) ||
      !make_map_3d(&mw2, w2, F, d, 1, BM) || !make_map_2d(&mx, x, d, M, kBoxRows) ||
      !make_map_2d(&mh, h, F, M, kBoxRows) || !make_map_2d(&mx64, x, d, M, kBigBoxRows) ||
      !make_map_2d(&mh64, h, F, M, kBigBoxRows))
    return MOE_ERR_CUDA;
  const Variant var = pick_variant(M, 1);
  if (launch_dense<kGateUp>(var, mw1, mw3, mx, mx64, tiles, M, F, d, h, nullptr, act, st, s,
                            false, part) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_dense<kDown>(var, mw2, mw2, mh, mh64, tiles, M, d, F, y, residual, act, st, s,
                             true, part) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // namespace moe

extern "C" int moe_set_wait_probe(int on) {
  return moe::g_wait_probe.exchange(on ? 1 : 0);
}
