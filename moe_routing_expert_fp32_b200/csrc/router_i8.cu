// router_i8.cu -- the router's fp32 gate GEMM on the int8 tensor cores, for
// batches large enough to fill the GPU.
//
// "Kimi K2 · Affinities", gate-forward excerpt: logits = F.linear of the fp32
// hidden states with the fp32 gate weight.  Tensor-core fp32 accumulation
// is not accurate enough for that (routing weights must agree to 1e-5), but
// integer accumulation is exact, so the product is split into exact int8
// pieces (a slicing scheme in the manner of Ozaki's error-free splitting):
//   * every row (a token's x, an expert's W) gets a power-of-two scale 2^sig
//     with |v| < 2^sig, and v / 2^sig is cut into PS = 4 signed 7-bit digits
//     (read off the float's bits; finite inputs):
//     v = 2^sig * sum_p a_p 2^(-7(p+1)) + r,   |r| < 2^(sig-28)
//     (bf16 x is always exact in 4 digits when its exponent range is < 20);
//   * x . w = 2^(sig_t + sig_e - 14) * sum_s 2^(-7s) S_s,
//     S_s = sum_{i+k=s} (x digits i) . (w digits k), an exact int32 dot product
//     over d (|S_s| < 4 * 127^2 * d < 2^31 for d <= 32768);
//   * pairs with i + k > 4 are dropped; with the digit truncation the logit
//     error stays below ~2e-8 for unit-variance x and 0.02-scale W, far below
//     one fp32 ulp of a logit of size 1.
// Kernels: k_slice_rows cuts W's rows into digit planes in memory (W is small
// and read by every token tile); k_row_sig takes each token row's scale;
// k_gate_i8 is persistent over (token tile, expert tile) pairs: TMA brings W's
// digit planes and the token tile as bf16, eight slicer warps cut the tile's
// digits into shared memory (so x's digit planes never exist in global
// memory), and one thread issues the 13 int8 products per k-block
// (tcgen05.mma kind::i8) into five int32 TMEM accumulators (one per s); the
// epilogue recombines them in double and rounds once to fp32.
#include <cuda.h>
#include <math.h>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int PS = 4;            // digits per operand
constexpr int SMAX = 4;          // keep digit pairs with i + k <= SMAX
constexpr int NACC = SMAX + 1;   // accumulators, one per i + k
constexpr int IM = 128;          // experts per tile (MMA M)
constexpr int INT = 96;          // tokens per tile (MMA N)
constexpr int IKB = 64;          // K bytes per stage (64-byte swizzle rows)
constexpr int IUK = 32;          // K per tcgen05.mma kind::i8
constexpr int ISTAGES = 3;

constexpr int kAStageBytes = PS * IM * IKB;   // 32 KB: W's digit planes
constexpr int kBStageBytes = PS * INT * IKB;  // 24 KB: the token tile's digit planes
static_assert(NACC * INT <= 512, "TMEM columns");

// ------------------------------------------------------------------ slicing
// Row scale: sig with max|v| < 2^sig (frexp exponent of the row maximum).
__device__ __forceinline__ int row_sig(float m) {
  int e = 0;
  frexp((double)m, &e);
  return m > 0.f ? e : 0;
}

// The 4 digits of v / 2^sig, read off the float's bits: |v| = M * 2^(Ebits-150)
// (M the 24-bit significand), so X = floor(|v| * 2^(28-sig)) is M shifted by
// Ebits - 122 - sig, and digit p is bits 21-7p .. 27-7p of X, with v's sign.
// This equals the truncation v/2^sig -> 128 r -> trunc -> ... done exactly.
__device__ __forceinline__ uint32_t fixed28(uint32_t bits, int sig) {
  const int eb = (int)((bits >> 23) & 0xFFu);
  const uint32_t mant = bits & 0x7FFFFFu;
  const uint32_t M = eb ? (mant | 0x800000u) : mant;
  const int sh = (eb ? eb : 1) - 122 - sig;
  if (sh >= 0) return M << sh;  // sh <= 4 because |v| < 2^sig
  return sh > -32 ? M >> (-sh) : 0u;
}
__device__ __forceinline__ void digits4(uint32_t bits, int sig, int8_t* d) {
  const uint32_t X = fixed28(bits, sig);
  const bool neg = (bits >> 31) != 0;
#pragma unroll
  for (int p = 0; p < PS; ++p) {
    const int a = (int)((X >> (7 * (PS - 1 - p))) & 0x7Fu);
    d[p] = (int8_t)(neg ? -a : a);
  }
}

template <typename T>
struct Vec;  // 16-byte loads: 4 fp32 or 8 bf16 per thread
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void bits(const uint4 r, uint32_t* b) {
    b[0] = r.x; b[1] = r.y; b[2] = r.z; b[3] = r.w;
  }
};
constexpr int kSliceThreads = 256;

// The largest |v| of one 16-byte vector, as the bits of an fp32 (|v| bits
// order like |v|).
template <typename T>
__device__ __forceinline__ uint32_t vec_absmax(const uint4 r) {
  uint32_t b[Vec<T>::n];
  Vec<T>::bits(r, b);
  uint32_t mx = 0;
#pragma unroll
  for (int i = 0; i < Vec<T>::n; ++i) mx = max(mx, b[i] & 0x7FFFFFFFu);
  return mx;
}
// bf16: the magnitudes of each pair maxed as bf16x2 (exact), then the pair.
template <>
__device__ __forceinline__ uint32_t vec_absmax<__nv_bfloat16>(const uint4 r) {
  const uint32_t w[4] = {r.x & 0x7FFF7FFFu, r.y & 0x7FFF7FFFu, r.z & 0x7FFF7FFFu,
                         r.w & 0x7FFF7FFFu};
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(w);
  const __nv_bfloat162 m2 = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
  const uint32_t mb = *reinterpret_cast<const uint32_t*>(&m2);
  return max(mb << 16, mb & 0xFFFF0000u);
}

// A row's scale: sig (max|v| < 2^sig) and 2^(28 - sig) as the product s1 * s2
// of two normal floats (28 - sig reaches 160 for the smallest bf16 rows).
struct RowScale {
  int sig;
  float s1, s2;
};
__device__ __forceinline__ RowScale row_scale(int sig) {
  const int k = 28 - sig;
  const int k1 = k < 127 ? k : 127;
  return {sig, __uint_as_float((uint32_t)(k1 + 127) << 23),
          __uint_as_float((uint32_t)(k - k1 + 127) << 23)};
}

// The PS digit planes of one vector of n elements starting at column j.
template <typename T>
__device__ __forceinline__ void store_digits(const uint4 r, const RowScale& sc,
                                             int8_t* __restrict__ out, int64_t plane,
                                             int64_t row, int d, int j) {
  constexpr int VN = Vec<T>::n;
  uint32_t b[VN];
  Vec<T>::bits(r, b);
  int8_t a[VN][PS];
#pragma unroll
  for (int i = 0; i < VN; ++i) digits4(b[i], sc.sig, a[i]);
#pragma unroll
  for (int p = 0; p < PS; ++p) {
    uint32_t w[VN / 4];
#pragma unroll
    for (int q = 0; q < VN / 4; ++q)
      w[q] = (uint32_t)(uint8_t)a[4 * q][p] | ((uint32_t)(uint8_t)a[4 * q + 1][p] << 8) |
             ((uint32_t)(uint8_t)a[4 * q + 2][p] << 16) |
             ((uint32_t)(uint8_t)a[4 * q + 3][p] << 24);
    int8_t* dst = out + p * plane + row * d + j;
    if (VN == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[VN / 4 - 1]);
    else *reinterpret_cast<uint32_t*>(dst) = w[0];
  }
}

// bf16 rows, four elements at a time.  X = floor(|v| * 2^(28 - sig)) in
// floating point: the products are power-of-two scalings, exact unless one
// falls below 2^-126 (then X is 0 either way), the result is below 2^28
// because |v| < 2^sig, and the conversion truncates.  spread_bf16 puts digit
// p of X in byte 3-p; a 4 x 4 byte transpose turns four such words into one
// word per digit plane, and negative elements are negated bytewise:
// -a == (0x80 - a) ^ 0x80 for 0 <= a <= 127, so no byte borrows.
__device__ __forceinline__ uint32_t spread_bf16(uint32_t abs_bits, const RowScale& sc) {
  const float v = __uint_as_float(abs_bits);  // |v| as fp32
  const uint32_t X = __float2uint_rz(__fmul_rn(__fmul_rn(v, sc.s1), sc.s2));
  return (X & 0x7Fu) | ((X << 1) & 0x7F00u) | ((X << 2) & 0x7F0000u) | ((X << 3) & 0x7F000000u);
}

// Byte i = 0xFF where element i of {a.lo, a.hi, b.lo, b.hi} is negative
// (prmt selectors with the sign-replicate bit, on bytes 1, 3, 5 and 7).
__device__ __forceinline__ uint32_t sign_bytes(uint32_t a, uint32_t b) {
  uint32_t m;
  asm("prmt.b32 %0, %1, %2, 0xFDB9;" : "=r"(m) : "r"(a), "r"(b));
  return m;
}

// The four digit-plane words of elements {a.lo, a.hi, b.lo, b.hi}.
__device__ __forceinline__ void planes4_bf16(uint32_t a, uint32_t b, const RowScale& sc,
                                             uint32_t* P) {
  const uint32_t y0 = spread_bf16((a & 0x7FFFu) << 16, sc), y1 = spread_bf16(a & 0x7FFF0000u, sc);
  const uint32_t y2 = spread_bf16((b & 0x7FFFu) << 16, sc), y3 = spread_bf16(b & 0x7FFF0000u, sc);
  const uint32_t lo01 = __byte_perm(y0, y1, 0x5140), hi01 = __byte_perm(y0, y1, 0x7362);
  const uint32_t lo23 = __byte_perm(y2, y3, 0x5140), hi23 = __byte_perm(y2, y3, 0x7362);
  const uint32_t m = sign_bytes(a, b);
  const uint32_t q[PS] = {__byte_perm(hi01, hi23, 0x7632), __byte_perm(hi01, hi23, 0x5410),
                          __byte_perm(lo01, lo23, 0x7632), __byte_perm(lo01, lo23, 0x5410)};
#pragma unroll
  for (int p = 0; p < PS; ++p) {
    const uint32_t neg = (0x80808080u - q[p]) ^ 0x80808080u;
    P[p] = (neg & m) | (q[p] & ~m);
  }
}

// One block per row: row maximum -> scale, then the 4 digits of every element
// (d % 8 == 0).  out: [PS][rows][d] int8.  With R > 0 (rows of at most
// R * 256 vectors) every thread keeps its R vectors in registers, so the row
// is read once with all of its loads in flight together; R == 0 reads the
// row twice (any d).
template <typename T, int R>
__global__ void __launch_bounds__(kSliceThreads) k_slice_rows(const T* __restrict__ v,
                                                              int64_t rows, int d,
                                                              int8_t* __restrict__ out,
                                                              int* __restrict__ sig_out) {
  pdl_wait();
  pdl_trigger();
  constexpr int VN = Vec<T>::n;
  constexpr int kStep = kSliceThreads * VN;
  __shared__ uint32_t wmax[kSliceThreads / 32];
  const int64_t row = blockIdx.x;
  const T* src = v + row * d;
  uint4 held[R > 0 ? R : 1];
  uint32_t mx = 0;
  if constexpr (R > 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = r * kStep + threadIdx.x * VN;
      held[r] = j < d ? *reinterpret_cast<const uint4*>(src + j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) mx = max(mx, vec_absmax<T>(held[r]));
  } else {
    for (int j = threadIdx.x * VN; j < d; j += kStep)
      mx = max(mx, vec_absmax<T>(*reinterpret_cast<const uint4*>(src + j)));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
  __syncthreads();
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kSliceThreads / 32; ++i) m = max(m, wmax[i]);
  const int sig = row_sig(__uint_as_float(m));
  if (threadIdx.x == 0) sig_out[row] = sig;
  const RowScale sc = row_scale(sig);
  const int64_t plane = rows * (int64_t)d;
  if constexpr (R > 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = r * kStep + threadIdx.x * VN;
      if (j < d) store_digits<T>(held[r], sc, out, plane, row, d, j);
    }
  } else {
    for (int j = threadIdx.x * VN; j < d; j += kStep)
      store_digits<T>(*reinterpret_cast<const uint4*>(src + j), sc, out, plane, row, d, j);
  }
}

// Launch with the smallest register tile that holds a row.
template <typename T>
cudaError_t launch_slice_rows(const T* v, int64_t rows, int d, int8_t* out, int* sig,
                              cudaStream_t s) {
  const int steps = (d + kSliceThreads * Vec<T>::n - 1) / (kSliceThreads * Vec<T>::n);
  const dim3 g((unsigned)rows), b(kSliceThreads);
  if (steps <= 1) return launch_pdl(k_slice_rows<T, 1>, g, b, 0, s, v, rows, d, out, sig);
  if (steps <= 2) return launch_pdl(k_slice_rows<T, 2>, g, b, 0, s, v, rows, d, out, sig);
  if (steps <= 4) return launch_pdl(k_slice_rows<T, 4>, g, b, 0, s, v, rows, d, out, sig);
  if (steps <= 8) return launch_pdl(k_slice_rows<T, 8>, g, b, 0, s, v, rows, d, out, sig);
  return launch_pdl(k_slice_rows<T, 0>, g, b, 0, s, v, rows, d, out, sig);
}

// Row scale of every token: one warp per row reads it once (16-byte vectors,
// bf16 maxima in pairs) and writes sig with max|x| < 2^sig (0 for a zero
// row), exactly as k_slice_rows computes it.
constexpr int kSigWarps = 8;
__global__ void __launch_bounds__(32 * kSigWarps) k_row_sig(const __nv_bfloat16* __restrict__ x,
                                                           int64_t rows, int d,
                                                           int* __restrict__ sig_out) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kSigWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * d);
  const int nv = d / 8;
  uint32_t mx = 0;
  int j = lane;
  for (; j + 96 < nv; j += 128) {  // four loads in flight per lane
    const uint4 a = src[j], b = src[j + 32], c = src[j + 64], e = src[j + 96];
    mx = max(mx, max(max(vec_absmax<__nv_bfloat16>(a), vec_absmax<__nv_bfloat16>(b)),
                     max(vec_absmax<__nv_bfloat16>(c), vec_absmax<__nv_bfloat16>(e))));
  }
  for (; j < nv; j += 32) mx = max(mx, vec_absmax<__nv_bfloat16>(src[j]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) sig_out[row] = row_sig(__uint_as_float(mx));
}

// ------------------------------------------------------------ the GEMM
// s8 x s8 -> s32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(IM >> 4) << 24);
}
__device__ __forceinline__ void umma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// K-major int8 operand in the 64-byte swizzle: rows of 64 bytes, 8-row groups
// 512 bytes apart.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return sm100::smem_desc(saddr, 512, 4);
}
// Byte offset of columns 8c .. 8c+7 of row r in a 64-byte-swizzled plane:
// 16-byte unit g of a row sits at unit g ^ ((r >> 1) & 3) (the swizzle
// repeats every 8 rows = 512 bytes).
__device__ __forceinline__ uint32_t sw64_off(int r, int c) {
  return (uint32_t)r * IKB + ((((uint32_t)c >> 1) ^ (((uint32_t)r >> 1) & 3u)) << 4) +
         ((uint32_t)c & 1u) * 8u;
}

// Persistent over tiles u = blockIdx.x, +gridDim.x, ...: token tile u / ET,
// expert tile u % ET (the expert tiles of one token tile run side by side, so
// its rows are read from L2 after the first).  Roles:
//   warp 0        TMA: W digit planes (4 x 128 rows x 64 B) and the token
//                 tile (96 rows x 64 bf16, zero rows past N) per k-block,
//                 both on tma_full[stage];
//   warp 1        TMEM owner; one thread issues the MMAs of a k-block once
//                 the slicers have filled it (full[stage]) and frees the
//                 stage by a commit to empty[stage];
//   warps 2-5     epilogue: the five accumulators of a tile -> logits;
//   warps 6-13    slicers: the token tile's digits into the stage's B planes
//                 (each thread: rows r, r+32, r+64, one 16-byte column chunk).
// One TMEM buffer (5 x 96 of 512 columns): the next tile's MMAs wait for the
// epilogue (tfull / tempty).  Every wait is bounded; a wait that runs out
// records MOE_ERR_DEVICE_TIMEOUT and the roles stop; the producer then waits
// (bounded) for the copies it issued, and TMEM is freed before the CTA exits.
constexpr int kSliceWarpsI8 = 8;
constexpr int kThreadsI8 = 32 * (6 + kSliceWarpsI8);
constexpr int kXStageRaw = INT * IKB * 2;  // the token tile as bf16, 128-byte rows
constexpr int kStageBytesI8 = kAStageBytes + kBStageBytes + kXStageRaw;
constexpr size_t kSmemI8 = (size_t)ISTAGES * kStageBytesI8 + 1024 + 256;
static_assert(kSmemI8 <= 227 * 1024, "shared memory");
static_assert(kStageBytesI8 % 1024 == 0, "stage alignment");
static_assert(kSliceWarpsI8 * 32 * 3 == INT * 8, "slicer threads: 3 row chunks each");

__global__ void __launch_bounds__(kThreadsI8, 1)
    k_gate_i8(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const int* __restrict__ sig_w, const int* __restrict__ sig_x, int64_t N, int E,
              int d, float* __restrict__ logits, DeviceStatus* st) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* tma_full = reinterpret_cast<uint64_t*>(smem + ISTAGES * kStageBytesI8);
  uint64_t* full = tma_full + ISTAGES;
  uint64_t* empty = full + ISTAGES;
  uint64_t* tfull = empty + ISTAGES;
  uint64_t* tempty = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ET = (E + IM - 1) / IM;
  const int64_t tiles = (int64_t)ET * ((N + INT - 1) / INT);
  const int KB = d / IKB;
  // W's digit planes and the row scales come from the two kernels before
  pdl_wait();
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < ISTAGES; ++s) {
      mbar_init(&tma_full[s], 1);
      mbar_init(&full[s], kSliceWarpsI8);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 128);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < tiles && ok; u += gridDim.x) {
        const int e0 = (int)(u % ET) * IM;
        const int t0 = (int)(u / ET) * INT;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * kStageBytesI8;
          uint8_t* sRaw = sA + kAStageBytes + kBStageBytes;
          mbar_arrive_expect_tx(&tma_full[stage], kAStageBytes + kXStageRaw);
#pragma unroll
          for (int p = 0; p < PS; ++p)
            tma_load_3d(&tmW, &tma_full[stage], sA + p * IM * IKB, kb * IKB, e0, p);
          tma_load_2d(&tmX, &tma_full[stage], sRaw, kb * IKB, t0);
          ++issued;
          if (++stage == ISTAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 300);
        *abort_flag = 1;
      }
      // no copy of this CTA may still be in flight when it exits
      volatile int never = 0;
      for (int64_t k = issued - 1; k >= 0 && k >= issued - ISTAGES; --k)
        if (!mbar_wait(&tma_full[k % ISTAGES], (uint32_t)((k / ISTAGES) & 1), &never))
          record_error(st, MOE_ERR_DEVICE_TIMEOUT, 301);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(INT);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int64_t u = blockIdx.x; u < tiles && ok; u += gridDim.x, ++local) {
        if (!mbar_wait(tempty, (local & 1) ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * kStageBytesI8);
          const uint32_t b0 = a0 + kAStageBytes;
          // digit pairs (i of x, k of W), grouped by s = i + k
#pragma unroll
          for (int s = 0; s <= SMAX; ++s) {
            bool first = kb == 0;
#pragma unroll
            for (int i = 0; i < PS; ++i) {
              const int k = s - i;
              if (k < 0 || k >= PS) continue;
#pragma unroll
              for (int h = 0; h < IKB / IUK; ++h) {
                umma_i8(tmem + s * INT, sw64_desc(a0 + k * IM * IKB + h * IUK),
                        sw64_desc(b0 + i * INT * IKB + h * IUK), idesc, first ? 0u : 1u);
                first = false;
              }
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == ISTAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) umma_commit(tfull);
      }
      if (!ok) {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 310);
        *abort_flag = 1;
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32 * quarter .. + 31
    const int el = quarter * 32 + lane;
    int local = 0;
    for (int64_t u = blockIdx.x; u < tiles; u += gridDim.x, ++local) {
      const int e = (int)(u % ET) * IM + el;
      const int64_t t0 = (u / ET) * INT;
      if (!mbar_wait(tfull, local & 1, abort_flag)) {
        if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 320);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
      const int sw = e < E ? sig_w[e] : 0;
      for (int c0 = 0; c0 < INT; c0 += 16) {
        // v = sum_s 2^(-7s) S_s by Horner from s = NACC - 1 down (exact in
        // double: every step is a power-of-two scaling and a 31-bit add)
        double v[16];
        uint32_t a[16];
        tmem_ld16(taddr + (NACC - 1) * INT + c0, a);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = (double)(int32_t)a[j];
#pragma unroll
        for (int s = NACC - 2; s >= 0; --s) {
          tmem_ld16(taddr + s * INT + c0, a);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = v[j] * 0x1p-7 + (double)(int32_t)a[j];
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int64_t t = t0 + c0 + j;
          if (t < N && e < E) logits[t * E + e] = (float)ldexp(v[j], sig_x[t] + sw - 14);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty);
    }
  } else {
    // ------------------------------------------------------------- slicers
    const int ts = threadIdx.x - 192;  // 0 .. 255
    const int c = ts & 7;              // 16-byte chunk of the 128-byte bf16 row
    const int r0 = ts >> 3;            // rows r0, r0 + 32, r0 + 64
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < tiles && ok; u += gridDim.x) {
      const int64_t t0 = (u / ET) * INT;
      RowScale sc[3];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int64_t t = t0 + r0 + 32 * j;
        sc[j] = row_scale(t < N ? sig_x[t] : 0);
      }
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&tma_full[stage], phase, abort_flag)) { ok = false; break; }
        uint8_t* sB = smem + stage * kStageBytesI8 + kAStageBytes;
        const uint8_t* sRaw = sB + kBStageBytes;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int r = r0 + 32 * j;
          const uint4 v = *reinterpret_cast<const uint4*>(sRaw + r * (IKB * 2) + c * 16);
          uint32_t P0[PS], P1[PS];
          planes4_bf16(v.x, v.y, sc[j], P0);
          planes4_bf16(v.z, v.w, sc[j], P1);
          const uint32_t off = sw64_off(r, c);
#pragma unroll
          for (int p = 0; p < PS; ++p)
            *reinterpret_cast<uint2*>(sB + p * INT * IKB + off) = make_uint2(P0[p], P1[p]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == ISTAGES) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) {
      if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 330);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

typedef CUresult (*EncodeTiledFnI8)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnI8 encode_i8() {
  static const EncodeTiledFnI8 fn = [] {  // looked up once (thread-safe static)
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFnI8>(p);
    return static_cast<EncodeTiledFnI8>(nullptr);
  }();
  return fn;
}

// [planes][rows][d] int8, box 64 bytes x box_rows x 1, 64-byte swizzle
bool map_planes(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFnI8 fn = encode_i8();
  if (!fn) return false;
  cuuint64_t dims[3] = {d, rows, (cuuint64_t)PS};
  cuuint64_t strides[2] = {d, d * rows};
  cuuint32_t box[3] = {(cuuint32_t)IKB, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// x [rows][d] bf16, box 64 columns x box_rows, no swizzle (128-byte rows);
// rows past the end read as zero
bool map_rows_bf16(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows,
                   uint32_t box_rows) {
  EncodeTiledFnI8 fn = encode_i8();
  if (!fn) return false;
  cuuint64_t dims[2] = {d, rows};
  cuuint64_t strides[1] = {d * 2};
  cuuint32_t box[2] = {(cuuint32_t)IKB, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct I8Layout {
  size_t logits, wd, ws, xs, total;
};

I8Layout i8_layout(int64_t N, int E, int d) {
  I8Layout L{};
  size_t o = 0;
  L.logits = o; o += align_up(sizeof(float) * (size_t)N * E, 256);
  L.wd = o; o += align_up((size_t)PS * E * d, 256);
  L.ws = o; o += align_up(sizeof(int) * (size_t)E, 256);
  L.xs = o; o += align_up(sizeof(int) * (size_t)N, 256);
  L.total = o;
  return L;
}

}  // namespace

bool gate_i8_applies(int64_t N, int E, int d_r) {
  const int64_t tiles = ((E + IM - 1) / IM) * ((N + INT - 1) / INT);
  return tiles >= 24 && d_r % IKB == 0 && d_r <= 32768;  // d_r % 64 also serves the slicers
}

size_t gate_i8_scratch_bytes(int64_t N, int E, int d_r) { return i8_layout(N, E, d_r).total; }

cudaError_t launch_gate_i8(const __nv_bfloat16* x, int64_t N, int d_r, const float* W, int E,
                           void* scratch, DeviceStatus* st, cudaStream_t s) {
  const I8Layout L = i8_layout(N, E, d_r);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  float* logits = reinterpret_cast<float*>(base + L.logits);
  int8_t* wd = reinterpret_cast<int8_t*>(base + L.wd);
  int* wsig = reinterpret_cast<int*>(base + L.ws);
  int* xsig = reinterpret_cast<int*>(base + L.xs);
  CUtensorMap mw, mx;
  if (!map_planes(&mw, wd, d_r, E, IM) || !map_rows_bf16(&mx, x, d_r, N, INT))
    return cudaErrorInvalidValue;
  static std::once_flag once[kMaxDevices];
  static cudaError_t set_up[kMaxDevices];
  const cudaError_t e0 = once_per_device(once, set_up, [](int) {
    return cudaFuncSetAttribute(k_gate_i8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemI8);
  });
  if (e0 != cudaSuccess) return e0;
  cudaError_t e = launch_slice_rows(W, E, d_r, wd, wsig, s);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_row_sig, dim3((unsigned)((N + kSigWarps - 1) / kSigWarps)),
                 dim3(32 * kSigWarps), 0, s, x, N, d_r, xsig);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (int64_t)((E + IM - 1) / IM) * ((N + INT - 1) / INT);
  const int64_t grid = tiles < dev_info()->sm_count ? tiles : dev_info()->sm_count;
  return launch_pdl(k_gate_i8, dim3((unsigned)grid), dim3(kThreadsI8), kSmemI8, s, mw, mx,
                    (const int*)wsig, (const int*)xsig, N, E, d_r, logits, st);
}

}  // namespace moe
