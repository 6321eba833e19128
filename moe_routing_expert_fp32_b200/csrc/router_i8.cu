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
// k_slice_* cut the rows; k_gate_i8 runs the 13 int8 products per k-block
// with tcgen05.mma kind::i8 into five int32 TMEM accumulators (one per s) and
// recombines them in double in its epilogue, rounding once to fp32.
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
constexpr int kThreadsI8 = 192;

constexpr int kAStageBytes = PS * IM * IKB;   // 32 KB
constexpr int kBStageBytes = PS * INT * IKB;  // 24 KB
constexpr int kStageBytesI8 = kAStageBytes + kBStageBytes;
constexpr size_t kSmemI8 = (size_t)ISTAGES * kStageBytesI8 + 1024 + 256;
static_assert(kSmemI8 <= 227 * 1024, "shared memory");
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
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void bits(const uint4 r, uint32_t* b) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      b[2 * i] = w[i] << 16;
      b[2 * i + 1] = w[i] & 0xFFFF0000u;
    }
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

template <>
__device__ __forceinline__ void store_digits<__nv_bfloat16>(const uint4 r, const RowScale& sc,
                                                            int8_t* __restrict__ out,
                                                            int64_t plane, int64_t row, int d,
                                                            int j) {
  uint32_t P0[PS], P1[PS];
  planes4_bf16(r.x, r.y, sc, P0);
  planes4_bf16(r.z, r.w, sc, P1);
#pragma unroll
  for (int p = 0; p < PS; ++p)
    *reinterpret_cast<uint2*>(out + p * plane + row * d + j) = make_uint2(P0[p], P1[p]);
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
void launch_slice_rows(const T* v, int64_t rows, int d, int8_t* out, int* sig, cudaStream_t s) {
  const int steps = (d + kSliceThreads * Vec<T>::n - 1) / (kSliceThreads * Vec<T>::n);
  const dim3 g((unsigned)rows), b(kSliceThreads);
  if (steps <= 1) k_slice_rows<T, 1><<<g, b, 0, s>>>(v, rows, d, out, sig);
  else if (steps <= 2) k_slice_rows<T, 2><<<g, b, 0, s>>>(v, rows, d, out, sig);
  else if (steps <= 4) k_slice_rows<T, 4><<<g, b, 0, s>>>(v, rows, d, out, sig);
  else if (steps <= 8) k_slice_rows<T, 8><<<g, b, 0, s>>>(v, rows, d, out, sig);
  else k_slice_rows<T, 0><<<g, b, 0, s>>>(v, rows, d, out, sig);
  (void)counted(cudaPeekAtLastError());
}

// -------------------------------------------------------------- PTX helpers
// (the shared ones are in sm100.cuh)
using sm100::mbar_arrive_expect_tx;
using sm100::mbar_init;
using sm100::mbar_wait;
using sm100::smem_u32;
using sm100::tc_fence_after;
using sm100::tc_fence_before;
using sm100::tma_load_3d;
using sm100::umma_commit;

__device__ __forceinline__ void umma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// 32 lanes x 16 consecutive int32 TMEM columns
__device__ __forceinline__ void tld16(uint32_t taddr, int32_t* v) {
  uint32_t r[16];
  sm100::tmem_ld16(taddr, r);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = (int32_t)r[i];
}
// K-major operand in 64-byte swizzle: rows of 64 bytes, 8-row groups 512 B apart.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return sm100::smem_desc(saddr, 512, 4);
}
// s8 x s8 -> s32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(IM >> 4) << 24);
}

// One 128-expert x 96-token tile per CTA.  Warp 0: TMA producer; warp 1: MMA
// issuer and TMEM owner; warps 2-5: epilogue.
__global__ void __launch_bounds__(kThreadsI8, 1)
    k_gate_i8(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
              const int* __restrict__ sig_w, const int* __restrict__ sig_x, int64_t N, int E,
              int d, float* __restrict__ logits, DeviceStatus* st) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ISTAGES * kStageBytesI8);
  uint64_t* empty = full + ISTAGES;
  uint64_t* tfull = empty + ISTAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * IM;
  const int64_t t0 = (int64_t)blockIdx.y * INT;
  const int KB = d / IKB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ISTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    sm100::mbar_init_fence();
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, 512);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
          record_error(st, MOE_ERR_DEVICE_TIMEOUT, 300);
          *abort_flag = 1;
          break;
        }
        uint8_t* sA = smem + stage * kStageBytesI8;
        uint8_t* sB = sA + kAStageBytes;
        mbar_arrive_expect_tx(&full[stage], kStageBytesI8);
#pragma unroll
        for (int p = 0; p < PS; ++p) {
          tma_load_3d(&tmW, &full[stage], sA + p * IM * IKB, kb * IKB, e0, p);
          tma_load_3d(&tmX, &full[stage], sB + p * INT * IKB, kb * IKB, (int)t0, p);
        }
        if (++stage == ISTAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(INT);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
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
      else {
        record_error(st, MOE_ERR_DEVICE_TIMEOUT, 310);
        *abort_flag = 1;
      }
    }
  } else {
    const int quarter = warp & 3;
    const int e = e0 + quarter * 32 + lane;
    if (mbar_wait(tfull, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16);
      const int sw = e < E ? sig_w[e] : 0;
      for (int c0 = 0; c0 < INT; c0 += 16) {
        int32_t acc[NACC][16];
#pragma unroll
        for (int s = 0; s < NACC; ++s) tld16(taddr + s * INT + c0, acc[s]);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int64_t t = t0 + c0 + j;
          if (t >= N || e >= E) continue;
          double v = 0.0;
#pragma unroll
          for (int s = NACC - 1; s >= 0; --s) v = v * 0x1p-7 + (double)acc[s][j];
          logits[t * E + e] = (float)ldexp(v, sig_x[t] + sw - 14);
        }
      }
    } else {
      if (lane == 0) record_error(st, MOE_ERR_DEVICE_TIMEOUT, 320);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
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

struct I8Layout {
  size_t logits, wd, ws, xd, xs, total;
};

I8Layout i8_layout(int64_t N, int E, int d) {
  I8Layout L{};
  size_t o = 0;
  L.logits = o; o += align_up(sizeof(float) * (size_t)N * E, 256);
  L.wd = o; o += align_up((size_t)PS * E * d, 256);
  L.ws = o; o += align_up(sizeof(int) * (size_t)E, 256);
  L.xd = o; o += align_up((size_t)PS * N * d, 256);
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
  int8_t* xd = reinterpret_cast<int8_t*>(base + L.xd);
  int* xsig = reinterpret_cast<int*>(base + L.xs);
  launch_slice_rows(W, E, d_r, wd, wsig, s);
  launch_slice_rows(x, N, d_r, xd, xsig, s);
  CUtensorMap mw, mx;
  if (!map_planes(&mw, wd, d_r, E, IM) || !map_planes(&mx, xd, d_r, N, INT))
    return cudaErrorInvalidValue;
  static std::once_flag once[kMaxDevices];
  static cudaError_t set_up[kMaxDevices];
  const cudaError_t e0 = once_per_device(once, set_up, [](int) {
    return cudaFuncSetAttribute(k_gate_i8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemI8);
  });
  if (e0 != cudaSuccess) return e0;
  dim3 grid((E + IM - 1) / IM, (unsigned)((N + INT - 1) / INT), 1);
  k_gate_i8<<<grid, kThreadsI8, kSmemI8, s>>>(mw, mx, wsig, xsig, N, E, d_r, logits, st);
  return counted(cudaGetLastError());  // the GEMM (each slicer launch was counted above)
}

}  // namespace moe
