// router.cu -- the fp32 router of the MoE layer.
//
// Follows "Kimi K2 · Affinities", gate-forward excerpt (MoEGate.forward with
// noaux_tc) and "DeepSeek-V3.2-Exp · Affinities", gate-forward excerpt
// (Gate.forward):
//   k_gate_partial : logits = x . W^T in fp32 (x upcast from bf16, W fp32) for
//                    batches too small to fill the GPU with int8 tensor-core
//                    tiles (router_i8.cu takes the others);
//                    decode batches split d_r over several CTAs (partials in
//                    double, summed by k_reduce_partials).  FMA chains are 32
//                    terms long and the 32-term blocks are added in double,
//                    which keeps the logit error near 1e-7 instead of the
//                    ~1e-5 of one 7168-term fp32 chain.
//   k_select       : one warp per token: sigmoid (or softmax), + bias, group
//                    top-2 sums (or group maxima),
//                    top-TG groups (others -> -inf), top-K experts by
//                    (score desc, index asc), unbiased weights, renormalise
//                    (sequential fp32 sum over k + 1e-20), route scale.
// Every fp32 step of k_select is an explicit round-to-nearest intrinsic, so no
// multiply-add is fused and the result is the IEEE result of the page's ops.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int GT = 64;    // tokens per tile
constexpr int GE = 64;    // experts per tile
constexpr int GK = 32;    // k per chunk = length of every fp32 FMA chain
constexpr int GEP = GE + 2;  // padded row of the transposed W tile (8-byte aligned)
constexpr float kNegInf = -INFINITY;

// logits (or split-K partials) of a 64-token x 64-expert tile.  Thread
// (tx = lane, ty = warp) owns tokens ty*8..ty*8+7 and experts tx*2, tx*2+1;
// the token values are warp-uniform (broadcast loads).  Each 32-wide k chunk
// is accumulated in fp32 (FMA) and then added to a double accumulator, so no
// fp32 rounding chain is longer than 32 terms.  Chunks are staged global ->
// registers -> shared memory one chunk ahead (double buffer).
__global__ void __launch_bounds__(256, 2) k_gate_partial(const __nv_bfloat16* __restrict__ x,
                                                         int64_t N, int d,
                                                         const float* __restrict__ W, int E,
                                                         int cps, int splits,
                                                         float* __restrict__ logits,
                                                         double* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float xs[2][GK][GT];
  __shared__ __align__(16) float wsm[2][GK][GEP];
  const int tid = threadIdx.x;
  const int tx = tid & 31, ty = tid >> 5;
  const int64_t t0 = (int64_t)blockIdx.y * GT;
  const int e0 = blockIdx.x * GE;
  const int nk = d / GK;
  const int kc0 = blockIdx.z * cps;
  const int kc1 = min(nk, kc0 + cps);

  // global -> register staging of one chunk: x 64 tokens x 32 k (one 16-byte
  // vector per thread), W 64 experts x 32 k (two float4 per thread)
  const int xtok = tid >> 2, xkk = (tid & 3) * 8;
  uint4 xr = make_uint4(0, 0, 0, 0);
  float4 wr[2];
  auto load_chunk = [&](int kc) {
    const int k0 = kc * GK;
    xr = make_uint4(0, 0, 0, 0);
    if (t0 + xtok < N) xr = *reinterpret_cast<const uint4*>(x + (t0 + xtok) * d + k0 + xkk);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + 256 * r;
      const int ex = i >> 3, kq = (i & 7) * 4;
      wr[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0 + ex < E)
        wr[r] = *reinterpret_cast<const float4*>(W + (int64_t)(e0 + ex) * d + k0 + kq);
    }
  };
  auto store_chunk = [&](int b) {
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&xr);
#pragma unroll
    for (int j = 0; j < 8; ++j) xs[b][xkk + j][xtok] = __bfloat162float(h[j]);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = tid + 256 * r;
      const int ex = i >> 3, kq = (i & 7) * 4;
      wsm[b][kq + 0][ex] = wr[r].x;
      wsm[b][kq + 1][ex] = wr[r].y;
      wsm[b][kq + 2][ex] = wr[r].z;
      wsm[b][kq + 3][ex] = wr[r].w;
    }
  };

  double acc[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = 0.0;
  // fp32 chains as packed pairs: p2[p][j] holds tokens 2p and 2p + 1 of
  // expert j; fma.rn.f32x2 rounds each half as fmaf does

  int buf = 0;
  if (kc0 < kc1) {
    load_chunk(kc0);
    store_chunk(0);
  }
  __syncthreads();
  for (int kc = kc0; kc < kc1; ++kc) {
    const bool more = kc + 1 < kc1;
    if (more) load_chunk(kc + 1);
    uint64_t p2[4][2];
#pragma unroll
    for (int q = 0; q < 4; ++q) p2[q][0] = p2[q][1] = 0ull;
#pragma unroll 8
    for (int k = 0; k < GK; ++k) {
      const ulonglong2 a0 = *reinterpret_cast<const ulonglong2*>(&xs[buf][k][ty * 8]);
      const ulonglong2 a1 = *reinterpret_cast<const ulonglong2*>(&xs[buf][k][ty * 8 + 4]);
      const float2 b = *reinterpret_cast<const float2*>(&wsm[buf][k][tx * 2]);
      const uint64_t av[4] = {a0.x, a0.y, a1.x, a1.y};
      uint64_t bb[2];
      asm("mov.b64 %0, {%1, %1};" : "=l"(bb[0]) : "r"(__float_as_uint(b.x)));
      asm("mov.b64 %0, {%1, %1};" : "=l"(bb[1]) : "r"(__float_as_uint(b.y)));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(p2[q][0]) : "l"(av[q]), "l"(bb[0]));
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(p2[q][1]) : "l"(av[q]), "l"(bb[1]));
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        acc[2 * q][j] += (double)__uint_as_float((uint32_t)p2[q][j]);
        acc[2 * q + 1][j] += (double)__uint_as_float((uint32_t)(p2[q][j] >> 32));
      }
    }
    if (more) store_chunk(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + ty * 8 + i;
    if (t >= N) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int e = e0 + tx * 2 + j;
      if (e >= E) continue;
      if (splits == 1) logits[t * E + e] = (float)acc[i][j];
      else part[((int64_t)blockIdx.z * N + t) * E + e] = acc[i][j];
    }
  }
}

// Split-K partials (double) -> logits, one thread per (token, expert): summed
// in split order in double and rounded once to fp32.
__global__ void __launch_bounds__(256) k_reduce_partials(const double* __restrict__ part,
                                                         int splits, int64_t NE,
                                                         float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < NE;
       i += (int64_t)gridDim.x * blockDim.x) {
    double a = 0.0;
    for (int z = 0; z < splits; ++z) a += part[(int64_t)z * NE + i];
    logits[i] = (float)a;
  }
}

// "a ranks before b": larger value first, ties to the lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_best(float& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (ranks_before(ov, oi, v, i)) { v = ov; i = oi; }
  }
}

constexpr int kSelWarps = 4;

__global__ void __launch_bounds__(32 * kSelWarps) k_select(
    const float* __restrict__ logits, int64_t N, int E, const float* __restrict__ bias,
    int G, int TG, int K, int norm, float route_scale, int score_func, int group_mode,
    int32_t* __restrict__ idx_out, float* __restrict__ w_out, DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* s_s = sm + warp * 2 * E;
  float* s_c = s_s + E;
  // softmax only: E doubles per warp after the float arrays
  double* s_x = reinterpret_cast<double*>(sm + kSelWarps * 2 * E) + warp * E;
  for (int64_t t = (int64_t)blockIdx.x * kSelWarps + warp; t < N;
       t += (int64_t)gridDim.x * kSelWarps) {
    const float* p = logits + t * E;
    // the token's logits first, all loads in flight together
    for (int e = lane; e < E; e += 32) s_s[e] = p[e];
    __syncwarp();
    if (score_func == MOE_SCORE_SOFTMAX) {
      // softmax over the E logits: exp(L - max) in double, summed in expert
      // order by one lane, quotient rounded once to fp32
      float mx = -INFINITY;
      for (int e = lane; e < E; e += 32) mx = fmaxf(mx, s_s[e]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      for (int e = lane; e < E; e += 32) s_x[e] = exp((double)s_s[e] - (double)mx);
      __syncwarp();
      double sum = 0.0;
      if (lane == 0)
        for (int e = 0; e < E; ++e) sum += s_x[e];
      sum = __shfl_sync(0xffffffffu, sum, 0);
      for (int e = lane; e < E; e += 32) {
        const float s = (float)(s_x[e] / sum);
        s_s[e] = s;
        s_c[e] = bias ? __fadd_rn(s, bias[e]) : s;
      }
    } else {
      for (int e = lane; e < E; e += 32) {
        // sigmoid: fp32 rounding of 1/(1+exp(-L)) evaluated in double
        // (__drcp_rn is the correctly rounded reciprocal, i.e. IEEE 1.0 / v)
        const float s = (float)__drcp_rn(1.0 + exp(-(double)s_s[e]));
        s_s[e] = s;
        s_c[e] = bias ? __fadd_rn(s, bias[e]) : s;
      }
    }
    __syncwarp();
    if (G > 1) {
      const int gsz = E / G;
      float gs = kNegInf;
      if (lane < G) {
        float a = kNegInf, b = kNegInf;
        for (int i = 0; i < gsz; ++i) {
          const float v = s_c[lane * gsz + i];
          if (v > a) { b = a; a = v; }
          else if (v > b) { b = v; }
        }
        gs = group_mode == MOE_GROUP_MAX ? a : __fadd_rn(a, b);
      }
      bool kept = false;
      for (int r = 0; r < TG; ++r) {
        float v = (lane < G && !kept) ? gs : kNegInf;
        int i = (lane < G && !kept) ? lane : 0x7fffffff;
        warp_best(v, i);
        if (lane == i) kept = true;
      }
      const unsigned keptmask = __ballot_sync(0xffffffffu, kept);
      for (int e = lane; e < E; e += 32)
        if (!((keptmask >> (e / gsz)) & 1u)) s_c[e] = kNegInf;
      __syncwarp();
    }
    unsigned chosen = 0;
    int my_e = 0;
    for (int k = 0; k < K; ++k) {
      float bv = kNegInf;
      int bi = 0x7fffffff;
      for (int i = 0, e = lane; e < E; ++i, e += 32) {
        if ((chosen >> i) & 1u) continue;
        const float v = s_c[e];
        if (ranks_before(v, e, bv, bi)) { bv = v; bi = e; }
      }
      warp_best(bv, bi);
      if (bi == 0x7fffffff) {  // cannot happen for a validated config
        record_error(st, MOE_ERR_DEVICE_BOUNDS, 1);
        bi = 0;
      }
      if ((bi & 31) == lane) chosen |= 1u << (bi >> 5);
      if (lane == k) my_e = bi;
    }
    float wk = (lane < K) ? s_s[my_e] : 0.f;
    if (K > 1 && norm) {
      float den = __shfl_sync(0xffffffffu, wk, 0);
      for (int k = 1; k < K; ++k) den = __fadd_rn(den, __shfl_sync(0xffffffffu, wk, k));
      den = __fadd_rn(den, 1e-20f);
      wk = __fdiv_rn(wk, den);
    }
    wk = __fmul_rn(wk, route_scale);
    if (lane < K) {
      idx_out[t * K + lane] = my_e;
      w_out[t * K + lane] = wk;
    }
    __syncwarp();
  }
}

// Small batches: one block per token, one thread per expert (blockDim = E
// rounded up to 32).  The logits come either from `logits` or, when the gate
// GEMM ran split over d_r, straight from its double partials (summed in split
// order and rounded once, exactly as k_reduce_partials does), so no reduce
// kernel runs.  The score of each expert is computed by its own thread.  Every
// "best of" step is a rank under the total order of k_select (value desc,
// index asc), computed by each candidate in parallel instead of rounds of
// warp arg-max: an expert's rank in its group gives the group's top-2 (or
// maximum), a group's rank among the groups decides whether it is kept, an
// expert's rank in its warp makes the warp's top-K candidates, and a
// candidate's rank among all candidates its place in the token's list.  The
// order is strict, so every rank is unique and the result is k_select's.
constexpr int kMaxSelWarps = 32;  // E <= 1024
constexpr int64_t kBlockSelectMaxN = 1024;  // batches up to this size: a block per token
__global__ void __launch_bounds__(1024) k_select_block(
    const float* __restrict__ logits, const double* __restrict__ part, int splits, int64_t N,
    int E, const float* __restrict__ bias, int G, int TG, int K, int norm, float route_scale,
    int score_func, int group_mode, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
    DeviceStatus* st) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_s[1024];
  __shared__ float s_c[1024];
  __shared__ double s_x[1024];
  __shared__ float cand_v[kMaxSelWarps * 16];
  __shared__ int cand_i[kMaxSelWarps * 16];
  __shared__ float s_red[kMaxSelWarps];
  __shared__ float s_g1[32], s_g2[32], s_gs[32];
  __shared__ unsigned s_kept;
  __shared__ double s_sum;
  __shared__ int sel_i[16];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int nw = blockDim.x >> 5;
  const int64_t t = blockIdx.x;
  const bool live = e < E;
  float L = 0.f;
  if (live) {
    if (part) {
      // all partial loads in flight before the sums (summed in split order)
      const double* p = part + t * E + e;
      const int64_t zs = N * (int64_t)E;
      double a = 0.0;
      for (int z0 = 0; z0 < splits; z0 += 16) {
        double v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = z0 + j < splits ? p[(int64_t)(z0 + j) * zs] : 0.0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (z0 + j < splits) a += v[j];
      }
      L = (float)a;
    } else {
      L = logits[t * E + e];
    }
  }
  float sv = 0.f;
  if (score_func == MOE_SCORE_SOFTMAX) {
    // block maximum, exp(L - max) in double, the normaliser summed by one
    // thread in expert order, quotient rounded once (as k_select)
    float mx = live ? L : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) s_red[warp] = mx;
    __syncthreads();
    mx = s_red[0];
    for (int i = 1; i < nw; ++i) mx = fmaxf(mx, s_red[i]);
    if (live) s_x[e] = exp((double)L - (double)mx);
    __syncthreads();
    if (e == 0) {
      double sum = 0.0;
      for (int i = 0; i < E; ++i) sum += s_x[i];
      s_sum = sum;
    }
    __syncthreads();
    if (live) sv = (float)(s_x[e] / s_sum);
  } else if (live) {
    sv = (float)__drcp_rn(1.0 + exp(-(double)L));
  }
  const int my = live ? e : 0x7fffffff;
  float cv = live ? (bias ? __fadd_rn(sv, bias[e]) : sv) : kNegInf;
  if (live) {
    s_s[e] = sv;
    s_c[e] = cv;
  }
  if (e < 32) s_g2[e] = kNegInf;  // a group of one expert has no second
  __syncthreads();
  if (G > 1) {
    // the expert's rank in its group: rank 0 is the group's maximum, rank 1
    // its second (equal values count twice, as in a top-2)
    const int gsz = E / G;
    if (live) {
      const int g = e / gsz, b0 = g * gsz;
      int r = 0;
      for (int j = 0; j < gsz; ++j) r += ranks_before(s_c[b0 + j], b0 + j, cv, e) ? 1 : 0;
      if (r == 0) s_g1[g] = cv;
      if (r == 1) s_g2[g] = cv;
    }
    __syncthreads();
    if (e < G) s_gs[e] = group_mode == MOE_GROUP_MAX ? s_g1[e] : __fadd_rn(s_g1[e], s_g2[e]);
    __syncthreads();
    // a group is kept when fewer than TG groups rank before it
    if (warp == 0) {
      bool kept = false;
      if (lane < G) {
        const float gs = s_gs[lane];
        int r = 0;
        for (int h = 0; h < G; ++h) r += ranks_before(s_gs[h], h, gs, lane) ? 1 : 0;
        kept = r < TG;
      }
      const unsigned m = __ballot_sync(0xffffffffu, kept);
      if (lane == 0) s_kept = m;
    }
    __syncthreads();
    if (live && !((s_kept >> (e / gsz)) & 1u)) cv = kNegInf;
    if (live) s_c[e] = cv;
    __syncthreads();
  }
  // the warp's top-K: its experts of rank < K in the warp (live experts only;
  // a warp with fewer than K live experts offers them all)
  const int w0 = warp * 32;
  const int nlive_w = E - w0 < 32 ? (E - w0 > 0 ? E - w0 : 0) : 32;
  const int kw = nlive_w < K ? nlive_w : K;
  if (live) {
    int r = 0;
    for (int j = 0; j < nlive_w; ++j) r += ranks_before(s_c[w0 + j], w0 + j, cv, my) ? 1 : 0;
    if (r < kw) {
      cand_v[warp * K + r] = cv;
      cand_i[warp * K + r] = e;
    }
  }
  __syncthreads();
  // each candidate's rank among all candidates: rank k is the token's k-th
  // expert.  A warp's candidates are stored best first, so the ones ranking
  // before a given candidate are a prefix: its length by binary search.
  const int nc = nw * K;
  if (e < nc) {
    const int cw = e / K, own = e - cw * K;
    const int cw0 = cw * 32;
    const int cnl = E - cw0 < 32 ? (E - cw0 > 0 ? E - cw0 : 0) : 32;
    if (own < (cnl < K ? cnl : K)) {
      const float v = cand_v[e];
      const int i = cand_i[e];
      int r = own;
      for (int w = 0; w < nw; ++w) {
        if (w == cw) continue;
        const int wl = E - w * 32 < 32 ? (E - w * 32 > 0 ? E - w * 32 : 0) : 32;
        int lo = 0, hi = wl < K ? wl : K;  // first entry not ranking before (v, i)
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (ranks_before(cand_v[w * K + mid], cand_i[w * K + mid], v, i)) lo = mid + 1;
          else hi = mid;
        }
        r += lo;
      }
      if (r < K) sel_i[r] = i;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int my_e = lane < K ? sel_i[lane] : 0;
    if (lane < K && (my_e < 0 || my_e >= E)) record_error(st, MOE_ERR_DEVICE_BOUNDS, 2);
    float wk = (lane < K && my_e >= 0 && my_e < E) ? s_s[my_e] : 0.f;
    if (K > 1 && norm) {
      float den = __shfl_sync(0xffffffffu, wk, 0);
      for (int k = 1; k < K; ++k) den = __fadd_rn(den, __shfl_sync(0xffffffffu, wk, k));
      den = __fadd_rn(den, 1e-20f);
      wk = __fdiv_rn(wk, den);
    }
    wk = __fmul_rn(wk, route_scale);
    if (lane < K) {
      idx_out[t * K + lane] = my_e;
      w_out[t * K + lane] = wk;
    }
  }
}

}  // namespace

int route_splits(int64_t N, int E, int d_r) {
  int64_t tiles = ((E + GE - 1) / GE) * ((N + GT - 1) / GT);
  if (tiles < 1) tiles = 1;
  const int nk = d_r / GK > 0 ? d_r / GK : 1;
  int64_t want = (296 + tiles - 1) / tiles;  // about two CTAs per SM
  int64_t maxs = nk / 4 > 0 ? nk / 4 : 1;    // at least 4 chunks per split
  if (want > maxs) want = maxs;
  if (want > 32) want = 32;
  if (want < 1) want = 1;
  const int cps = (int)((nk + want - 1) / want);
  return (nk + cps - 1) / cps;
}

// Router scratch: [logits N x E fp32][partials splits x N x E double, if split]
size_t route_partial_bytes(int64_t N, int E, int d_r) {
  if (gate_i8_applies(N, E, d_r)) return gate_i8_scratch_bytes(N, E, d_r);
  const int splits = route_splits(N, E, d_r);
  const size_t ne = (size_t)N * (size_t)E;
  return align_up(sizeof(float) * ne, 256) +
         (splits > 1 ? align_up(sizeof(double) * (size_t)splits * ne, 256) : 0);
}

float* route_logits_of(void* scratch) { return static_cast<float*>(scratch); }

static double* route_part_of(void* scratch, int64_t N, int E) {
  return reinterpret_cast<double*>(static_cast<uint8_t*>(scratch) +
                                   align_up(sizeof(float) * (size_t)N * (size_t)E, 256));
}

const double* route_fused_partials(void* scratch, int64_t N, int E, int d_r, int* splits) {
  *splits = 1;
  if (gate_i8_applies(N, E, d_r)) return nullptr;
  const int sp = route_splits(N, E, d_r);
  if (sp <= 1) return nullptr;
  *splits = sp;
  return route_part_of(scratch, N, E);
}

cudaError_t launch_gate(const __nv_bfloat16* x, int64_t N, int d_r, const float* W, int E,
                        void* scratch, DeviceStatus* st, cudaStream_t s, bool reduce) {
  if (gate_i8_applies(N, E, d_r)) return launch_gate_i8(x, N, d_r, W, E, scratch, st, s);
  const int splits = route_splits(N, E, d_r);
  const int nk = d_r / GK;
  const int cps = (nk + splits - 1) / splits;
  float* logits = route_logits_of(scratch);
  double* part = route_part_of(scratch, N, E);
  dim3 grid((E + GE - 1) / GE, (unsigned)((N + GT - 1) / GT), splits);
  cudaError_t e = launch_pdl(k_gate_partial, grid, dim3(256), 0, s, x, N, d_r, W, E, cps, splits,
                             logits, part);
  if (e != cudaSuccess) return e;
  if (splits > 1 && reduce) {
    const int64_t ne = N * (int64_t)E;
    int64_t blocks = (ne + 255) / 256;
    const int64_t cap = (int64_t)dev_info()->sm_count * 16;
    if (blocks > cap) blocks = cap;
    e = launch_pdl(k_reduce_partials, dim3((unsigned)blocks), dim3(256), 0, s,
                   (const double*)part, splits, ne, logits);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const float* logits, int64_t N, const float* bias,
                          const moe_route_cfg& cfg, int32_t* idx, float* w, DeviceStatus* st,
                          cudaStream_t s, const double* part, int splits) {
  const int E = cfg.num_experts;
  if (part || N <= kBlockSelectMaxN) {
    const int threads = (E + 31) / 32 * 32;
    return launch_pdl(k_select_block, dim3((unsigned)N), dim3(threads), 0, s, logits, part,
                      splits, N, E, bias, cfg.n_group, cfg.topk_group, cfg.top_k,
                      cfg.norm_topk_prob, cfg.route_scale, cfg.score_func, cfg.group_score, idx,
                      w, st);
  }
  const bool softmax = cfg.score_func == MOE_SCORE_SOFTMAX;
  const size_t smem = sizeof(float) * 2 * E * kSelWarps + (softmax ? sizeof(double) * E * kSelWarps : 0);
  if (softmax && smem > 48 * 1024) {
    static std::once_flag once[kMaxDevices];
    static cudaError_t set_up[kMaxDevices];
    const cudaError_t e0 = once_per_device(once, set_up, [](int) {
      return cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  64 * 1024);
    });
    if (e0 != cudaSuccess) return e0;
  }
  int64_t blocks = (N + kSelWarps - 1) / kSelWarps;
  const int64_t cap = (int64_t)dev_info()->sm_count * 16;
  if (blocks > cap) blocks = cap;
  const cudaError_t e = launch_pdl(
      k_select, dim3((unsigned)blocks), dim3(32 * kSelWarps), smem, s, logits, N, E, bias,
      cfg.n_group, cfg.topk_group, cfg.top_k, cfg.norm_topk_prob, cfg.route_scale,
      cfg.score_func, cfg.group_score, idx, w, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
