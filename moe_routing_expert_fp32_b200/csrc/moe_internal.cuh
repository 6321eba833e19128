// moe_internal.cuh -- definitions shared by the kernels of libmoe (not part of
// the public ABI).  sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include "moe.h"

namespace moe {

// ------------------------------------------------------------ status word
// The first 256 bytes of every workspace; kernels record the first error.
struct DeviceStatus {
  int code;       // 0 or a negative moe_status
  int detail;     // kernel-specific: where it happened
};
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void record_error(DeviceStatus* st, int code, int detail) {
  if (st && atomicCAS(&st->code, 0, code) == 0) st->detail = detail;
}

// Bounded waits: ~2^28 polls is seconds on any healthy GPU; a wait that runs
// out records MOE_ERR_DEVICE_TIMEOUT and gives up instead of hanging.
constexpr uint32_t kSpinLimit = 1u << 28;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------- per-device set-up
// Runs init() once per device, however many host threads call at once, and
// returns its result to every caller (kernel attributes, launch grids).
constexpr int kMaxDevices = 64;
template <typename F>
cudaError_t once_per_device(std::once_flag* flags, cudaError_t* results, F&& init) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  std::call_once(flags[dev], [&] { results[dev] = init(dev); });
  return results[dev];
}

// ------------------------------------------- programmatic dependent launch
// The short kernels of the layer are launched as programmatic dependents of
// the kernel before them on the stream (launch_pdl): their CTAs may be
// scheduled while that kernel is still running, which hides the launch
// latency between back-to-back small kernels.  Each such kernel starts with
// pdl_wait() (no read or write of memory the predecessor touches before it),
// then pdl_trigger() so that its own dependent can be scheduled in turn.
// Launched without the attribute, both instructions return at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Every kernel launch of the library is counted (moe_launch_count): the
// launch sites pass their result through counted(), which adds n launches
// when the launch was accepted.
void count_launches(int n);
inline cudaError_t counted(cudaError_t e, int n = 1) {
  if (e == cudaSuccess) count_launches(n);
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted(cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...));
}

// --------------------------------------------------------- kernel launches
// (all enqueue on `stream`, no synchronisation)

// router.cu
int route_splits(int64_t N, int E, int d_r);
size_t route_partial_bytes(int64_t N, int E, int d_r);
// gate GEMM into the router scratch; the fp32 logits [N, E] are at its start.
// reduce = false leaves split-K partials unsummed (route_fused_partials says
// where they are; the selection sums them).
cudaError_t launch_gate(const __nv_bfloat16* x, int64_t N, int d_r, const float* W, int E,
                        void* scratch, DeviceStatus* st, cudaStream_t s, bool reduce = true);
// the gate GEMM's double partials [splits, N, E] when the fp32 path splits
// over d_r (*splits set), else nullptr (*splits = 1)
const double* route_fused_partials(void* scratch, int64_t N, int E, int d_r, int* splits);

// router_i8.cu: the same GEMM on the int8 tensor cores (exact digit products),
// used when the batch fills enough 128x96 tiles
bool gate_i8_applies(int64_t N, int E, int d_r);
size_t gate_i8_scratch_bytes(int64_t N, int E, int d_r);
cudaError_t launch_gate_i8(const __nv_bfloat16* x, int64_t N, int d_r, const float* W, int E,
                           void* scratch, DeviceStatus* st, cudaStream_t s);
float* route_logits_of(void* scratch);
// part (optional): take the logits as the sum of the gate GEMM's split
// partials instead of reading `logits`
cudaError_t launch_select(const float* logits, int64_t N, const float* bias,
                          const moe_route_cfg& cfg, int32_t* idx, float* w, DeviceStatus* st,
                          cudaStream_t s, const double* part = nullptr, int splits = 1);

// dispatch.cu
int dispatch_chunks(int64_t S);
size_t dispatch_scratch_bytes(int64_t S, int E);
// xs == nullptr: counts, offsets, perm and pos only (no gather)
cudaError_t launch_dispatch(const int32_t* idx, int64_t N, int K, int E, const __nv_bfloat16* x_e,
                            int d_e, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* pos, __nv_bfloat16* xs, int32_t* scratch, DeviceStatus* st,
                            cudaStream_t s);

// offsets [n+1] = exclusive prefix of counts [n] (n <= 1024)
cudaError_t launch_counts_offsets(const int32_t* counts, int n, int32_t* offsets,
                                  DeviceStatus* st, cudaStream_t s);

// expert_gemm.cu
size_t expert_scratch_bytes(int64_t S, int E, int F);
// Token rows gathered inside the w1/w3 kernel instead of read from xs: sorted
// row j is x_e[perm[j] / K], x_e [N, d_e].
struct GatherSrc {
  const __nv_bfloat16* x_e;
  const int32_t* perm;
  int64_t N;
  int K;
};
// whether the variant chosen for (S, E) gathers inside the kernel (the CTA-pair
// variant reads a gathered xs)
bool expert_gather_fusable(int64_t S, int E);
// residual (optional, [S, d_e] bf16): y = bf16(bf16(x.w2^T) + residual);
// gather (optional): xs is not read, the rows come from gather->x_e;
// n_weights: E segments (offsets[E+1]) use weights s % n_weights of the
// stacked w1/w3/w2 ([n_weights, ...]); 0 means n_weights = E;
// y_rows (optional, [S]): sorted row j of the output is stored at row
// y_rows[j] of y (the slot-order scatter; not with a residual)
int expert_ffn_run(const __nv_bfloat16* xs, const int32_t* offsets, int E, int64_t S, int d_e,
                   int F, const __nv_bfloat16* w1, const __nv_bfloat16* w3,
                   const __nv_bfloat16* w2, const moe_act_cfg& act, __nv_bfloat16* y,
                   void* scratch, DeviceStatus* st, cudaStream_t s, cudaEvent_t after_gate_up,
                   const __nv_bfloat16* residual = nullptr, const GatherSrc* gather = nullptr,
                   int n_weights = 0, const int32_t* y_rows = nullptr);
// Dense layers on the same kernels (one expert, every row): `tiles` is 8 int32
// of device memory written by launch_dense_tiles(M) before use.
constexpr size_t kDenseTilesBytes = 256;
cudaError_t launch_dense_tiles(int64_t M, int32_t* tiles, cudaStream_t s);
// fp32 split-K partials a dense layer of M rows needs (0: it runs unsplit);
// gate_up: the w1/w3 GEMM of an MLP of hidden width Nout
size_t dense_part_bytes(int64_t M, int K, int Nout, bool gate_up);
// y [M, Nout] = bf16(x [M, K] . W [Nout, K]^T) (+ residual [M, Nout]).
// pdl_ok: the kernel may start as a programmatic dependent of the preceding
// kernel; allowed only if `tiles` was written before that kernel started.
// part: dense_part_bytes(M, K, Nout, false) bytes of scratch, or nullptr
// (no split).
int linear_run(const __nv_bfloat16* x, int64_t M, int K, const __nv_bfloat16* W, int Nout,
               const __nv_bfloat16* residual, __nv_bfloat16* y, const int32_t* tiles,
               DeviceStatus* st, cudaStream_t s, bool pdl_ok, float* part);
// the gated MLP of one expert on every row of x [M, d]; h: [M, F] bf16 scratch;
// part: max(dense_part_bytes(M, d, F, true), dense_part_bytes(M, F, d, false))
// bytes, or nullptr.  Its down kernel is a programmatic dependent of the
// kernel before it.
int shared_ffn_run(const __nv_bfloat16* x, int64_t M, int d, int F, const __nv_bfloat16* w1,
                   const __nv_bfloat16* w3, const __nv_bfloat16* w2, const moe_act_cfg& act,
                   const __nv_bfloat16* residual, __nv_bfloat16* y, __nv_bfloat16* h,
                   const int32_t* tiles, DeviceStatus* st, cudaStream_t s, float* part);

// combine.cu
// residual (optional, [N, d_e]): out = bf16(bf16(sum) + residual);
// pos == nullptr: y is in slot order (token t's K rows at t*K .. t*K+K-1)
cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* pos, const float* w, int64_t N,
                           int K, int d_e, int64_t S, __nv_bfloat16* out, DeviceStatus* st,
                           cudaStream_t s, const __nv_bfloat16* residual = nullptr);
// combine followed by the RMSNorm of each combined row (one warp per token)
cudaError_t launch_combine_rms_norm(const __nv_bfloat16* y, const int32_t* pos, const float* w,
                                    int64_t N, int K, int d_e, int64_t S,
                                    const __nv_bfloat16* norm_w, float eps,
                                    __nv_bfloat16* out, DeviceStatus* st, cudaStream_t s);
// out [N, d] = RMSNorm(x) with a bf16 weight
cudaError_t launch_rms_norm(const __nv_bfloat16* x, int64_t N, int d, const __nv_bfloat16* w,
                            float eps, __nv_bfloat16* out, cudaStream_t s);

// ep_rows.cu: the expert-parallel exchange over peer memory (moe_ep_dispatch_rows,
// moe_ep_combine_rows).  Passed by value as a __grid_constant__ kernel argument.
struct PeerTable {
  int P;        // ranks
  int E_local;  // experts per rank
  __nv_bfloat16* rows[MOE_MAX_PEERS];
  int64_t first[MOE_MAX_PEERS];
  int64_t cap[MOE_MAX_PEERS];
};
cudaError_t launch_ep_dispatch_rows(const __nv_bfloat16* x, int64_t N, int K, int d,
                                    const int32_t* pos, const int32_t* offsets, int64_t S,
                                    const PeerTable& pt, DeviceStatus* st, cudaStream_t s);
cudaError_t launch_ep_combine_rows(const PeerTable& pt, const int32_t* pos,
                                   const int32_t* offsets, int64_t S, const float* w, int64_t N,
                                   int K, int d, __nv_bfloat16* out, DeviceStatus* st,
                                   cudaStream_t s);

// device properties, read once per device
struct DevInfo {
  int sm_count;
  int cc_major;
  int cc_minor;
  size_t smem_optin;
};
const DevInfo* dev_info();

}  // namespace moe
