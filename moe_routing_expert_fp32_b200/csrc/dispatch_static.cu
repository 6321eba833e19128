// dispatch_static.cu -- moe_dispatch for callers that cannot allocate device
// memory.
//
// Some callers have no way to obtain a device buffer of their own: a plugin
// that a host framework hands only its input and output tensors, a serving
// loop whose device memory is fully reserved up front by another allocator,
// or a latency-critical path where cudaMalloc's implicit synchronisation is
// not acceptable.  moe_dispatch_static computes exactly what moe_dispatch
// computes, with the same kernels, but takes no workspace: its scratch (the
// per-chunk expert counts of the stable sort) lives in the fixed-size device
// array below.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library holds MOE_DISPATCH_STATIC_SCRATCH_BYTES of it until the process
// exits.  In host code `g_dispatch_scratch` names a host-side stand-in, not a
// device address; the device address is looked up with cudaGetSymbolAddress
// once per device context (the first call made with that context current,
// normally the device's primary context) and passed to the kernels.
#include <cuda.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __align__(256) uint8_t g_dispatch_scratch[MOE_DISPATCH_STATIC_SCRATCH_BYTES];

// The driver context current on this thread, or nullptr (none current, or
// the driver entry point is unavailable).  The symbol's device address is
// valid only in the context it was looked up in, so the cache below is keyed
// by context rather than by device number: a caller that switches between a
// device's primary context and a context of its own gets each one's address.
void* current_context() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  static const CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_dispatch_scratch in the current context.  The lookup
// runs on the first call made with a context current and is cached only when
// it succeeds; a failed lookup (for instance a first call made during stream
// capture) clears its error and returns nullptr, so a later call can retry.
uint8_t* static_scratch_ptr() {
  struct Entry {
    void* ctx;
    uint8_t* ptr;
  };
  static std::mutex mu;
  static Entry cache[kMaxDevices];
  static int n_cached = 0;
  std::lock_guard<std::mutex> lock(mu);
  void* ctx = current_context();
  if (ctx)
    for (int i = 0; i < n_cached; ++i)
      if (cache[i].ctx == ctx) return cache[i].ptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();  // leave no pending error behind
    return nullptr;
  }
  ctx = current_context();  // the lookup makes the primary context current if none was
  if (ctx && n_cached < kMaxDevices) cache[n_cached++] = Entry{ctx, static_cast<uint8_t*>(p)};
  return static_cast<uint8_t*>(p);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_dispatch_static(const int32_t* topk_idx, int64_t N, int K, int E,
                                   const moe_bf16* x_e, int d_e, int32_t* counts,
                                   int32_t* offsets, int32_t* perm, int32_t* pos, moe_bf16* xs,
                                   void* stream) {
  if (N < 0 || K < 1 || E < 1 || d_e <= 0) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || K > 16) return MOE_ERR_UNSUPPORTED;
  if (d_e % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (N * (int64_t)K > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  // xs == NULL: the sort only, x_e is not read (as in moe_dispatch)
  if (N > 0 && (!topk_idx || !perm || !pos || (xs && !x_e))) return MOE_ERR_INVALID_ARG;
  if (N > 0 && xs && ((reinterpret_cast<uintptr_t>(x_e) & 15u) ||
                      (reinterpret_cast<uintptr_t>(xs) & 15u)))
    return MOE_ERR_ALIGNMENT;
  // The per-chunk counts of this call must fit in the fixed array.
  if (dispatch_scratch_bytes(N * K, E) > MOE_DISPATCH_STATIC_SCRATCH_BYTES)
    return MOE_ERR_UNSUPPORTED;
  const DevInfo* di = dev_info();
  if (!di || di->cc_major != 10) return MOE_ERR_NO_DEVICE;
  uint8_t* scratch = static_scratch_ptr();
  if (!scratch) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // Nothing in the array has to start at zero: the histogram pass writes every
  // count it reads back.  No status word: an out-of-range expert index is
  // skipped exactly as in moe_dispatch, but it is not reported.
  return launch_dispatch(topk_idx, N, K, E, reinterpret_cast<const __nv_bfloat16*>(x_e), d_e,
                         counts, offsets, perm, pos, reinterpret_cast<__nv_bfloat16*>(xs),
                         reinterpret_cast<int32_t*>(scratch), nullptr, s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
