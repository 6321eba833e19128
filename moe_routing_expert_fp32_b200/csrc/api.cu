// api.cu -- the C ABI of libmoe: argument validation, workspace layout, launch
// sequencing.  Nothing here computes the layer; every step runs in the
// kernels of router.cu, dispatch.cu, expert_gemm.cu and combine.cu.
#include <math.h>

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

const DevInfo* dev_info() {
  static std::mutex mu;
  static DevInfo info[64];
  static bool have[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DevInfo d{};
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return nullptr;
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.smem_optin = (size_t)optin;
    info[dev] = d;
    have[dev] = true;
  }
  return &info[dev];
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around the host-side enqueue of one stage ("moe.route",
// "moe.dispatch", ...): a profiler that records NVTX (Nsight Systems) shows
// each stage's kernels under its name; without one the calls cost nothing.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

int check_device() {
  const DevInfo* d = dev_info();
  if (!d || d->cc_major != 10) return MOE_ERR_NO_DEVICE;
  return MOE_OK;
}

int check_route_cfg(const moe_route_cfg* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  const int E = c->num_experts, G = c->n_group, TG = c->topk_group, K = c->top_k;
  if (E < 1 || G < 1 || TG < 1 || K < 1) return MOE_ERR_INVALID_ARG;
  if (E % G != 0 || TG > G) return MOE_ERR_INVALID_ARG;
  if (G > 1 && E / G < 2) return MOE_ERR_INVALID_ARG;
  if ((int64_t)K > (int64_t)TG * (E / G)) return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->route_scale)) return MOE_ERR_INVALID_ARG;
  if (c->score_func != MOE_SCORE_SIGMOID && c->score_func != MOE_SCORE_SOFTMAX)
    return MOE_ERR_INVALID_ARG;
  if (c->group_score != MOE_GROUP_TOP2_SUM && c->group_score != MOE_GROUP_MAX)
    return MOE_ERR_INVALID_ARG;
  if (E > 1024 || G > 32 || K > 16) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int check_act(const moe_act_cfg* a) {
  if (!a) return MOE_ERR_INVALID_ARG;
  if (a->kind != MOE_ACT_SILU && a->kind != MOE_ACT_SITU) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_WORKSPACE;
  if (have < need) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Resets the status word of a workspace at the start of a call.
int reset_status(void* ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

DeviceStatus* status_of(void* ws) { return static_cast<DeviceStatus*>(ws); }
uint8_t* body_of(void* ws) { return static_cast<uint8_t*>(ws) + kStatusBytes; }

size_t route_body(int64_t N, int d_r, int E) { return route_partial_bytes(N, E, d_r); }

int route_impl(const __nv_bfloat16* x, int64_t N, int d_r, const float* W, const float* bias,
               const moe_route_cfg& cfg, int32_t* idx, float* w, uint8_t* scratch,
               DeviceStatus* st, cudaStream_t s) {
  const int E = cfg.num_experts;
  // split-K partials of the gate GEMM (decode batches) are summed by the
  // selection kernel itself, so no reduce kernel runs between them
  int splits = 1;
  const double* part = route_fused_partials(scratch, N, E, d_r, &splits);
  if (launch_gate(x, N, d_r, W, E, scratch, st, s, part == nullptr) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_select(route_logits_of(scratch), N, bias, cfg, idx, w, st, s, part, splits) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "shape outside the supported limits";
    case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
    case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
    case MOE_ERR_DEVICE_BOUNDS: return "a kernel met an index out of range";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown moe_status";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_get_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus h{};
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return h.code;
}

// ------------------------------------------------------------------ router
size_t moe_route_workspace_size(int64_t N, int d_r, const moe_route_cfg* cfg) {
  if (!cfg || N < 0 || d_r <= 0 || cfg->num_experts <= 0) return 0;
  return kStatusBytes + route_body(N, d_r, cfg->num_experts);
}

int moe_route(const moe_bf16* x, int64_t N, int d_r, const float* W, const float* bias,
              const moe_route_cfg* cfg, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, void* stream) {
  int rc = check_route_cfg(cfg);
  if (rc) return rc;
  if (N < 0 || d_r <= 0) return MOE_ERR_INVALID_ARG;
  if (d_r % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (N > 0 && (!x || !W || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!aligned16(x) || !aligned16(W))) return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_route_workspace_size(N, d_r, cfg)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  return route_impl(reinterpret_cast<const __nv_bfloat16*>(x), N, d_r, W, bias, *cfg, topk_idx,
                    topk_w, body_of(ws), status_of(ws), s);
}

size_t moe_gate_logits_workspace_size(int64_t N, int d_r, int E) {
  if (N < 0 || d_r <= 0 || E <= 0) return 0;
  return kStatusBytes + route_body(N, d_r, E);
}

int moe_gate_logits(const moe_bf16* x, int64_t N, int d_r, const float* W, int E, float* logits,
                    void* ws, size_t ws_bytes, void* stream) {
  if (N < 0 || d_r <= 0 || E < 1) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED;
  if (d_r % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (N > 0 && (!x || !W || !logits)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!aligned16(x) || !aligned16(W))) return MOE_ERR_ALIGNMENT;
  int rc;
  if ((rc = check_ws(ws, ws_bytes, moe_gate_logits_workspace_size(N, d_r, E)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  uint8_t* scratch = body_of(ws);
  if (launch_gate(reinterpret_cast<const __nv_bfloat16*>(x), N, d_r, W, E, scratch, status_of(ws),
                  s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaMemcpyAsync(logits, route_logits_of(scratch), sizeof(float) * (size_t)N * E,
                         cudaMemcpyDeviceToDevice, s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int moe_route_from_logits(const float* logits, int64_t N, const float* bias,
                          const moe_route_cfg* cfg, int32_t* topk_idx, float* topk_w, void* ws,
                          size_t ws_bytes, void* stream) {
  int rc = check_route_cfg(cfg);
  if (rc) return rc;
  if (N < 0) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
  if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  return launch_select(logits, N, bias, *cfg, topk_idx, topk_w, status_of(ws), s) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------- dispatch
size_t moe_dispatch_workspace_size(int64_t N, int K, int E) {
  if (N < 0 || K <= 0 || E <= 0) return 0;
  return kStatusBytes + dispatch_scratch_bytes(N * K, E);
}

int moe_dispatch(const int32_t* topk_idx, int64_t N, int K, int E, const moe_bf16* x_e, int d_e,
                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos, moe_bf16* xs,
                 void* ws, size_t ws_bytes, void* stream) {
  if (N < 0 || K < 1 || E < 1 || d_e <= 0) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || K > 16) return MOE_ERR_UNSUPPORTED;
  if (d_e % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (N * (int64_t)K > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  // xs == NULL: the sort only, x_e is not read
  if (N > 0 && (!topk_idx || !perm || !pos || (xs && !x_e))) return MOE_ERR_INVALID_ARG;
  if (N > 0 && xs && (!aligned16(x_e) || !aligned16(xs))) return MOE_ERR_ALIGNMENT;
  int rc;
  if ((rc = check_ws(ws, ws_bytes, moe_dispatch_workspace_size(N, K, E)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return launch_dispatch(topk_idx, N, K, E, reinterpret_cast<const __nv_bfloat16*>(x_e), d_e,
                         counts, offsets, perm, pos, reinterpret_cast<__nv_bfloat16*>(xs),
                         reinterpret_cast<int32_t*>(body_of(ws)), status_of(ws), s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// ------------------------------------------------------------- expert MLP
size_t moe_expert_ffn_workspace_size(int64_t S, int d_e, int E, int F) {
  if (S < 0 || d_e <= 0 || E <= 0 || F <= 0) return 0;
  return kStatusBytes + expert_scratch_bytes(S, E, F);
}

static int check_expert_shape(int64_t S, int d_e, int E, int F) {
  if (S < 0 || d_e <= 0 || E < 1 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || d_e % 128 != 0 || F % 128 != 0 || S > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int moe_expert_ffn(const moe_bf16* xs, const int32_t* offsets, int E, int64_t S, int d_e, int F,
                   const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                   const moe_act_cfg* act, moe_bf16* y, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_expert_shape(S, d_e, E, F);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (!offsets || !w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!xs || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_ALIGNMENT;
  if (S > 0 && (!aligned16(xs) || !aligned16(y))) return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_expert_ffn_workspace_size(S, d_e, E, F)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (S == 0) return MOE_OK;
  return expert_ffn_run(reinterpret_cast<const __nv_bfloat16*>(xs), offsets, E, S, d_e, F,
                        reinterpret_cast<const __nv_bfloat16*>(w1),
                        reinterpret_cast<const __nv_bfloat16*>(w3),
                        reinterpret_cast<const __nv_bfloat16*>(w2), *act,
                        reinterpret_cast<__nv_bfloat16*>(y), body_of(ws), status_of(ws), s,
                        nullptr);
}

// The expert MLP writing each output row to its slot (the scatter inside the
// w2 kernel's epilogue): y_slots[perm[j]] = the MLP of sorted row j.
int moe_expert_ffn_to_slots(const moe_bf16* xs, const int32_t* offsets, const int32_t* perm,
                            int E, int64_t S, int d_e, int F, const moe_bf16* w1,
                            const moe_bf16* w3, const moe_bf16* w2, const moe_act_cfg* act,
                            moe_bf16* y_slots, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_expert_shape(S, d_e, E, F);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (!offsets || !w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!xs || !perm || !y_slots)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_ALIGNMENT;
  if (S > 0 && (!aligned16(xs) || !aligned16(y_slots))) return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_expert_ffn_workspace_size(S, d_e, E, F)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (S == 0) return MOE_OK;
  return expert_ffn_run(reinterpret_cast<const __nv_bfloat16*>(xs), offsets, E, S, d_e, F,
                        reinterpret_cast<const __nv_bfloat16*>(w1),
                        reinterpret_cast<const __nv_bfloat16*>(w3),
                        reinterpret_cast<const __nv_bfloat16*>(w2), *act,
                        reinterpret_cast<__nv_bfloat16*>(y_slots), body_of(ws), status_of(ws), s,
                        nullptr, nullptr, nullptr, 0, perm);
}

// The expert MLP reading its token rows straight from x_e through perm (the
// gather inside the w1/w3 kernel): no S x d_e copy of the tokens.
int moe_expert_ffn_gathered(const moe_bf16* x_e, int64_t N, int K, const int32_t* perm,
                            const int32_t* offsets, int E, int d_e, int F, const moe_bf16* w1,
                            const moe_bf16* w3, const moe_bf16* w2, const moe_act_cfg* act,
                            moe_bf16* y, void* ws, size_t ws_bytes, void* stream) {
  if (N < 0 || K < 1) return MOE_ERR_INVALID_ARG;
  const int64_t S = N * (int64_t)K;
  int rc = check_expert_shape(S, d_e, E, F);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (!expert_gather_fusable(S, E)) return MOE_ERR_UNSUPPORTED;
  if (!offsets || !w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!x_e || !perm || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_ALIGNMENT;
  if (S > 0 && (!aligned16(x_e) || !aligned16(y))) return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_expert_ffn_workspace_size(S, d_e, E, F)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (S == 0) return MOE_OK;
  const GatherSrc g{reinterpret_cast<const __nv_bfloat16*>(x_e), perm, N, K};
  return expert_ffn_run(nullptr, offsets, E, S, d_e, F, reinterpret_cast<const __nv_bfloat16*>(w1),
                        reinterpret_cast<const __nv_bfloat16*>(w3),
                        reinterpret_cast<const __nv_bfloat16*>(w2), *act,
                        reinterpret_cast<__nv_bfloat16*>(y), body_of(ws), status_of(ws), s,
                        nullptr, nullptr, &g);
}

// ------------------------------------------------ expert parallel receive side
size_t moe_ep_expert_ffn_workspace_size(int64_t R, int d_e, int P, int E_local, int F) {
  if (R < 0 || d_e <= 0 || P < 1 || E_local < 1 || F <= 0) return 0;
  const int n = P * E_local;
  return kStatusBytes + align_up(sizeof(int32_t) * (size_t)(n + 1), 256) +
         expert_scratch_bytes(R, n, F);
}

int moe_ep_expert_ffn(const moe_bf16* xr, int64_t R, const int32_t* recv_counts, int P,
                      int E_local, int d_e, int F, const moe_bf16* w1, const moe_bf16* w3,
                      const moe_bf16* w2, const moe_act_cfg* act, moe_bf16* y, void* ws,
                      size_t ws_bytes, void* stream) {
  if (P < 1 || E_local < 1 || !recv_counts) return MOE_ERR_INVALID_ARG;
  if ((int64_t)P * E_local > 1024) return MOE_ERR_UNSUPPORTED;
  const int n = P * E_local;
  int rc = check_expert_shape(R, d_e, n, F);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (!w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (R > 0 && (!xr || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_ALIGNMENT;
  if (R > 0 && (!aligned16(xr) || !aligned16(y))) return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_ep_expert_ffn_workspace_size(R, d_e, P, E_local, F))))
    return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (R == 0) return MOE_OK;
  uint8_t* body = body_of(ws);
  int32_t* offsets = reinterpret_cast<int32_t*>(body);
  uint8_t* scratch = body + align_up(sizeof(int32_t) * (size_t)(n + 1), 256);
  if (launch_counts_offsets(recv_counts, n, offsets, status_of(ws), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return expert_ffn_run(reinterpret_cast<const __nv_bfloat16*>(xr), offsets, n, R, d_e, F,
                        reinterpret_cast<const __nv_bfloat16*>(w1),
                        reinterpret_cast<const __nv_bfloat16*>(w3),
                        reinterpret_cast<const __nv_bfloat16*>(w2), *act,
                        reinterpret_cast<__nv_bfloat16*>(y), scratch, status_of(ws), s, nullptr,
                        nullptr, nullptr, E_local);
}

// ----------------------------------------------------------------- combine
size_t moe_combine_workspace_size(void) { return kStatusBytes; }

int moe_combine(const moe_bf16* y, const int32_t* pos, const float* topk_w, int64_t N, int K,
                int d_e, moe_bf16* out, void* ws, size_t ws_bytes, void* stream) {
  if (N < 0 || K < 1 || d_e <= 0) return MOE_ERR_INVALID_ARG;
  if (K > 16) return MOE_ERR_UNSUPPORTED;
  if (d_e % 8 != 0) return MOE_ERR_UNSUPPORTED;
  // pos == NULL: y is in slot order (moe_expert_ffn_to_slots)
  if (N > 0 && (!y || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!aligned16(y) || !aligned16(out))) return MOE_ERR_ALIGNMENT;
  int rc;
  if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  return launch_combine(reinterpret_cast<const __nv_bfloat16*>(y), pos, topk_w, N, K, d_e,
                        N * K, reinterpret_cast<__nv_bfloat16*>(out), status_of(ws), s) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// ------------------------------------- expert parallelism over peer memory
namespace {
int peer_table(const moe_peer_rows* peers, int E, PeerTable* pt) {
  if (!peers) return MOE_ERR_INVALID_ARG;
  const int P = peers->num_ranks;
  if (P < 1 || P > MOE_MAX_PEERS) return MOE_ERR_UNSUPPORTED;
  if (E % P != 0) return MOE_ERR_INVALID_ARG;
  pt->P = P;
  pt->E_local = E / P;
  for (int q = 0; q < MOE_MAX_PEERS; ++q) {
    pt->rows[q] = nullptr;
    pt->first[q] = 0;
    pt->cap[q] = 0;
    if (q >= P) continue;
    if (peers->first_row[q] < 0 || peers->capacity[q] < 0) return MOE_ERR_INVALID_ARG;
    if (peers->capacity[q] > 0 && !peers->rows[q]) return MOE_ERR_INVALID_ARG;
    if (peers->rows[q] && !aligned16(peers->rows[q])) return MOE_ERR_ALIGNMENT;
    pt->rows[q] = static_cast<__nv_bfloat16*>(peers->rows[q]);
    pt->first[q] = peers->first_row[q];
    pt->cap[q] = peers->capacity[q];
  }
  return MOE_OK;
}

int check_ep_rows(int64_t N, int K, int d_e, int E, const int32_t* pos, const int32_t* offsets) {
  if (N < 0 || K < 1 || E < 1 || d_e <= 0) return MOE_ERR_INVALID_ARG;
  if (K > 16 || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (d_e % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (N * (int64_t)K > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (N > 0 && (!pos || !offsets)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace

int moe_ep_dispatch_rows(const moe_bf16* x_e, int64_t N, int K, int d_e, const int32_t* pos,
                         const int32_t* offsets, int E, const moe_peer_rows* peers, void* ws,
                         size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_ep_rows(N, K, d_e, E, pos, offsets))) return rc;
  if (N > 0 && !x_e) return MOE_ERR_INVALID_ARG;
  if (N > 0 && !aligned16(x_e)) return MOE_ERR_ALIGNMENT;
  PeerTable pt;
  if ((rc = peer_table(peers, E, &pt))) return rc;
  if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  return launch_ep_dispatch_rows(reinterpret_cast<const __nv_bfloat16*>(x_e), N, K, d_e, pos,
                                 offsets, N * K, pt, status_of(ws), s) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

int moe_ep_combine_rows(const moe_peer_rows* peers, const int32_t* pos, const int32_t* offsets,
                        int E, const float* topk_w, int64_t N, int K, int d_e, moe_bf16* out,
                        void* ws, size_t ws_bytes, void* stream) {
  int rc;
  if ((rc = check_ep_rows(N, K, d_e, E, pos, offsets))) return rc;
  if (N > 0 && (!topk_w || !out)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && !aligned16(out)) return MOE_ERR_ALIGNMENT;
  PeerTable pt;
  if ((rc = peer_table(peers, E, &pt))) return rc;
  if ((rc = check_ws(ws, ws_bytes, kStatusBytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  return launch_ep_combine_rows(pt, pos, offsets, N * K, topk_w, N, K, d_e,
                                reinterpret_cast<__nv_bfloat16*>(out), status_of(ws), s) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// ------------------------------------------------------------ whole layer
namespace {
// Whether moe_forward scatters y into slot order in the w2 epilogue (and
// combines contiguous rows) or keeps y sorted (and combines through pos).
constexpr bool kForwardSlotOrder = false;

struct ForwardLayout {
  size_t stage;                    // shared scratch of the stages
  size_t idx, w, counts, offsets, perm, pos, xs, y, total;
};

ForwardLayout forward_layout(int64_t N, int d_r, int d_e, int E, int K, int F) {
  ForwardLayout L{};
  const int64_t S = N * K;
  size_t stage = route_body(N, d_r, E);
  const size_t disp = dispatch_scratch_bytes(S, E);
  const size_t exp = expert_scratch_bytes(S, E, F);
  if (disp > stage) stage = disp;
  if (exp > stage) stage = exp;
  size_t o = kStatusBytes;
  L.stage = o; o += align_up(stage, 256);
  L.idx = o; o += align_up(sizeof(int32_t) * (size_t)S, 256);
  L.w = o; o += align_up(sizeof(float) * (size_t)S, 256);
  L.counts = o; o += align_up(sizeof(int32_t) * (size_t)E, 256);
  L.offsets = o; o += align_up(sizeof(int32_t) * (size_t)(E + 1), 256);
  L.perm = o; o += align_up(sizeof(int32_t) * (size_t)S, 256);
  L.pos = o; o += align_up(sizeof(int32_t) * (size_t)S, 256);
  L.xs = o; o += align_up(sizeof(__nv_bfloat16) * (size_t)S * (size_t)d_e, 256);
  L.y = o; o += align_up(sizeof(__nv_bfloat16) * (size_t)S * (size_t)d_e, 256);
  L.total = o;
  return L;
}
}  // namespace

size_t moe_workspace_size(int64_t N, int d_r, int d_e, const moe_route_cfg* cfg, int F) {
  if (!cfg || N < 0 || d_r <= 0 || d_e <= 0 || F <= 0 || cfg->num_experts <= 0 ||
      cfg->top_k <= 0)
    return 0;
  return forward_layout(N, d_r, d_e, cfg->num_experts, cfg->top_k, F).total;
}

int moe_forward(const moe_bf16* x_r, const moe_bf16* x_e, int64_t N, int d_r, int d_e,
                const float* W, const float* bias, const moe_route_cfg* cfg, const moe_bf16* w1,
                const moe_bf16* w3, const moe_bf16* w2, int F, const moe_act_cfg* act,
                moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out, void* ws,
                size_t ws_bytes, void* stream, const moe_stage_events* events) {
  int rc = check_route_cfg(cfg);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (N < 0 || d_r <= 0) return MOE_ERR_INVALID_ARG;
  if (!x_e) {
    if (d_e != d_r) return MOE_ERR_INVALID_ARG;
    x_e = x_r;
  }
  const int E = cfg->num_experts, K = cfg->top_k;
  if ((rc = check_expert_shape(N * (int64_t)K, d_e, E, F))) return rc;
  if (d_r % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (!W || !w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!x_r || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(w1) || !aligned16(w3) || !aligned16(w2))
    return MOE_ERR_ALIGNMENT;
  if (N > 0 && (!aligned16(x_r) || !aligned16(x_e) || !aligned16(out))) return MOE_ERR_ALIGNMENT;
  const ForwardLayout L = forward_layout(N, d_r, d_e, E, K, F);
  if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  DeviceStatus* st = status_of(ws);
  uint8_t* stage = base + L.stage;
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(base + L.idx);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + L.w);
  int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(base + L.perm);
  int32_t* pos = reinterpret_cast<int32_t*>(base + L.pos);
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(base + L.xs);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(base + L.y);
  auto rec = [&](void* ev) {
    return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev), s) == cudaSuccess : true;
  };
  const Range layer("moe.forward");
  {
    const Range r("moe.route");
    if ((rc = route_impl(reinterpret_cast<const __nv_bfloat16*>(x_r), N, d_r, W, bias, *cfg, idx,
                         w, stage, st, s)))
      return rc;
  }
  if (events && !rec(events->after_route)) return MOE_ERR_CUDA;
  {
    const Range r("moe.dispatch");
    if (launch_dispatch(idx, N, K, E, reinterpret_cast<const __nv_bfloat16*>(x_e), d_e, counts,
                        offsets, perm, pos, xs, reinterpret_cast<int32_t*>(stage), st,
                        s) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (events && !rec(events->after_dispatch)) return MOE_ERR_CUDA;
  // with kForwardSlotOrder the w2 epilogue writes y in slot order (row
  // perm[j] for sorted row j) and the combine reads each token's K rows
  // contiguously; otherwise y stays sorted and the combine reads it via pos
  {
    const Range r("moe.expert_ffn");
    if ((rc = expert_ffn_run(xs, offsets, E, N * K, d_e, F,
                             reinterpret_cast<const __nv_bfloat16*>(w1),
                             reinterpret_cast<const __nv_bfloat16*>(w3),
                             reinterpret_cast<const __nv_bfloat16*>(w2), *act, y, stage, st, s,
                             events ? static_cast<cudaEvent_t>(events->after_gate_up) : nullptr,
                             nullptr, nullptr, 0, kForwardSlotOrder ? perm : nullptr)))
      return rc;
  }
  if (events && !rec(events->after_down)) return MOE_ERR_CUDA;
  {
    const Range r("moe.combine");
    if (launch_combine(y, kForwardSlotOrder ? nullptr : pos, w, N, K, d_e, N * K,
                       reinterpret_cast<__nv_bfloat16*>(out), st, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (events && !rec(events->after_combine)) return MOE_ERR_CUDA;
  return MOE_OK;
}

// ------------------------------------------------------------ dense layers
size_t moe_linear_workspace_size(int64_t M, int K, int N_out) {
  if (M < 0 || K <= 0 || N_out <= 0 || K % 128 != 0 || N_out % 128 != 0) return 0;
  return kStatusBytes + kDenseTilesBytes + dense_part_bytes(M, K, N_out, false);
}

int moe_linear(const moe_bf16* x, int64_t M, int K, const moe_bf16* W, int N_out,
               const moe_bf16* residual, moe_bf16* y, void* ws, size_t ws_bytes, void* stream) {
  if (M < 0 || K <= 0 || N_out <= 0) return MOE_ERR_INVALID_ARG;
  if (K % 128 != 0 || N_out % 128 != 0 || M > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!W) return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W)) return MOE_ERR_ALIGNMENT;
  if (M > 0 && (!aligned16(x) || !aligned16(y) || (residual && !aligned16(residual))))
    return MOE_ERR_ALIGNMENT;
  int rc;
  if ((rc = check_ws(ws, ws_bytes, moe_linear_workspace_size(M, K, N_out)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (M == 0) return MOE_OK;
  int32_t* tiles = reinterpret_cast<int32_t*>(body_of(ws));
  float* part = dense_part_bytes(M, K, N_out, false)
                    ? reinterpret_cast<float*>(body_of(ws) + kDenseTilesBytes)
                    : nullptr;
  if (launch_dense_tiles(M, tiles, s) != cudaSuccess) return MOE_ERR_CUDA;
  return linear_run(reinterpret_cast<const __nv_bfloat16*>(x), M, K,
                    reinterpret_cast<const __nv_bfloat16*>(W), N_out,
                    reinterpret_cast<const __nv_bfloat16*>(residual),
                    reinterpret_cast<__nv_bfloat16*>(y), tiles, status_of(ws), s,
                    /*pdl_ok=*/false, part);  // the tile list was written just before
}

size_t moe_shared_experts_workspace_size(int64_t M, int d, int F) {
  if (M < 0 || d <= 0 || F <= 0 || d % 128 != 0 || F % 128 != 0) return 0;
  const size_t p1 = dense_part_bytes(M, d, F, true), p2 = dense_part_bytes(M, F, d, false);
  return kStatusBytes + kDenseTilesBytes +
         align_up(sizeof(__nv_bfloat16) * (size_t)M * (size_t)F, 256) + (p1 > p2 ? p1 : p2);
}

int moe_shared_experts(const moe_bf16* x, int64_t M, int d, int F, const moe_bf16* w1,
                       const moe_bf16* w3, const moe_bf16* w2, const moe_act_cfg* act,
                       const moe_bf16* residual, moe_bf16* y, void* ws, size_t ws_bytes,
                       void* stream) {
  if (M < 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 != 0 || F % 128 != 0 || M > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  int rc;
  if ((rc = check_act(act))) return rc;
  if (!w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_ALIGNMENT;
  if (M > 0 && (!aligned16(x) || !aligned16(y) || (residual && !aligned16(residual))))
    return MOE_ERR_ALIGNMENT;
  if ((rc = check_ws(ws, ws_bytes, moe_shared_experts_workspace_size(M, d, F)))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (M == 0) return MOE_OK;
  uint8_t* body = body_of(ws);
  int32_t* tiles = reinterpret_cast<int32_t*>(body);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(body + kDenseTilesBytes);
  const size_t hb = align_up(sizeof(__nv_bfloat16) * (size_t)M * (size_t)F, 256);
  float* part = reinterpret_cast<float*>(body + kDenseTilesBytes + hb);
  const size_t p1 = dense_part_bytes(M, d, F, true), p2 = dense_part_bytes(M, F, d, false);
  if (launch_dense_tiles(M, tiles, s) != cudaSuccess) return MOE_ERR_CUDA;
  return shared_ffn_run(reinterpret_cast<const __nv_bfloat16*>(x), M, d, F,
                        reinterpret_cast<const __nv_bfloat16*>(w1),
                        reinterpret_cast<const __nv_bfloat16*>(w3),
                        reinterpret_cast<const __nv_bfloat16*>(w2), *act,
                        reinterpret_cast<const __nv_bfloat16*>(residual),
                        reinterpret_cast<__nv_bfloat16*>(y), h, tiles, status_of(ws), s,
                        (p1 || p2) ? part : nullptr);
}

int moe_rms_norm(const moe_bf16* x, int64_t N, int d, const moe_bf16* weight, float eps,
                 moe_bf16* out, void* stream) {
  if (N < 0 || d <= 0 || !(eps >= 0.0f) || !isfinite(eps)) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0 || d > 8192) return MOE_ERR_UNSUPPORTED;
  if (!weight) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!x || !out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(weight) || (N > 0 && (!aligned16(x) || !aligned16(out))))
    return MOE_ERR_ALIGNMENT;
  int rc;
  if ((rc = check_device())) return rc;
  if (N == 0) return MOE_OK;
  return launch_rms_norm(reinterpret_cast<const __nv_bfloat16*>(x), N, d,
                         reinterpret_cast<const __nv_bfloat16*>(weight), eps,
                         reinterpret_cast<__nv_bfloat16*>(out),
                         static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// ------------------------------------------------------------ whole block
namespace {
struct BlockLayout {
  ForwardLayout fwd;     // the routed layer's regions (status word at 0)
  size_t tiles, xe, yc, sh, hsh, part, part_bytes, total;
};

BlockLayout block_layout(int64_t N, const moe_block_dims& d, const moe_route_cfg& c,
                         bool latent, bool shared) {
  BlockLayout L{};
  L.fwd = forward_layout(N, d.d_r, d.d_e, c.num_experts, c.top_k, d.F);
  size_t o = L.fwd.total;
  L.tiles = o; o += kDenseTilesBytes;
  const size_t ne = sizeof(__nv_bfloat16) * (size_t)N * (size_t)d.d_e;
  if (latent) {
    L.xe = o; o += align_up(ne, 256);
    L.yc = o; o += align_up(ne, 256);
  }
  size_t pb = 0;
  auto upd = [&](size_t b) { pb = b > pb ? b : pb; };
  if (latent) {
    upd(dense_part_bytes(N, d.d_r, d.d_e, false));
    upd(dense_part_bytes(N, d.d_e, d.d_r, false));
  }
  if (shared) {
    L.sh = o; o += align_up(sizeof(__nv_bfloat16) * (size_t)N * (size_t)d.d_r, 256);
    L.hsh = o; o += align_up(sizeof(__nv_bfloat16) * (size_t)N * (size_t)d.F_shared, 256);
    upd(dense_part_bytes(N, d.d_r, d.F_shared, true));
    upd(dense_part_bytes(N, d.F_shared, d.d_r, false));
  }
  L.part = o; o += pb;
  L.part_bytes = pb;
  L.total = o;
  return L;
}

int check_block(int64_t N, const moe_block_dims* d, const moe_block_weights* wt,
                const moe_route_cfg* cfg, bool* latent, bool* shared) {
  if (!d || !wt) return MOE_ERR_INVALID_ARG;
  int rc = check_route_cfg(cfg);
  if (rc) return rc;
  if (N < 0 || d->d_r <= 0 || d->d_e <= 0 || d->F <= 0 || d->F_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (!(d->norm_eps >= 0.0f) || !isfinite(d->norm_eps)) return MOE_ERR_INVALID_ARG;
  *latent = wt->down_proj != nullptr;
  *shared = wt->shared_w1 != nullptr;
  if ((wt->up_proj != nullptr) != *latent) return MOE_ERR_INVALID_ARG;
  if (!*latent && (d->d_e != d->d_r || wt->norm_weight)) return MOE_ERR_INVALID_ARG;
  if ((wt->shared_w3 != nullptr) != *shared || (wt->shared_w2 != nullptr) != *shared ||
      (d->F_shared > 0) != *shared)
    return MOE_ERR_INVALID_ARG;
  if (!wt->gate_weight || !wt->w1 || !wt->w3 || !wt->w2) return MOE_ERR_INVALID_ARG;
  if ((rc = check_expert_shape(N * (int64_t)cfg->top_k, d->d_e, cfg->num_experts, d->F)))
    return rc;
  if (d->d_r % 128 != 0 || d->F_shared % 128 != 0 || d->d_e > 8192 || N > INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {wt->gate_weight, wt->down_proj, wt->norm_weight, wt->up_proj, wt->w1,
                        wt->w3, wt->w2, wt->shared_w1, wt->shared_w3, wt->shared_w2};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}
}  // namespace

size_t moe_block_workspace_size(int64_t N, const moe_block_dims* dims,
                                const moe_block_weights* weights, const moe_route_cfg* cfg) {
  bool latent = false, shared = false;
  if (check_block(N, dims, weights, cfg, &latent, &shared) != MOE_OK) return 0;
  return block_layout(N, *dims, *cfg, latent, shared).total;
}

int moe_block_forward(const moe_bf16* x, int64_t N, const moe_block_dims* dims,
                      const moe_block_weights* wt, const moe_route_cfg* cfg,
                      const moe_act_cfg* act, moe_bf16* out, int32_t* topk_idx_out,
                      float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  bool latent = false, shared = false;
  int rc = check_block(N, dims, wt, cfg, &latent, &shared);
  if (rc) return rc;
  if ((rc = check_act(act))) return rc;
  if (N > 0 && (!x || !out)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!aligned16(x) || !aligned16(out))) return MOE_ERR_ALIGNMENT;
  const BlockLayout L = block_layout(N, *dims, *cfg, latent, shared);
  if ((rc = check_ws(ws, ws_bytes, L.total))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(ws, s))) return rc;
  if (N == 0) return MOE_OK;
  const int d_r = dims->d_r, d_e = dims->d_e, E = cfg->num_experts, K = cfg->top_k;
  uint8_t* base = static_cast<uint8_t*>(ws);
  DeviceStatus* st = status_of(ws);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(base + off); };
  auto cbf = [](const moe_bf16* p) { return reinterpret_cast<const __nv_bfloat16*>(p); };
  const ForwardLayout& F = L.fwd;
  uint8_t* stage = base + F.stage;
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(base + F.idx);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + F.w);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + F.offsets);
  int32_t* pos = reinterpret_cast<int32_t*>(base + F.pos);
  int32_t* tiles = reinterpret_cast<int32_t*>(base + L.tiles);
  const __nv_bfloat16* xr = cbf(x);
  __nv_bfloat16* sh = shared ? bf(L.sh) : nullptr;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  float* part = L.part_bytes ? reinterpret_cast<float*>(base + L.part) : nullptr;

  const Range block("moe.block_forward");
  if (launch_dense_tiles(N, tiles, s) != cudaSuccess) return MOE_ERR_CUDA;
  // gate on the full-width input
  {
    const Range r("moe.route");
    if ((rc = route_impl(xr, N, d_r, wt->gate_weight, wt->gate_bias, *cfg, idx, w, stage, st,
                         s)))
      return rc;
  }
  // shared experts on the full-width input (their output is the residual of
  // the last step)
  if (shared && (rc = shared_ffn_run(xr, N, d_r, dims->F_shared, cbf(wt->shared_w1),
                                     cbf(wt->shared_w3), cbf(wt->shared_w2), *act, nullptr, sh,
                                     bf(L.hsh), tiles, st, s, part)))
    return rc;
  // routed_expert_down_proj
  const __nv_bfloat16* xe = xr;
  if (latent) {
    // (the tile list was written before the router's kernels: a programmatic
    // dependent launch is safe here and below)
    if ((rc = linear_run(xr, N, d_r, cbf(wt->down_proj), d_e, nullptr, bf(L.xe), tiles, st, s,
                         true, part)))
      return rc;
    xe = bf(L.xe);
  }
  // moe_infer
  if (launch_dispatch(idx, N, K, E, xe, d_e, reinterpret_cast<int32_t*>(base + F.counts), offsets,
                      reinterpret_cast<int32_t*>(base + F.perm), pos, bf(F.xs),
                      reinterpret_cast<int32_t*>(stage), st, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((rc = expert_ffn_run(bf(F.xs), offsets, E, N * K, d_e, dims->F, cbf(wt->w1), cbf(wt->w3),
                           cbf(wt->w2), *act, bf(F.y), stage, st, s, nullptr)))
    return rc;
  if (!latent)
    return launch_combine(bf(F.y), pos, w, N, K, d_e, N * K, o, st, s, sh) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  // routed_expert_norm (fused with the combine) and routed_expert_up_proj,
  // whose epilogue adds the shared experts' output
  cudaError_t e = wt->norm_weight
                      ? launch_combine_rms_norm(bf(F.y), pos, w, N, K, d_e, N * K,
                                                cbf(wt->norm_weight), dims->norm_eps, bf(L.yc),
                                                st, s)
                      : launch_combine(bf(F.y), pos, w, N, K, d_e, N * K, bf(L.yc), st, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return linear_run(bf(L.yc), N, d_e, cbf(wt->up_proj), d_r, sh, o, tiles, st, s, true, part);
}

}  // extern "C"
