// api.cu -- the C ABI of libmoe: argument validation, workspace layout, launch
// sequencing.  Nothing here computes the layer; every step runs in the
// kernels of router.cu, dispatch.cu, expert_gemm.cu and combine.cu.
#include <math.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {

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
  if (launch_gate(x, N, d_r, W, E, scratch, st, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_select(route_logits_of(scratch), 1, N, bias, cfg, idx, w, st, s) != cudaSuccess)
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
  return launch_select(logits, 1, N, bias, *cfg, topk_idx, topk_w, status_of(ws), s) ==
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
  if (N > 0 && (!topk_idx || !x_e || !perm || !pos || !xs)) return MOE_ERR_INVALID_ARG;
  if (N > 0 && (!aligned16(x_e) || !aligned16(xs))) return MOE_ERR_ALIGNMENT;
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

// ----------------------------------------------------------------- combine
size_t moe_combine_workspace_size(void) { return kStatusBytes; }

int moe_combine(const moe_bf16* y, const int32_t* pos, const float* topk_w, int64_t N, int K,
                int d_e, moe_bf16* out, void* ws, size_t ws_bytes, void* stream) {
  if (N < 0 || K < 1 || d_e <= 0) return MOE_ERR_INVALID_ARG;
  if (K > 16) return MOE_ERR_UNSUPPORTED;
  if (d_e % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (N > 0 && (!y || !pos || !topk_w || !out)) return MOE_ERR_INVALID_ARG;
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

// ------------------------------------------------------------ whole layer
namespace {
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
  if ((rc = route_impl(reinterpret_cast<const __nv_bfloat16*>(x_r), N, d_r, W, bias, *cfg, idx, w,
                       stage, st, s)))
    return rc;
  if (events && !rec(events->after_route)) return MOE_ERR_CUDA;
  if (launch_dispatch(idx, N, K, E, reinterpret_cast<const __nv_bfloat16*>(x_e), d_e, counts,
                      offsets, perm, pos, xs, reinterpret_cast<int32_t*>(stage), st,
                      s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (events && !rec(events->after_dispatch)) return MOE_ERR_CUDA;
  if ((rc = expert_ffn_run(xs, offsets, E, N * K, d_e, F,
                           reinterpret_cast<const __nv_bfloat16*>(w1),
                           reinterpret_cast<const __nv_bfloat16*>(w3),
                           reinterpret_cast<const __nv_bfloat16*>(w2), *act, y, stage, st, s,
                           events ? static_cast<cudaEvent_t>(events->after_gate_up) : nullptr)))
    return rc;
  if (events && !rec(events->after_down)) return MOE_ERR_CUDA;
  if (launch_combine(y, pos, w, N, K, d_e, N * K, reinterpret_cast<__nv_bfloat16*>(out), st, s) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (events && !rec(events->after_combine)) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
