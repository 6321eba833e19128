"""Python binding of libmoe.so, the B200 (sm_100a) inference MoE layer.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); every call enqueues on ``torch.cuda.current_stream()`` and returns
without synchronising.  The entry points and their semantics are those of
``include/moe.h``.

There is no fallback: if ``libmoe.so`` has not been built, importing the
binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_ACT_SILU, MOE_ACT_SITU = 0, 1
_ERR = {
    0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "misaligned pointer",
    -4: "workspace too small or misaligned", -5: "CUDA call failed",
    -6: "device wait timed out", -7: "device index out of range", -8: "no sm_100 device",
}


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({_ERR.get(code, 'unknown')})")
        self.code = code


class _RouteCfg(ctypes.Structure):
    _fields_ = [("num_experts", ctypes.c_int), ("n_group", ctypes.c_int),
                ("topk_group", ctypes.c_int), ("top_k", ctypes.c_int),
                ("norm_topk_prob", ctypes.c_int), ("route_scale", ctypes.c_float),
                ("score_func", ctypes.c_int), ("group_score", ctypes.c_int)]


class _ActCfg(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("beta", ctypes.c_float),
                ("linear_beta", ctypes.c_float)]


class _StageEvents(ctypes.Structure):
    _fields_ = [("after_route", ctypes.c_void_p), ("after_dispatch", ctypes.c_void_p),
                ("after_gate_up", ctypes.c_void_p), ("after_down", ctypes.c_void_p),
                ("after_combine", ctypes.c_void_p)]


@dataclass(frozen=True)
class RouteConfig:
    num_experts: int
    n_group: int
    topk_group: int
    top_k: int
    route_scale: float
    norm_topk_prob: bool = True
    score_func: str = "sigmoid"   # or "softmax"
    group_score: str = "top2_sum"  # or "max"

    def _c(self) -> _RouteCfg:
        return _RouteCfg(self.num_experts, self.n_group, self.topk_group, self.top_k,
                         int(bool(self.norm_topk_prob)), self.route_scale,
                         {"sigmoid": 0, "softmax": 1}[self.score_func],
                         {"top2_sum": 0, "max": 1}[self.group_score])


class _BlockDims(ctypes.Structure):
    _fields_ = [("d_r", ctypes.c_int), ("d_e", ctypes.c_int), ("F", ctypes.c_int),
                ("F_shared", ctypes.c_int), ("norm_eps", ctypes.c_float)]


MOE_MAX_PEERS = 64


class _PeerRows(ctypes.Structure):
    _fields_ = [("num_ranks", ctypes.c_int), ("rows", ctypes.c_void_p * MOE_MAX_PEERS),
                ("first_row", ctypes.c_int64 * MOE_MAX_PEERS),
                ("capacity", ctypes.c_int64 * MOE_MAX_PEERS)]


def peer_rows(rows, first_row, capacity) -> _PeerRows:
    """The moe_peer_rows table: rows[q] is rank q's row buffer as a device
    address of this GPU (an int, or a tensor on this GPU), first_row[q] this
    rank's first row in it, capacity[q] its rows."""
    P = len(rows)
    if not (1 <= P <= MOE_MAX_PEERS and len(first_row) == P and len(capacity) == P):
        raise ValueError("peer_rows: 1..64 ranks, one first_row and capacity per rank")
    t = _PeerRows()
    t.num_ranks = P
    for q in range(P):
        r = rows[q]
        t.rows[q] = r if isinstance(r, int) else (None if r is None else r.data_ptr())
        t.first_row[q] = int(first_row[q])
        t.capacity[q] = int(capacity[q])
    return t


class _BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "gate_weight", "gate_bias", "down_proj", "norm_weight", "up_proj", "w1", "w3", "w2",
        "shared_w1", "shared_w3", "shared_w2")]


@dataclass
class BlockWeights:
    """Device tensors of one MoE block (None marks an absent part).

    gate_weight [E, d_r] fp32, gate_bias [E] fp32; down_proj [d_e, d_r],
    norm_weight [d_e], up_proj [d_r, d_e]; routed w1, w3 [E, F, d_e], w2
    [E, d_e, F]; shared_w1, shared_w3 [F_sh, d_r], shared_w2 [d_r, F_sh]; bf16.
    """
    gate_weight: object
    w1: object
    w3: object
    w2: object
    gate_bias: object = None
    down_proj: object = None
    norm_weight: object = None
    up_proj: object = None
    shared_w1: object = None
    shared_w3: object = None
    shared_w2: object = None

    def _c(self) -> _BlockWeights:
        return _BlockWeights(*[None if getattr(self, n) is None else getattr(self, n).data_ptr()
                               for n, _ in _BlockWeights._fields_])


@dataclass(frozen=True)
class ActConfig:
    kind: str = "silu"        # "silu" or "situ"
    beta: float = 1.0
    linear_beta: float = 0.0  # 0 = not set

    def _c(self) -> _ActCfg:
        return _ActCfg({"silu": MOE_ACT_SILU, "situ": MOE_ACT_SITU}[self.kind], self.beta,
                       self.linear_beta)


_lib = None
EXPORTS = ("moe_route_workspace_size", "moe_route", "moe_route_from_logits",
           "moe_gate_logits_workspace_size", "moe_gate_logits",
           "moe_dispatch_workspace_size", "moe_dispatch", "moe_expert_ffn_workspace_size",
           "moe_expert_ffn", "moe_combine_workspace_size", "moe_combine", "moe_workspace_size",
           "moe_forward", "moe_get_status", "moe_strerror", "moe_dispatch_static",
           "moe_linear_workspace_size", "moe_linear", "moe_rms_norm", "moe_block_workspace_size",
           "moe_block_forward", "moe_shared_experts_workspace_size", "moe_shared_experts",
           "moe_ep_expert_ffn_workspace_size", "moe_ep_expert_ffn", "moe_expert_ffn_gathered",
           "moe_ep_dispatch_rows", "moe_ep_combine_rows", "moe_launch_count",
           "moe_set_wait_probe", "moe_expert_ffn_to_slots")


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m moe_routing_expert_fp32_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    rc, ac, ev = ctypes.POINTER(_RouteCfg), ctypes.POINTER(_ActCfg), ctypes.POINTER(_StageEvents)
    bd, bw = ctypes.POINTER(_BlockDims), ctypes.POINTER(_BlockWeights)
    pr = ctypes.POINTER(_PeerRows)
    sig = {
        "moe_route_workspace_size": ([i64, i32, rc], sz),
        "moe_route": ([vp, i64, i32, vp, vp, rc, vp, vp, vp, sz, vp], i32),
        "moe_route_from_logits": ([vp, i64, vp, rc, vp, vp, vp, sz, vp], i32),
        "moe_gate_logits_workspace_size": ([i64, i32, i32], sz),
        "moe_gate_logits": ([vp, i64, i32, vp, i32, vp, vp, sz, vp], i32),
        "moe_dispatch_workspace_size": ([i64, i32, i32], sz),
        "moe_dispatch": ([vp, i64, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "moe_expert_ffn_workspace_size": ([i64, i32, i32, i32], sz),
        "moe_expert_ffn": ([vp, vp, i32, i64, i32, i32, vp, vp, vp, ac, vp, vp, sz, vp], i32),
        "moe_combine_workspace_size": ([], sz),
        "moe_combine": ([vp, vp, vp, i64, i32, i32, vp, vp, sz, vp], i32),
        "moe_workspace_size": ([i64, i32, i32, rc, i32], sz),
        "moe_forward": ([vp, vp, i64, i32, i32, vp, vp, rc, vp, vp, vp, i32, ac, vp, vp, vp, vp,
                         sz, vp, ev], i32),
        "moe_get_status": ([vp, vp], i32),
        "moe_dispatch_static": ([vp, i64, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp], i32),
        "moe_strerror": ([i32], ctypes.c_char_p),
        "moe_linear_workspace_size": ([i64, i32, i32], sz),
        "moe_linear": ([vp, i64, i32, vp, i32, vp, vp, vp, sz, vp], i32),
        "moe_rms_norm": ([vp, i64, i32, vp, ctypes.c_float, vp, vp], i32),
        "moe_shared_experts_workspace_size": ([i64, i32, i32], sz),
        "moe_ep_expert_ffn_workspace_size": ([i64, i32, i32, i32, i32], sz),
        "moe_expert_ffn_gathered": ([vp, i64, i32, vp, vp, i32, i32, i32, vp, vp, vp, ac, vp, vp,
                                     sz, vp], i32),
        "moe_ep_expert_ffn": ([vp, i64, vp, i32, i32, i32, i32, vp, vp, vp, ac, vp, vp, sz, vp],
                              i32),
        "moe_shared_experts": ([vp, i64, i32, i32, vp, vp, vp, ac, vp, vp, vp, sz, vp], i32),
        "moe_block_workspace_size": ([i64, bd, bw, rc], sz),
        "moe_block_forward": ([vp, i64, bd, bw, rc, ac, vp, vp, vp, vp, sz, vp], i32),
        "moe_ep_dispatch_rows": ([vp, i64, i32, i32, vp, vp, i32, pr, vp, sz, vp], i32),
        "moe_ep_combine_rows": ([pr, vp, vp, i32, vp, i64, i32, i32, vp, vp, sz, vp], i32),
        "moe_launch_count": ([], ctypes.c_uint64),
        "moe_set_wait_probe": ([i32], i32),
        "moe_expert_ffn_to_slots": ([vp, vp, vp, i32, i64, i32, i32, vp, vp, vp, ac, vp, vp, sz,
                                     vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def launch_count() -> int:
    """Kernels libmoe has launched in this process so far (moe_launch_count)."""
    return int(lib().moe_launch_count())


def set_wait_probe(on: bool) -> bool:
    """Diagnostics: make the grouped expert GEMM's bounded wait run out (see
    moe_set_wait_probe in include/moe.h).  Returns the previous setting."""
    return bool(lib().moe_set_wait_probe(1 if on else 0))


# ----------------------------------------------------------------- helpers
def _torch():
    import torch
    return torch


def _stream():
    return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise MoeError(fn, code)


def _need(t, dtype, shape=None, name="tensor"):
    torch = _torch()
    if not (t.is_cuda and t.is_contiguous() and t.dtype == dtype):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return torch


def workspace(nbytes: int, device=None):
    """A 256-byte aligned device buffer of at least nbytes (torch allocations are)."""
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def get_status(ws) -> int:
    """Device status of the last call on this workspace (synchronises)."""
    return int(lib().moe_get_status(_ptr(ws), _stream()))


# --------------------------------------------------------------- entry points
def route(x, W, bias, cfg: RouteConfig, ws=None):
    torch = _torch()
    N, d_r = x.shape
    _need(x, torch.bfloat16, name="x")
    _need(W, torch.float32, (cfg.num_experts, d_r), "W")
    if bias is not None:
        _need(bias, torch.float32, (cfg.num_experts,), "bias")
    c = cfg._c()
    need = lib().moe_route_workspace_size(N, d_r, ctypes.byref(c))
    ws = workspace(need, x.device) if ws is None else ws
    idx = torch.empty((N, cfg.top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((N, cfg.top_k), dtype=torch.float32, device=x.device)
    _check("moe_route", lib().moe_route(_ptr(x), N, d_r, _ptr(W), _ptr(bias), ctypes.byref(c),
                                        _ptr(idx), _ptr(w), _ptr(ws), ws.numel(), _stream()))
    return idx, w


def gate_logits(x, W, ws=None):
    """fp32 logits [N, E] of the router's gate GEMM (moe_gate_logits)."""
    torch = _torch()
    N, d_r = x.shape
    E = W.shape[0]
    _need(x, torch.bfloat16, name="x")
    _need(W, torch.float32, (E, d_r), "W")
    need = lib().moe_gate_logits_workspace_size(N, d_r, E)
    ws = workspace(need, x.device) if ws is None else ws
    out = torch.empty((N, E), dtype=torch.float32, device=x.device)
    _check("moe_gate_logits", lib().moe_gate_logits(_ptr(x), N, d_r, _ptr(W), E, _ptr(out),
                                                    _ptr(ws), ws.numel(), _stream()))
    return out


def route_from_logits(logits, bias, cfg: RouteConfig, ws=None):
    torch = _torch()
    N, E = logits.shape
    _need(logits, torch.float32, name="logits")
    if E != cfg.num_experts:
        raise ValueError("logits width != num_experts")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    ws = workspace(256, logits.device) if ws is None else ws
    idx = torch.empty((N, cfg.top_k), dtype=torch.int32, device=logits.device)
    w = torch.empty((N, cfg.top_k), dtype=torch.float32, device=logits.device)
    c = cfg._c()
    _check("moe_route_from_logits",
           lib().moe_route_from_logits(_ptr(logits), N, _ptr(bias), ctypes.byref(c), _ptr(idx),
                                       _ptr(w), _ptr(ws), ws.numel(), _stream()))
    return idx, w


def dispatch(topk_idx, x_e, num_experts: int, ws=None, gather=True):
    """(counts [E], offsets [E+1], perm [S], pos [S], xs [S, d_e]); with
    gather=False the rows are not copied and xs is None."""
    torch = _torch()
    N, K = topk_idx.shape
    d_e = x_e.shape[1]
    _need(topk_idx, torch.int32, name="topk_idx")
    _need(x_e, torch.bfloat16, (N, d_e), "x_e")
    E = num_experts
    S = N * K
    dev = x_e.device
    need = lib().moe_dispatch_workspace_size(N, K, E)
    ws = workspace(need, dev) if ws is None else ws
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(S, dtype=torch.int32, device=dev)
    pos = torch.empty(S, dtype=torch.int32, device=dev)
    xs = torch.empty((S, d_e), dtype=torch.bfloat16, device=dev) if gather else None
    _check("moe_dispatch",
           lib().moe_dispatch(_ptr(topk_idx), N, K, E, _ptr(x_e), d_e, _ptr(counts),
                              _ptr(offsets), _ptr(perm), _ptr(pos), _ptr(xs), _ptr(ws),
                              ws.numel(), _stream()))
    return counts, offsets, perm, pos, xs


def dispatch_static(topk_idx, x_e, num_experts: int, gather=True):
    """moe_dispatch without a workspace, for callers that cannot allocate device
    memory: the scratch is a fixed 2 MiB array inside libmoe.so (see
    moe_dispatch_static in include/moe.h for its limit and sharing rules).
    This Python wrapper still allocates its outputs with torch; a caller that
    cannot allocate passes its own buffers to the C entry point.  With
    gather=False the rows are not copied and xs is None."""
    torch = _torch()
    N, K = topk_idx.shape
    d_e = x_e.shape[1]
    _need(topk_idx, torch.int32, name="topk_idx")
    _need(x_e, torch.bfloat16, (N, d_e), "x_e")
    E = num_experts
    S = N * K
    dev = x_e.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(S, dtype=torch.int32, device=dev)
    pos = torch.empty(S, dtype=torch.int32, device=dev)
    xs = torch.empty((S, d_e), dtype=torch.bfloat16, device=dev) if gather else None
    _check("moe_dispatch_static",
           lib().moe_dispatch_static(_ptr(topk_idx), N, K, E, _ptr(x_e), d_e, _ptr(counts),
                                     _ptr(offsets), _ptr(perm), _ptr(pos), _ptr(xs), _stream()))
    return counts, offsets, perm, pos, xs


def expert_ffn(xs, offsets, w1, w3, w2, act: ActConfig, ws=None, y=None):
    torch = _torch()
    S, d_e = xs.shape
    E, F, _ = w1.shape
    _need(xs, torch.bfloat16, name="xs")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(w1, torch.bfloat16, (E, F, d_e), "w1")
    _need(w3, torch.bfloat16, (E, F, d_e), "w3")
    _need(w2, torch.bfloat16, (E, d_e, F), "w2")
    dev = xs.device
    need = lib().moe_expert_ffn_workspace_size(S, d_e, E, F)
    ws = workspace(need, dev) if ws is None else ws
    y = torch.empty((S, d_e), dtype=torch.bfloat16, device=dev) if y is None else y
    a = act._c()
    _check("moe_expert_ffn",
           lib().moe_expert_ffn(_ptr(xs), _ptr(offsets), E, S, d_e, F, _ptr(w1), _ptr(w3),
                                _ptr(w2), ctypes.byref(a), _ptr(y), _ptr(ws), ws.numel(),
                                _stream()))
    return y


def expert_ffn_to_slots(xs, offsets, perm, w1, w3, w2, act: ActConfig, ws=None, y=None):
    """moe_expert_ffn writing output row j to row perm[j] (slot order)."""
    torch = _torch()
    S, d_e = xs.shape
    E, F, _ = w1.shape
    _need(xs, torch.bfloat16, name="xs")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    _need(perm, torch.int32, (S,), "perm")
    _need(w1, torch.bfloat16, (E, F, d_e), "w1")
    _need(w3, torch.bfloat16, (E, F, d_e), "w3")
    _need(w2, torch.bfloat16, (E, d_e, F), "w2")
    dev = xs.device
    need = lib().moe_expert_ffn_workspace_size(S, d_e, E, F)
    ws = workspace(need, dev) if ws is None else ws
    y = torch.empty((S, d_e), dtype=torch.bfloat16, device=dev) if y is None else y
    a = act._c()
    _check("moe_expert_ffn_to_slots",
           lib().moe_expert_ffn_to_slots(_ptr(xs), _ptr(offsets), _ptr(perm), E, S, d_e, F,
                                         _ptr(w1), _ptr(w3), _ptr(w2), ctypes.byref(a), _ptr(y),
                                         _ptr(ws), ws.numel(), _stream()))
    return y


def combine(y, pos, topk_w, ws=None):
    """pos None: y is in slot order (moe_expert_ffn_to_slots)."""
    torch = _torch()
    N, K = topk_w.shape
    d_e = y.shape[1]
    _need(y, torch.bfloat16, (N * K, d_e), "y")
    if pos is not None:
        _need(pos, torch.int32, (N * K,), "pos")
    _need(topk_w, torch.float32, name="topk_w")
    ws = workspace(256, y.device) if ws is None else ws
    out = torch.empty((N, d_e), dtype=torch.bfloat16, device=y.device)
    _check("moe_combine", lib().moe_combine(_ptr(y), _ptr(pos), _ptr(topk_w), N, K, d_e,
                                            _ptr(out), _ptr(ws), ws.numel(), _stream()))
    return out


def workspace_size(N: int, d_r: int, d_e: int, cfg: RouteConfig, F: int) -> int:
    c = cfg._c()
    return int(lib().moe_workspace_size(N, d_r, d_e, ctypes.byref(c), F))


def forward(x_r, W, bias, cfg: RouteConfig, w1, w3, w2, act: ActConfig, x_e=None, ws=None,
            out=None, topk_idx=None, topk_w=None, events=None):
    """The routed MoE layer (moe_forward). Returns ``out`` [N, d_e] bf16.

    ``events``: optional dict of torch.cuda.Event recorded between the stages
    (keys after_route, after_dispatch, after_gate_up, after_down, after_combine).
    """
    torch = _torch()
    N, d_r = x_r.shape
    E, F, d_e = w1.shape
    _need(x_r, torch.bfloat16, name="x_r")
    if x_e is not None:
        _need(x_e, torch.bfloat16, (N, d_e), "x_e")
    elif d_e != d_r:
        raise ValueError("x_e is required when the experts' width differs from the router's")
    _need(W, torch.float32, (E, d_r), "W")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    dev = x_r.device
    c = cfg._c()
    a = act._c()
    need = lib().moe_workspace_size(N, d_r, d_e, ctypes.byref(c), F)
    ws = workspace(need, dev) if ws is None else ws
    out = torch.empty((N, d_e), dtype=torch.bfloat16, device=dev) if out is None else out
    evp = None
    if events:
        se = _StageEvents(*[ctypes.c_void_p(events[k].cuda_event) if k in events else None
                            for k in ("after_route", "after_dispatch", "after_gate_up",
                                      "after_down", "after_combine")])
        evp = ctypes.byref(se)
    _check("moe_forward",
           lib().moe_forward(_ptr(x_r), _ptr(x_e), N, d_r, d_e, _ptr(W), _ptr(bias),
                             ctypes.byref(c), _ptr(w1), _ptr(w3), _ptr(w2), F, ctypes.byref(a),
                             _ptr(out), _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel(),
                             _stream(), evp))
    return out


# ------------------------------------------------------- the block around it
def linear(x, W, residual=None, out=None, ws=None):
    """bf16(x . W^T) (+ residual) through moe_linear; x [M, K], W [N_out, K]."""
    torch = _torch()
    M, K = x.shape
    N_out = W.shape[0]
    _need(x, torch.bfloat16, name="x")
    _need(W, torch.bfloat16, (N_out, K), "W")
    if residual is not None:
        _need(residual, torch.bfloat16, (M, N_out), "residual")
    need = lib().moe_linear_workspace_size(M, K, N_out)
    if need == 0:
        raise MoeError("moe_linear_workspace_size", -1)
    ws = workspace(need, x.device) if ws is None else ws
    out = torch.empty((M, N_out), dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("moe_linear", lib().moe_linear(_ptr(x), M, K, _ptr(W), N_out, _ptr(residual),
                                          _ptr(out), _ptr(ws), ws.numel(), _stream()))
    return out


def expert_ffn_gathered(x_e, K, perm, offsets, w1, w3, w2, act: ActConfig, ws=None, y=None):
    """moe_expert_ffn_gathered: the expert MLP on the rows x_e[perm // K]
    without a gathered copy (decode and mid-size batches)."""
    torch = _torch()
    N, d_e = x_e.shape
    E, F, _ = w1.shape
    S = N * K
    _need(x_e, torch.bfloat16, name="x_e")
    _need(perm, torch.int32, (S,), "perm")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    need = lib().moe_expert_ffn_workspace_size(S, d_e, E, F)
    ws = workspace(need, x_e.device) if ws is None else ws
    y = torch.empty((S, d_e), dtype=torch.bfloat16, device=x_e.device) if y is None else y
    a = act._c()
    _check("moe_expert_ffn_gathered",
           lib().moe_expert_ffn_gathered(_ptr(x_e), N, K, _ptr(perm), _ptr(offsets), E, d_e, F,
                                         _ptr(w1), _ptr(w3), _ptr(w2), ctypes.byref(a), _ptr(y),
                                         _ptr(ws), ws.numel(), _stream()))
    return y


def ep_expert_ffn(xr, recv_counts, w1, w3, w2, act: ActConfig, y=None, ws=None):
    """The local experts on rows received from P ranks (moe_ep_expert_ffn):
    xr [R, d_e] grouped by source rank, then local expert; recv_counts
    [P, E_local] int32 on the device; w1, w3 [E_local, F, d_e], w2
    [E_local, d_e, F]."""
    torch = _torch()
    R, d_e = xr.shape
    P, E_local = recv_counts.shape
    F = w1.shape[1]
    _need(xr, torch.bfloat16, name="xr")
    _need(recv_counts, torch.int32, (P, E_local), "recv_counts")
    _need(w1, torch.bfloat16, (E_local, F, d_e), "w1")
    _need(w3, torch.bfloat16, (E_local, F, d_e), "w3")
    _need(w2, torch.bfloat16, (E_local, d_e, F), "w2")
    need = lib().moe_ep_expert_ffn_workspace_size(R, d_e, P, E_local, F)
    ws = workspace(need, xr.device) if ws is None else ws
    y = torch.empty((R, d_e), dtype=torch.bfloat16, device=xr.device) if y is None else y
    a = act._c()
    _check("moe_ep_expert_ffn",
           lib().moe_ep_expert_ffn(_ptr(xr), R, _ptr(recv_counts), P, E_local, d_e, F, _ptr(w1),
                                   _ptr(w3), _ptr(w2), ctypes.byref(a), _ptr(y), _ptr(ws),
                                   ws.numel(), _stream()))
    return y


def ep_dispatch_rows(x_e, pos, offsets, num_experts: int, peers: _PeerRows, K: int, ws=None):
    """Store every token row of x_e [N, d_e] into the receiving ranks' buffers
    (moe_ep_dispatch_rows); pos [N*K], offsets [E+1] from dispatch()."""
    torch = _torch()
    N, d_e = x_e.shape
    _need(x_e, torch.bfloat16, name="x_e")
    _need(pos, torch.int32, (N * K,), "pos")
    _need(offsets, torch.int32, (num_experts + 1,), "offsets")
    ws = workspace(256, x_e.device) if ws is None else ws
    _check("moe_ep_dispatch_rows",
           lib().moe_ep_dispatch_rows(_ptr(x_e), N, K, d_e, _ptr(pos), _ptr(offsets), num_experts,
                                      ctypes.byref(peers), _ptr(ws), ws.numel(), _stream()))


def ep_combine_rows(peers: _PeerRows, pos, offsets, num_experts: int, topk_w, d_e: int, out=None,
                    ws=None):
    """The weighted combine with each slot's output loaded from the rank that
    computed it (moe_ep_combine_rows); returns out [N, d_e] bf16."""
    torch = _torch()
    N, K = topk_w.shape
    _need(topk_w, torch.float32, name="topk_w")
    _need(pos, torch.int32, (N * K,), "pos")
    _need(offsets, torch.int32, (num_experts + 1,), "offsets")
    dev = topk_w.device
    ws = workspace(256, dev) if ws is None else ws
    out = torch.empty((N, d_e), dtype=torch.bfloat16, device=dev) if out is None else out
    _check("moe_ep_combine_rows",
           lib().moe_ep_combine_rows(ctypes.byref(peers), _ptr(pos), _ptr(offsets), num_experts,
                                     _ptr(topk_w), N, K, d_e, _ptr(out), _ptr(ws), ws.numel(),
                                     _stream()))
    return out


def shared_experts(x, w1, w3, w2, act: ActConfig, residual=None, out=None, ws=None):
    """The shared experts' gated MLP on every row (moe_shared_experts)."""
    torch = _torch()
    M, d = x.shape
    F = w1.shape[0]
    _need(x, torch.bfloat16, name="x")
    _need(w1, torch.bfloat16, (F, d), "w1")
    _need(w3, torch.bfloat16, (F, d), "w3")
    _need(w2, torch.bfloat16, (d, F), "w2")
    if residual is not None:
        _need(residual, torch.bfloat16, (M, d), "residual")
    need = lib().moe_shared_experts_workspace_size(M, d, F)
    if need == 0:
        raise MoeError("moe_shared_experts_workspace_size", -1)
    ws = workspace(need, x.device) if ws is None else ws
    out = torch.empty((M, d), dtype=torch.bfloat16, device=x.device) if out is None else out
    a = act._c()
    _check("moe_shared_experts",
           lib().moe_shared_experts(_ptr(x), M, d, F, _ptr(w1), _ptr(w3), _ptr(w2),
                                    ctypes.byref(a), _ptr(residual), _ptr(out), _ptr(ws),
                                    ws.numel(), _stream()))
    return out


def rms_norm(x, weight, eps, out=None):
    torch = _torch()
    N, d = x.shape
    _need(x, torch.bfloat16, name="x")
    _need(weight, torch.bfloat16, (d,), "weight")
    out = torch.empty_like(x) if out is None else out
    _check("moe_rms_norm", lib().moe_rms_norm(_ptr(x), N, d, _ptr(weight), float(eps), _ptr(out),
                                              _stream()))
    return out


def block_forward(x, weights: BlockWeights, cfg: RouteConfig, act: ActConfig, norm_eps=1e-6,
                  ws=None, out=None, topk_idx=None, topk_w=None):
    """KimiSparseMoeBlock.forward (moe_block_forward). Returns ``out`` [N, d_r] bf16."""
    torch = _torch()
    N, d_r = x.shape
    E, F, d_e = weights.w1.shape
    _need(x, torch.bfloat16, name="x")
    _need(weights.gate_weight, torch.float32, (E, d_r), "gate_weight")
    if weights.down_proj is not None:
        _need(weights.down_proj, torch.bfloat16, (d_e, d_r), "down_proj")
        _need(weights.up_proj, torch.bfloat16, (d_r, d_e), "up_proj")
    F_sh = 0 if weights.shared_w1 is None else weights.shared_w1.shape[0]
    dims = _BlockDims(d_r, d_e, F, F_sh, float(norm_eps))
    wc = weights._c()
    c = cfg._c()
    a = act._c()
    need = lib().moe_block_workspace_size(N, ctypes.byref(dims), ctypes.byref(wc), ctypes.byref(c))
    if need == 0:
        raise MoeError("moe_block_workspace_size", -1)
    ws = workspace(need, x.device) if ws is None else ws
    out = torch.empty((N, d_r), dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("moe_block_forward",
           lib().moe_block_forward(_ptr(x), N, ctypes.byref(dims), ctypes.byref(wc),
                                   ctypes.byref(c), ctypes.byref(a), _ptr(out), _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(ws), ws.numel(), _stream()))
    return out
