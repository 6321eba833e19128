"""ctypes binding of the CPU reference (``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check of the
graft entry point and by the CPU-baseline leg of ``bench.py``, never by the
product.  bf16 arrays are numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build

ACT_SILU, ACT_SITU = 0, 1
SCORE_SIGMOID, SCORE_SOFTMAX = 0, 1
GROUP_TOP2_SUM, GROUP_MAX = 0, 1
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build())
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "oracle_set_threads": ([i32], None),
            "oracle_max_threads": ([], i32),
            "oracle_gate_logits": ([vp, i64, i32, vp, i32, vp], None),
            "oracle_sigmoid": ([f32], f32),
            "oracle_group_scores": ([vp, i64, i32, i32, vp], None),
            "oracle_route_from_logits": ([vp, i64, i32, vp, i32, i32, i32, i32, f32, vp, vp, vp],
                                         None),
            "oracle_route_from_logits_ex": ([vp, i64, i32, vp, i32, i32, i32, i32, f32, i32, i32,
                                             vp, vp, vp], None),
            "oracle_group_scores_ex": ([vp, i64, i32, i32, i32, vp], None),
            "oracle_choice_scores_ex": ([vp, i64, i32, vp, i32, i32, i32, i32, vp], None),
            "oracle_choice_scores": ([vp, i64, i32, vp, i32, i32, vp], None),
            "oracle_dispatch": ([vp, i64, i32, i32, vp, vp, vp, vp], None),
            "oracle_gather": ([vp, i32, vp, i64, i32, vp], None),
            "oracle_expert_ffn": ([vp, i64, i32, i32, vp, vp, vp, i32, f32, f32, vp], None),
            "oracle_combine": ([vp, vp, vp, i64, i32, i32, vp], None),
            "oracle_moe_infer_ws_bytes": ([i64, i32, i32, i32], ctypes.c_size_t),
            "oracle_moe_infer": ([vp, i64, i32, vp, vp, i32, i32, i32, vp, vp, vp, i32, f32, f32,
                                  vp, vp], None),
            "oracle_moe_dense": ([vp, i64, i32, vp, vp, i32, i32, vp, vp, vp, i32, f32, f32, vp],
                                 None),
            "oracle_linear": ([vp, i64, i32, vp, i32, vp], None),
            "oracle_add": ([vp, vp, i64, vp], None),
            "oracle_rms_norm": ([vp, i64, i32, vp, f32, vp], None),
            "oracle_bf16_round_double": ([ctypes.c_double], ctypes.c_uint16),
            "oracle_bf16_round_float": ([f32], ctypes.c_uint16),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def act_code(act: str) -> int:
    return {"silu": ACT_SILU, "situ": ACT_SITU}[act]


# ------------------------------------------------------------------ router
def gate_logits(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    x = _c(x, np.uint16)
    W = _c(W, np.float32)
    N, d = x.shape
    E = W.shape[0]
    assert W.shape[1] == d
    out = np.empty((N, E), dtype=np.float32)
    lib().oracle_gate_logits(_p(x), N, d, _p(W), E, _p(out))
    return out


def sigmoid(L: float) -> float:
    return float(lib().oracle_sigmoid(float(L)))


def group_scores(c: np.ndarray, G: int, mode: int = GROUP_TOP2_SUM) -> np.ndarray:
    c = _c(c, np.float32)
    N, E = c.shape
    out = np.empty((N, G), dtype=np.float32)
    lib().oracle_group_scores_ex(_p(c), N, E, G, int(mode), _p(out))
    return out


def route_from_logits(logits, bias, G, TG, K, route_scale, norm=True, score=SCORE_SIGMOID,
                      group=GROUP_TOP2_SUM):
    """(idx int32 [N,K], w fp32 [N,K], margin float64 [N])."""
    logits = _c(logits, np.float32)
    N, E = logits.shape
    b = None if bias is None else _c(bias, np.float32)
    idx = np.empty((N, K), dtype=np.int32)
    w = np.empty((N, K), dtype=np.float32)
    margin = np.empty((N,), dtype=np.float64)
    lib().oracle_route_from_logits_ex(_p(logits), N, E, _p(b), G, TG, K, int(bool(norm)),
                                      float(route_scale), int(score), int(group), _p(idx), _p(w),
                                      _p(margin))
    return idx, w, margin


def choice_scores(logits, bias, G, TG, score=SCORE_SIGMOID, group=GROUP_TOP2_SUM) -> np.ndarray:
    logits = _c(logits, np.float32)
    N, E = logits.shape
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((N, E), dtype=np.float32)
    lib().oracle_choice_scores_ex(_p(logits), N, E, _p(b), G, TG, int(score), int(group), _p(out))
    return out


def route(x, W, bias, G, TG, K, route_scale, norm=True, score=SCORE_SIGMOID,
          group=GROUP_TOP2_SUM):
    return route_from_logits(gate_logits(x, W), bias, G, TG, K, route_scale, norm, score, group)


# --------------------------------------------------------------- moe_infer
def dispatch(idx: np.ndarray, E: int):
    """(counts [E], offsets [E+1], perm [S], pos [S]) as int32."""
    idx = _c(idx, np.int32)
    N, K = idx.shape
    S = N * K
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(S, np.int32)
    pos = np.empty(S, np.int32)
    lib().oracle_dispatch(_p(idx), N, K, E, _p(counts), _p(offsets), _p(perm), _p(pos))
    return counts, offsets, perm, pos


def gather(x: np.ndarray, perm: np.ndarray, K: int) -> np.ndarray:
    x = _c(x, np.uint16)
    perm = _c(perm, np.int32)
    S = perm.size
    d = x.shape[1]
    xs = np.empty((S, d), dtype=np.uint16)
    lib().oracle_gather(_p(x), d, _p(perm), S, K, _p(xs))
    return xs


def expert_ffn(xs, w1, w3, w2, act="silu", beta=1.0, lbeta=0.0) -> np.ndarray:
    xs = _c(xs, np.uint16)
    w1, w3, w2 = (_c(a, np.uint16) for a in (w1, w3, w2))
    n, d = xs.shape
    F = w1.shape[0]
    assert w1.shape == (F, d) and w3.shape == (F, d) and w2.shape == (d, F)
    y = np.empty((n, d), dtype=np.uint16)
    if n:
        lib().oracle_expert_ffn(_p(xs), n, d, F, _p(w1), _p(w3), _p(w2), act_code(act),
                                float(beta), float(lbeta), _p(y))
    return y


def combine(y, pos, w, K: int) -> np.ndarray:
    y = _c(y, np.uint16)
    pos = _c(pos, np.int32)
    w = _c(w, np.float32)
    N = w.size // K
    d = y.shape[1]
    out = np.empty((N, d), dtype=np.uint16)
    lib().oracle_combine(_p(y), _p(pos), _p(w), N, K, d, _p(out))
    return out


def moe_infer(x_e, idx, w, w1, w3, w2, act="silu", beta=1.0, lbeta=0.0) -> np.ndarray:
    """Sorted-dispatch moe_infer on stacked weights (w1/w3 [E,F,d], w2 [E,d,F])."""
    x_e = _c(x_e, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    w1, w3, w2 = (_c(a, np.uint16) for a in (w1, w3, w2))
    N, d = x_e.shape
    K = idx.shape[1]
    E, F = w1.shape[0], w1.shape[1]
    ws = np.empty(int(lib().oracle_moe_infer_ws_bytes(N, K, E, d)), dtype=np.uint8)
    out = np.empty((N, d), dtype=np.uint16)
    lib().oracle_moe_infer(_p(x_e), N, d, _p(idx), _p(w), K, E, F, _p(w1), _p(w3), _p(w2),
                           act_code(act), float(beta), float(lbeta), _p(out), _p(ws))
    return out


def moe_dense(x_e, idx, w, w1, w3, w2, act="silu", beta=1.0, lbeta=0.0) -> np.ndarray:
    """The same layer as a per-token dense loop (no sort)."""
    x_e = _c(x_e, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    w1, w3, w2 = (_c(a, np.uint16) for a in (w1, w3, w2))
    N, d = x_e.shape
    K = idx.shape[1]
    F = w1.shape[1]
    out = np.empty((N, d), dtype=np.uint16)
    lib().oracle_moe_dense(_p(x_e), N, d, _p(idx), _p(w), K, F, _p(w1), _p(w3), _p(w2),
                           act_code(act), float(beta), float(lbeta), _p(out))
    return out


# ----------------------------------------------------- the block around it
def linear(x, W) -> np.ndarray:
    """Bias-free bf16 Linear: bf16(x . W^T), x [M, K], W [N_out, K]."""
    x = _c(x, np.uint16)
    W = _c(W, np.uint16)
    M, K = x.shape
    Nout = W.shape[0]
    assert W.shape[1] == K
    y = np.empty((M, Nout), dtype=np.uint16)
    if M:
        lib().oracle_linear(_p(x), M, K, _p(W), Nout, _p(y))
    return y


def add(a, b) -> np.ndarray:
    a = _c(a, np.uint16)
    b = _c(b, np.uint16)
    assert a.shape == b.shape
    out = np.empty_like(a)
    lib().oracle_add(_p(a), _p(b), a.size, _p(out))
    return out


def rms_norm(x, w, eps: float) -> np.ndarray:
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    N, d = x.shape
    assert w.shape == (d,)
    out = np.empty_like(x)
    if N:
        lib().oracle_rms_norm(_p(x), N, d, _p(w), float(eps), _p(out))
    return out


def block_forward(x, W, bias, G, TG, K, route_scale, w1, w3, w2, act="silu", beta=1.0,
                  lbeta=0.0, norm=True, down_proj=None, norm_w=None, eps=1e-6, up_proj=None,
                  shared=None, score=SCORE_SIGMOID, group=GROUP_TOP2_SUM):
    """KimiSparseMoeBlock.forward ("Kimi K3 · Add shared output", moe-forward):
    gate on the full-width x; optional routed_expert_down_proj; moe_infer;
    optional routed_expert_norm and routed_expert_up_proj; plus the shared
    experts (w1, w3, w2) on x.  Returns (out, idx, w, margin)."""
    idx, w, margin = route(x, W, bias, G, TG, K, route_scale, norm, score, group)
    xe = linear(x, down_proj) if down_proj is not None else _c(x, np.uint16)
    y = moe_infer(xe, idx, w, w1, w3, w2, act, beta, lbeta)
    if down_proj is not None:
        if norm_w is not None:
            y = rms_norm(y, norm_w, eps)
        y = linear(y, up_proj)
    if shared is not None:
        y = add(y, expert_ffn(x, *shared, act=act, beta=beta, lbeta=lbeta))
    return y, idx, w, margin


def bf16_round_double(v: float) -> int:
    return int(lib().oracle_bf16_round_double(float(v)))


def bf16_round_float(v: float) -> int:
    return int(lib().oracle_bf16_round_float(float(v)))
