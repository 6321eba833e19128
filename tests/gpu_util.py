"""Helpers for the GPU parity tests: moving bf16 bit patterns between numpy and
torch, comparison metrics, and the parity tolerances."""
from __future__ import annotations

import numpy as np

# Tolerances of the parity contract.
REL_L2_OUT = 2e-2     # layer / expert outputs, relative L2 in bf16
W_REL = 1e-5          # routing weights (end to end, aligned by expert id)
MARGIN = 1e-5         # biased-score margin above which end-to-end indices must match


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(a_bits: np.ndarray) -> np.ndarray:
    return (a_bits.astype(np.uint32) << 16).view(np.float32)


def rel_l2(got_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    g = f32(got_bits).astype(np.float64)
    r = f32(ref_bits).astype(np.float64)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / (den if den > 0 else 1.0))


def ulp_diff(got_bits: np.ndarray, ref_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place (sign-magnitude aware)."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), b + 0x8000)
    return np.abs(ordered(got_bits) - ordered(ref_bits))


def random_topk(N: int, K: int, E: int, rng, skew: float = 0.0) -> np.ndarray:
    """Distinct expert ids per token; skew > 0 draws with Zipf-like popularity."""
    if skew > 0:
        p = np.arange(1, E + 1, dtype=np.float64) ** -skew
        p /= p.sum()
        keys = rng.random((N, E)) ** (1.0 / p)[None, :]  # weighted sampling w/o replacement
        return np.argsort(-keys, axis=1)[:, :K].astype(np.int32)
    keys = rng.random((N, E))
    return np.argsort(keys, axis=1)[:, :K].astype(np.int32)
