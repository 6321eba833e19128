"""Seeded synthetic inputs for the MoE layer, bit-identical on host and GPU.

The generator (``csrc/synth.h``) maps (seed, tensor id, element index) to a
value; it performs none of the layer's arithmetic.  Tests feed the host twin's
arrays to the CPU reference and the device twin's tensors to the CUDA library.

Host arrays are numpy: bf16 tensors are ``uint16`` bit patterns, fp32 tensors
are ``float32``.  Device tensors are torch CUDA tensors (bf16 / fp32).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .workloads import (  # noqa: F401
    WORKLOADS, Workload, TID_X, TID_W, TID_BIAS, TID_W1, TID_W3, TID_W2, TID_XE, TID_POP,
    get_workload,
)

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        from . import build as _b
        path = _b.build()
        L = ctypes.CDLL(path)
        u64, u32, i64, f32, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                 ctypes.c_float, ctypes.c_void_p)
        for name in ("synth_host_normal_f32", "synth_host_normal_bf16"):
            getattr(L, name).argtypes = [u64, u32, u64, i64, f32, vp]
            getattr(L, name).restype = None
        L.synth_host_uniform_f32.argtypes = [u64, u32, u64, i64, f32, f32, vp]
        L.synth_host_uniform_f32.restype = None
        L.synth_host_raw.argtypes = [u64, u32, u64, i64, vp]
        L.synth_host_raw.restype = None
        for name in ("synth_dev_normal_f32", "synth_dev_normal_bf16"):
            getattr(L, name).argtypes = [u64, u32, u64, i64, f32, vp, vp]
            getattr(L, name).restype = ctypes.c_int
        L.synth_dev_uniform_f32.argtypes = [u64, u32, u64, i64, f32, f32, vp, vp]
        L.synth_dev_uniform_f32.restype = ctypes.c_int
        _lib = L
    return _lib


# ---------------------------------------------------------------- host twin
def host_normal_bf16(seed: int, tid: int, shape, sigma: float, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    lib().synth_host_normal_bf16(seed, tid, start, out.size, sigma, out.ctypes.data)
    return out


def host_normal_f32(seed: int, tid: int, shape, sigma: float, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().synth_host_normal_f32(seed, tid, start, out.size, sigma, out.ctypes.data)
    return out


def host_uniform_f32(seed: int, tid: int, shape, lo: float, hi: float, start: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    lib().synth_host_uniform_f32(seed, tid, start, out.size, lo, hi, out.ctypes.data)
    return out


def host_raw(seed: int, tid: int, count: int, start: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    lib().synth_host_raw(seed, tid, start, count, out.ctypes.data)
    return out


# -------------------------------------------------------------- device twin
def _stream_handle(torch_mod):
    return ctypes.c_void_p(torch_mod.cuda.current_stream().cuda_stream)


def dev_normal_bf16(t, seed: int, tid: int, sigma: float, start: int = 0):
    import torch
    assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    rc = lib().synth_dev_normal_bf16(seed, tid, start, t.numel(), sigma, t.data_ptr(),
                                     _stream_handle(torch))
    if rc != 0:
        raise RuntimeError(f"synth_dev_normal_bf16 failed: cuda error {rc}")
    return t


def dev_normal_f32(t, seed: int, tid: int, sigma: float, start: int = 0):
    import torch
    assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    rc = lib().synth_dev_normal_f32(seed, tid, start, t.numel(), sigma, t.data_ptr(),
                                    _stream_handle(torch))
    if rc != 0:
        raise RuntimeError(f"synth_dev_normal_f32 failed: cuda error {rc}")
    return t


def dev_uniform_f32(t, seed: int, tid: int, lo: float, hi: float, start: int = 0):
    import torch
    assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    rc = lib().synth_dev_uniform_f32(seed, tid, start, t.numel(), lo, hi, t.data_ptr(),
                                     _stream_handle(torch))
    if rc != 0:
        raise RuntimeError(f"synth_dev_uniform_f32 failed: cuda error {rc}")
    return t


# ------------------------------------------------------------ bf16 helpers
def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 values (exact)."""
    return (a.astype(np.uint32) << 16).view(np.float32)
