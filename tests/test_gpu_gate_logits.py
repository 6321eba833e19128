"""The router's gate GEMM alone (moe_gate_logits) against the reference's
double-accumulated, once-rounded fp32 logits, on both kernel paths:
  * fp32 FMA chains of 32 terms added in double (batches too small to fill the
    GPU with tensor-core tiles): |error| <= 2e-6 on unit-scale data;
  * exact int8 products of 7-bit digits on the tensor cores (larger batches):
    |error| <= 2e-7 + 2^-22 |L|, i.e. within about two fp32 ulps.
On rows spanning many binades both are held to the scale of the standard dot
product error bound, |error| <= 2^-19 * sum_j |x_j w_j|.  All of these are far
inside what the 1e-5 routing-weight tolerance needs."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def _bf16(a):
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def uses_int8(N, E, d):
    """The library's choice: int8 tiles (128 experts x 96 tokens) when at least
    24 of them fill the GPU."""
    return ((E + 127) // 128) * ((N + 95) // 96) >= 24 and d % 64 == 0


def _check(moe, x, W, rows=None, wide=False):
    import torch
    N, d = x.shape
    E = W.shape[0]
    L = moe.gate_logits(dev_bf16(x), torch.from_numpy(W).cuda()).cpu().numpy()
    if rows is None:
        rows = np.arange(N)
    xr = np.ascontiguousarray(x[rows])
    ref = oracle.gate_logits(xr, W).astype(np.float64)
    got = L[rows].astype(np.float64)
    err = np.abs(got - ref)
    i8 = uses_int8(N, E, d)
    if wide:
        xf = (xr.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        scale = np.abs(xf) @ np.abs(W.astype(np.float64)).T
        bound = 2.0 ** -19 * scale + 1e-30
    elif i8:
        bound = 2e-7 + 2.0 ** -22 * np.abs(ref)
    else:
        bound = np.full_like(ref, 2e-6)
    exact = float((got == ref).mean())
    print(f"N={N} E={E} d={d} {'int8' if i8 else 'fp32'}: max err {err.max():.3e}, "
          f"worst err/bound {(err / bound).max():.3f}, bit-exact {exact:.4f}")
    assert (err <= bound).all(), float((err / bound).max())
    return exact


@pytest.fixture(scope="module")
def moe():
    import moe_routing_expert_fp32_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("N,d,E", [(64, 256, 16), (128, 7168, 256), (64, 7168, 896),
                                   (4096, 7168, 384), (3000, 512, 100), (2000, 1024, 1024),
                                   (2304, 9216, 128), (2304, 16448, 128)])
def test_gate_logits_match_reference(moe, N, d, E):
    x = synth.host_normal_bf16(5, 1, (N, d), 1.0)
    W = synth.host_normal_f32(5, 2, (E, d), 0.02)
    rows = None if N * E * d <= 2e9 else np.unique(
        np.concatenate([np.arange(64), np.arange(N - 64, N),
                        np.random.default_rng(0).choice(N, 256, False)]))
    _check(moe, x, W, rows)


@pytest.mark.parametrize("N", [64, 6144])
def test_gate_logits_wide_range_and_zero_rows(moe, N):
    rng = np.random.default_rng(N)
    d, E = 1024, 200
    x = rng.standard_normal((N, d)).astype(np.float32)
    x[rng.random((N, d)) < 0.1] = 0.0           # zeros inside rows
    x[3] = 0.0                                   # an all-zero token
    x[5] *= np.float32(2.0 ** -30)               # a tiny token
    x = _bf16(x)
    W = (rng.standard_normal((E, d)) * 0.02 *
         2.0 ** rng.uniform(-20, 0, (E, d))).astype(np.float32)  # 20 binades inside a row
    W[7] = 0.0                                    # an all-zero expert
    W[9] *= np.float32(2.0 ** 40)                 # a huge expert
    _check(moe, x, W, wide=True)
