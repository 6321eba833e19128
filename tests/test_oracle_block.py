"""Pins of the CPU reference's block around moe_infer against things other than itself.

Block: KimiSparseMoeBlock.forward ("Kimi K3 · Add shared output", moe-forward
excerpt): routed_expert_down_proj, moe_infer, routed_expert_norm,
routed_expert_up_proj, plus shared_experts(identity).  Pins used here:
  * Linear outputs equal the correctly rounded bf16 of the exact rational dot
    product, with a trap that an fp32 running sum fails;
  * the bf16 add equals the correctly rounded exact sum;
  * RMSNorm against a 60-digit decimal evaluation of its definition, and its
    closed forms (constant rows, one-hot rows, power-of-two scale invariance);
  * the block against a per-token loop over tokens and experts built from the
    pinned parts, and its reductions when a part is zero or the identity.
"""
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.helpers import bf16_to_f32, fraction_to_bf16_bits, near_midpoint


def _bf16(a):
    """fp32 values that are exactly bf16 -> bit patterns."""
    u = np.asarray(a, np.float32).view(np.uint32)
    assert (u & 0xFFFF == 0).all()
    return (u >> 16).astype(np.uint16)


def _rand_bf16(rng, shape, scale=1.0):
    v = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 will do


# ------------------------------------------------------------------- linear
@pytest.mark.parametrize("M,K,N", [(5, 64, 7), (3, 256, 4), (1, 1, 1), (9, 33, 2)])
def test_linear_exact(M, K, N):
    rng = np.random.default_rng(M * 100 + K + N)
    x = _rand_bf16(rng, (M, K))
    W = _rand_bf16(rng, (N, K), 0.05)
    y = oracle.linear(x, W)
    xf = [[Fraction(float(v)) for v in row] for row in bf16_to_f32(x)]
    wf = [[Fraction(float(v)) for v in row] for row in bf16_to_f32(W)]
    for m in range(M):
        for n in range(N):
            q = sum(a * b for a, b in zip(xf[m], wf[n]))
            if not near_midpoint(q, 8, 1e-12):
                assert int(y[m, n]) == fraction_to_bf16_bits(q), (m, n)


def test_linear_accumulates_exactly():
    # 2^24, then 64 halves, then -2^24: exact 32; an fp32 running sum gives 0
    x = np.array([[2.0 ** 12] + [0.5] * 64 + [-(2.0 ** 12)]], np.float32)
    W = np.array([[2.0 ** 12] + [1.0] * 64 + [2.0 ** 12]], np.float32)
    assert oracle.linear(_bf16(x), _bf16(W))[0, 0] == _bf16([32.0])[0]


def test_linear_identity_and_empty():
    rng = np.random.default_rng(3)
    x = _rand_bf16(rng, (6, 32))
    eye = _bf16(np.eye(32, dtype=np.float32))
    assert np.array_equal(oracle.linear(x, eye), x)
    assert oracle.linear(np.zeros((0, 32), np.uint16), eye).shape == (0, 32)


# ---------------------------------------------------------------------- add
def test_add_is_rounded_exact_sum():
    rng = np.random.default_rng(4)
    a = _rand_bf16(rng, (4000,))
    b = _rand_bf16(rng, (4000,), 0.01)
    out = oracle.add(a, b)
    af, bf = bf16_to_f32(a), bf16_to_f32(b)
    for i in range(0, 4000, 7):
        q = Fraction(float(af[i])) + Fraction(float(bf[i]))
        if q != 0 and not near_midpoint(q, 8, 1e-15):
            assert int(out[i]) == fraction_to_bf16_bits(q), i
    assert np.array_equal(out, oracle.add(b, a))
    # a tie (1 + 2^-8) goes to even; 1 + 3*2^-9 rounds up
    assert oracle.add(_bf16([1.0, 1.0]), _bf16([2.0 ** -8, 3 * 2.0 ** -9])).tolist() == \
        _bf16([1.0, 1.0 + 2.0 ** -7]).tolist()


# ------------------------------------------------------------------ RMSNorm
def _decimal_rms(row, w, eps, prec=60):
    """Each output's exact n_i = y_i / sqrt(mean(y^2) + eps), as a Fraction."""
    getcontext().prec = prec
    ys = [Decimal(float(v)) for v in row]
    ms = sum((v * v for v in ys), Decimal(0)) / Decimal(len(ys)) + Decimal(float(np.float32(eps)))
    r = Decimal(1) / ms.sqrt()
    return [Fraction(v * r) for v in ys]


@pytest.mark.parametrize("d,eps,scale", [(128, 1e-6, 1.0), (2048, 1e-6, 3.0), (64, 1e-2, 0.01),
                                         (256, 0.0, 1.0)])
def test_rms_norm_matches_decimal(d, eps, scale):
    rng = np.random.default_rng(d + int(eps * 1e6))
    x = _rand_bf16(rng, (4, d), scale)
    w = _bf16(np.float32(1.0) + (rng.integers(-64, 64, d) / 128.0).astype(np.float32))
    out = oracle.rms_norm(x, w, eps)
    wf = bf16_to_f32(w)
    checked = 0
    for t in range(4):
        for i, q in enumerate(_decimal_rms(bf16_to_f32(x[t]), w, eps)):
            if near_midpoint(q, 8, 1e-13):
                continue
            n = Fraction(float(bf16_to_f32(np.array([fraction_to_bf16_bits(q)], np.uint16))[0]))
            ref = fraction_to_bf16_bits(n * Fraction(float(wf[i])))
            assert int(out[t, i]) == ref, (t, i)
            checked += 1
    assert checked >= 4 * d - 2


def test_rms_norm_closed_forms():
    d = 64
    w = _bf16(np.linspace(0.5, 1.5, d, dtype=np.float32).astype(np.float32).view(np.uint32)
              .__and__(0xFFFF0000).view(np.float32))
    # constant rows with eps = 0 normalise to +-1: out = +-w
    x = _bf16(np.array([[3.0] * d, [-0.125] * d], np.float32))
    out = oracle.rms_norm(x, w, 0.0)
    assert np.array_equal(out[0], w)
    assert np.array_equal(out[1], w | 0x8000)
    # one nonzero value v: n = sqrt(d) * sign(v) there, 0 elsewhere (d = 64: exactly 8)
    x = np.zeros((1, d), np.float32)
    x[0, 5] = -2.5
    out = oracle.rms_norm(_bf16(x), _bf16(np.ones(d, np.float32)), 0.0)
    assert bf16_to_f32(out)[0, 5] == -8.0 and (np.delete(out[0], 5) == 0).all()
    # scaling a row by a power of two changes nothing (eps = 0)
    rng = np.random.default_rng(8)
    x = _rand_bf16(rng, (5, d))
    x4 = _bf16(bf16_to_f32(x) * np.float32(4.0))
    assert np.array_equal(oracle.rms_norm(x, w, 0.0), oracle.rms_norm(x4, w, 0.0))


# -------------------------------------------------------------------- block
def _tiny_block(seed=0, latent=True, shared=True, norm=True):
    rng = np.random.default_rng(seed)
    N, d_r, d_e, E, F, F_sh, K = 12, 64, 32, 8, 32, 48, 2
    x = _rand_bf16(rng, (N, d_r))
    W = (rng.standard_normal((E, d_r)) * 0.1).astype(np.float32)
    b = (rng.uniform(-0.01, 0.01, E)).astype(np.float32)
    de = d_e if latent else d_r
    w1 = _rand_bf16(rng, (E, F, de), 0.1)
    w3 = _rand_bf16(rng, (E, F, de), 0.1)
    w2 = _rand_bf16(rng, (E, de, F), 0.1)
    kw = dict(act="situ", beta=4.0, lbeta=8.0)
    if latent:
        kw["down_proj"] = _rand_bf16(rng, (d_e, d_r), 0.1)
        kw["up_proj"] = _rand_bf16(rng, (d_r, d_e), 0.1)
        if norm:
            kw["norm_w"] = _bf16(np.float32(0.75) + (rng.integers(0, 64, d_e) / 128.0)
                                 .astype(np.float32))
    if shared:
        kw["shared"] = (_rand_bf16(rng, (F_sh, d_r), 0.1), _rand_bf16(rng, (F_sh, d_r), 0.1),
                        _rand_bf16(rng, (d_r, F_sh), 0.1))
    return (x, W, b, 2, 1, K, 2.5, w1, w3, w2), kw


@pytest.mark.parametrize("latent,shared,norm", [(True, True, True), (True, False, True),
                                                (True, True, False), (False, True, False),
                                                (False, False, False)])
def test_block_equals_per_token_loop(latent, shared, norm):
    """The batched block equals a loop over tokens and their K experts built
    from the separately pinned parts (linear, expert MLP, combine, norm, add)."""
    args, kw = _tiny_block(1, latent, shared, norm)
    out, idx, w, _ = oracle.block_forward(*args, **kw)
    x, W, b, G, TG, K, rs, w1, w3, w2 = args
    a = dict(act=kw["act"], beta=kw["beta"], lbeta=kw["lbeta"])
    for t in range(x.shape[0]):
        xt = x[t:t + 1]
        xe = oracle.linear(xt, kw["down_proj"]) if latent else xt
        ys = np.concatenate([oracle.expert_ffn(xe, w1[e], w3[e], w2[e], **a) for e in idx[t]])
        y = oracle.combine(ys, np.arange(K, dtype=np.int32), w[t], K)
        if latent:
            if norm:
                y = oracle.rms_norm(y, kw["norm_w"], kw.get("eps", 1e-6))
            y = oracle.linear(y, kw["up_proj"])
        if shared:
            y = oracle.add(y, oracle.expert_ffn(xt, *kw["shared"], **a))
        assert np.array_equal(out[t:t + 1], y), t


def test_block_routes_on_the_full_width_input():
    args, kw = _tiny_block(2)
    _, idx, w, _ = oracle.block_forward(*args, **kw)
    x, W, b, G, TG, K, rs = args[:7]
    i2, w2_, _ = oracle.route(x, W, b, G, TG, K, rs)
    assert np.array_equal(idx, i2) and np.array_equal(w, w2_)


def test_block_reductions():
    args, kw = _tiny_block(3)
    x = args[0]
    a = dict(act=kw["act"], beta=kw["beta"], lbeta=kw["lbeta"])
    # a zero up projection leaves only the shared experts' output on x
    kz = dict(kw, up_proj=np.zeros_like(kw["up_proj"]))
    out, *_ = oracle.block_forward(*args, **kz)
    assert np.array_equal(out, oracle.expert_ffn(x, *kw["shared"], **a))
    # zero shared weights leave the routed branch unchanged (adding +0)
    ks = dict(kw, shared=tuple(np.zeros_like(s) for s in kw["shared"]))
    out_s, *_ = oracle.block_forward(*args, **ks)
    kn = dict(kw, shared=None)
    out_n, *_ = oracle.block_forward(*args, **kn)
    assert np.array_equal(out_s & 0x7FFF, out_n & 0x7FFF)  # -0 + +0 = +0
