"""Pins of the CPU reference's moe_infer half: dispatch, expert MLP, combine.

Definitions: "Kimi K3 · Add shared output" moe-forward excerpt (moe_infer) and
"Kimi K3 · Gate features" expert / situ excerpts (KimiBlockSparseMLP,
SituAndMul).  Pins used here:
  * the stable slot sort equals numpy's stable argsort, counts equal bincount;
  * the expert MLP on identity-structured weights reduces to closed forms of
    SiLU and SiTU evaluated with 60-digit decimal arithmetic;
  * the combine on exactly representable inputs equals the exact weighted sum;
  * the sorted moe_infer equals a per-token dense loop bit for bit, and is
    invariant under any reordering of rows inside an expert's segment.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.helpers import (bf16_to_f32, decimal_sigmoid, decimal_tanh, fraction_to_bf16_bits,
                           near_midpoint)


def bf16_bits(v):
    """Nearest-even bf16 bit patterns of fp32 values (finite inputs)."""
    u = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


# ------------------------------------------------------------- rounding
def test_bf16_rounding_points():
    r = oracle.bf16_round_double
    assert r(1.0) == 0x3F80
    assert r(1.0 + 2 ** -8) == 0x3F80            # tie -> even
    assert r(1.0 + 3 * 2 ** -8) == 0x3F82        # tie -> even (up)
    assert r(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81  # just above the tie
    assert r(-(1.0 + 2 ** -8 + 2 ** -40)) == 0xBF81
    assert r(3.0e38) == 0x7F80 or r(3.0e38) == 0x7F62
    assert r(1e39) == 0x7F80
    assert r(0.0) == 0x0000
    # agrees with torch's fp32 -> bf16 conversion on fp32-representable values
    import torch
    v = np.random.default_rng(0).standard_normal(2000).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([r(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, ref)
    got_f = np.array([oracle.bf16_round_float(float(a)) for a in v], np.uint16)
    assert np.array_equal(got_f, ref)


# ------------------------------------------------------------- dispatch
@pytest.mark.parametrize("N,K,E", [(64, 4, 16), (1, 8, 384), (300, 8, 256), (5, 1, 3)])
def test_dispatch_is_stable_counting_sort(N, K, E):
    rng = np.random.default_rng(N + K + E)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    flat = idx.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(pos[perm], np.arange(N * K))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all()


def test_dispatch_all_to_one_expert_and_empty_experts():
    N, K, E = 40, 1, 8
    idx = np.full((N, K), 5, np.int32)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    assert counts.tolist() == [0, 0, 0, 0, 0, 40, 0, 0]
    assert offsets.tolist() == [0, 0, 0, 0, 0, 0, 40, 40, 40]
    assert np.array_equal(perm, np.arange(N))


# ------------------------------------------------------------ expert MLP
POINTS = [0.0, 0.5, -0.5, 1.0, -1.0, 4.0, -4.0, 8.0, -8.0, 30.0, -30.0]


def _identity_expert(d, a=1.0, c=1.0):
    eye = np.eye(d, dtype=np.float32)
    return bf16_bits(eye * a), bf16_bits(eye * c), bf16_bits(eye)


def _row(vals, d):
    r = np.zeros(d, np.float32)
    r[:len(vals)] = vals
    return bf16_bits(r)[None, :]


def _exact_silu_and_mul(g: float, u: float) -> int:
    a = Fraction(g) * decimal_sigmoid(g)
    a16 = fraction_to_bf16_bits(a)
    return fraction_to_bf16_bits(Fraction(float(bf16_to_f32(np.uint16(a16)))) * Fraction(u))


def test_silu_closed_forms():
    d = 64
    w1, w3, w2 = _identity_expert(d)
    x = _row(POINTS, d)
    y = oracle.expert_ffn(x, w1, w3, w2, "silu")
    yv = bf16_to_f32(y[0])
    assert yv[0] == 0.0                          # silu(0) = 0
    assert yv[3] == np.float32(0.73046875)       # bf16(sigmoid(1)) * 1
    assert yv[9] == 900.0                        # silu(30) rounds to 30 in bf16
    assert 0 < yv[10] < 1e-9                     # silu(-30) * (-30): tiny, positive
    for i, g in enumerate(POINTS):
        assert y[0, i] == _exact_silu_and_mul(g, g), (g, yv[i])


def _exact_situ(g: float, u: float, beta: float, lbeta) -> Fraction:
    G, U, B = Fraction(g), Fraction(u), Fraction(beta)
    a = B * decimal_tanh(G / B) * decimal_sigmoid(g)
    up = Fraction(lbeta) * decimal_tanh(U / Fraction(lbeta)) if lbeta else U
    return a * up


@pytest.mark.parametrize("beta,lbeta", [(4.0, 8.0), (1.0, None), (4.0, None), (2.0, 0.5)])
def test_situ_closed_forms(beta, lbeta):
    d = 64
    w1, w3, w2 = _identity_expert(d, a=1.0, c=0.5)   # u = x / 2 exactly
    x = _row(POINTS, d)
    y = oracle.expert_ffn(x, w1, w3, w2, "situ", beta=beta, lbeta=lbeta or 0.0)
    yv = bf16_to_f32(y[0])
    assert yv[0] == 0.0                           # SiTU(0, u) = 0
    for i, g in enumerate(POINTS):
        q = _exact_situ(g, g / 2, beta, lbeta)
        if not near_midpoint(q, 8, 1e-12):
            assert y[0, i] == fraction_to_bf16_bits(q), (g, yv[i], float(q))
    # g -> +inf: beta*tanh(g/beta)*sigmoid(g) -> beta
    up30 = (lbeta * np.tanh(15.0 / lbeta)) if lbeta else 15.0
    assert abs(yv[9] - beta * up30) <= abs(beta * up30) * 2 ** -7
    assert abs(yv[10]) < 1e-9                     # g -> -inf: -> 0


def test_situ_large_beta_tends_to_silu_without_inner_rounding():
    d = 64
    w1, w3, w2 = _identity_expert(d)
    x = _row(POINTS, d)
    y = oracle.expert_ffn(x, w1, w3, w2, "situ", beta=1e30, lbeta=0.0)
    for i, g in enumerate(POINTS):
        q = Fraction(g) * decimal_sigmoid(g) * Fraction(g)
        if not near_midpoint(q, 8, 1e-12):
            assert y[0, i] == fraction_to_bf16_bits(q)


def test_situ_zero_beta_means_one_and_zero_linear_beta_means_unset():
    rng = np.random.default_rng(3)
    d, F = 64, 128
    x = bf16_bits(rng.standard_normal((5, d)).astype(np.float32))
    w1, w3 = (bf16_bits((rng.standard_normal((F, d)) * 0.1).astype(np.float32)) for _ in range(2))
    w2 = bf16_bits((rng.standard_normal((d, F)) * 0.1).astype(np.float32))
    a = oracle.expert_ffn(x, w1, w3, w2, "situ", beta=0.0, lbeta=float("nan"))
    b = oracle.expert_ffn(x, w1, w3, w2, "situ", beta=1.0, lbeta=0.0)
    assert np.array_equal(a, b)


def test_expert_dot_products_exact():
    """g, u and y are the bf16 roundings of exact dot products (linear act: w3
    output fed straight through by a SiTU with huge beta and g constant)."""
    rng = np.random.default_rng(11)
    d, F = 64, 64
    x = bf16_bits(rng.standard_normal((3, d)).astype(np.float32))
    w3 = bf16_bits((rng.standard_normal((F, d)) * 0.1).astype(np.float32))
    w2 = bf16_bits((rng.standard_normal((d, F)) * 0.1).astype(np.float32))
    w1 = bf16_bits(np.zeros((F, d), np.float32))  # g = 0 -> h = 0 -> y = 0
    y0 = oracle.expert_ffn(x, w1, w3, w2, "silu")
    assert (bf16_to_f32(y0) == 0).all()
    # with huge beta SiTU(g,u) = g*sigmoid(g)*u; put g = 40 (sigmoid = 1 in any precision)
    w1 = np.zeros((F, d), np.float32)
    w1[:, 0] = 40.0
    xx = x.copy()
    xx[:, 0] = bf16_bits(np.float32(1.0))
    w1 = bf16_bits(w1)
    y = oracle.expert_ffn(xx, w1, w3, w2, "situ", beta=1e30, lbeta=0.0)
    xf = bf16_to_f32(xx).astype(np.float64)
    for r in range(xx.shape[0]):
        u = [fraction_to_bf16_bits(sum(Fraction(float(a)) * Fraction(float(b))
                                       for a, b in zip(xf[r], bf16_to_f32(w3[f]).astype(np.float64))))
             for f in range(F)]
        uf = bf16_to_f32(np.array(u, np.uint16)).astype(np.float64)
        h = [fraction_to_bf16_bits(Fraction(40.0) * Fraction(float(v))) for v in uf]  # exact-ish
        hf = bf16_to_f32(np.array(h, np.uint16)).astype(np.float64)
        for i in range(d):
            q = sum(Fraction(float(a)) * Fraction(float(b))
                    for a, b in zip(hf, bf16_to_f32(w2[i]).astype(np.float64)))
            if not near_midpoint(q, 8, 1e-12):
                assert y[r, i] == fraction_to_bf16_bits(q)


# --------------------------------------------------------------- combine
def test_combine_exact_on_representable_inputs():
    rng = np.random.default_rng(12)
    N, K, d = 20, 8, 64
    S = N * K
    y = bf16_bits(rng.integers(-100, 100, (S, d)).astype(np.float32))
    w = rng.choice(np.array([0.25, 0.5, 1.0, 2.0], np.float32), size=(N, K))
    pos = rng.permutation(S).astype(np.int32)
    out = oracle.combine(y, pos, w, K)
    yf = bf16_to_f32(y).astype(np.float64)
    for t in range(N):
        exact = sum(yf[pos[t * K + k]] * float(w[t, k]) for k in range(K))
        assert np.array_equal(out[t], bf16_bits(exact.astype(np.float32)))


def test_combine_single_slot_unit_weight_is_a_copy():
    rng = np.random.default_rng(13)
    y = bf16_bits(rng.standard_normal((10, 64)).astype(np.float32))
    pos = rng.permutation(10).astype(np.int32)
    out = oracle.combine(y, pos, np.ones((10, 1), np.float32), 1)
    assert np.array_equal(out, y[pos])


def test_combine_sums_products_in_slot_order():
    """Sequential fp32 sum over k: (2^24 + 1) + 1 rounds twice to 2^24, while the
    exact sum 2^24 + 2 would round to 2^24 + 2 in fp32; both give bf16 2^24, so
    probe with values where the orders differ after bf16 rounding."""
    # p0 = 2^24, p1 = p2 = ... = 1 (K = 9): sequential fp32 stays at 2^24,
    # the exact sum 2^24 + 8 rounds in bf16 to 2^24 as well; use 2^17 steps
    y = bf16_bits(np.array([[2.0 ** 24], [2.0 ** 16], [2.0 ** 16], [2.0 ** 16]], np.float32)
                  * np.ones((1, 64), np.float32))
    w = np.array([[1.0, 1.0, 1.0, 1.0]], np.float32)
    out = oracle.combine(y, np.arange(4, dtype=np.int32), w, 4)
    # fp32: 2^24 + 2^16 is exact; the sum 2^24 + 3*2^16 is exact in fp32; bf16 of it:
    exact = np.float32(2.0 ** 24 + 3 * 2.0 ** 16)
    assert (out[0] == bf16_bits(exact)).all()


# --------------------------------------------------------- whole moe_infer
def _small_problem(N, d, E, F, K, seed, skew=False):
    rng = np.random.default_rng(seed)
    x = bf16_bits(rng.standard_normal((N, d)).astype(np.float32))
    if skew:
        p = np.arange(1, E + 1, dtype=np.float64) ** -1.5
        p /= p.sum()
        idx = np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(N)]).astype(np.int32)
    else:
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
    w = rng.uniform(0.05, 1.0, (N, K)).astype(np.float32)
    w1 = bf16_bits((rng.standard_normal((E, F, d)) * 0.05).astype(np.float32))
    w3 = bf16_bits((rng.standard_normal((E, F, d)) * 0.05).astype(np.float32))
    w2 = bf16_bits((rng.standard_normal((E, d, F)) * 0.05).astype(np.float32))
    return x, idx, w, w1, w3, w2


@pytest.mark.parametrize("N,d,E,F,K,act,skew", [
    (64, 64, 16, 128, 4, "silu", False),
    (33, 128, 12, 64, 3, "situ", False),
    (50, 64, 20, 64, 1, "silu", True),
    (1, 64, 8, 64, 8, "situ", False),
    (40, 64, 32, 64, 6, "silu", True),
])
def test_moe_infer_equals_dense_loop(N, d, E, F, K, act, skew):
    x, idx, w, w1, w3, w2 = _small_problem(N, d, E, F, K, seed=N * 7 + E, skew=skew)
    kw = dict(act=act, beta=4.0, lbeta=8.0) if act == "situ" else dict(act=act)
    a = oracle.moe_infer(x, idx, w, w1, w3, w2, **kw)
    b = oracle.moe_dense(x, idx, w, w1, w3, w2, **kw)
    assert np.array_equal(a, b)


def test_moe_infer_invariant_under_segment_shuffle():
    N, d, E, F, K = 48, 64, 10, 64, 4
    x, idx, w, w1, w3, w2 = _small_problem(N, d, E, F, K, seed=99, skew=True)
    ref = oracle.moe_infer(x, idx, w, w1, w3, w2)
    counts, offsets, perm, pos = oracle.dispatch(idx, E)
    rng = np.random.default_rng(1)
    perm2 = perm.copy()
    for e in range(E):
        seg = perm2[offsets[e]:offsets[e + 1]]
        perm2[offsets[e]:offsets[e + 1]] = rng.permutation(seg)
    pos2 = np.empty_like(pos)
    pos2[perm2] = np.arange(perm2.size, dtype=np.int32)
    xs = oracle.gather(x, perm2, K)
    ys = np.zeros_like(xs)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            ys[a:b] = oracle.expert_ffn(xs[a:b], w1[e], w3[e], w2[e])
    out = oracle.combine(ys, pos2, w, K)
    assert np.array_equal(out, ref)


def test_expert_accumulation_is_exact_across_a_bf16_boundary():
    """g = 2^24 + 2^16 + 62 * 0.5: the exact sum lies above the bf16 midpoint
    2^24 + 2^16, so it rounds up to 2^24 + 2^17; an fp32 running sum would
    drop every 0.5 (half an fp32 ulp at 2^24 or less) and land on the midpoint,
    which rounds to even (2^24)."""
    d = F = 64
    xr = np.ones(d, np.float32)
    xr[0], xr[1] = 2.0 ** 12, 2.0 ** 8
    wr = np.full(d, 0.5, np.float32)
    wr[0], wr[1] = 2.0 ** 12, 2.0 ** 8
    w1 = bf16_bits(np.tile(wr, (F, 1)))
    w2 = bf16_bits(np.eye(d, F, dtype=np.float32))
    y = oracle.expert_ffn(bf16_bits(xr)[None, :], w1, w1, w2, "silu")
    g = 2.0 ** 24 + 2.0 ** 17
    assert (bf16_to_f32(y[0]) == bf16_to_f32(bf16_bits(np.float32(g * g)))).all()
