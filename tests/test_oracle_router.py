"""Pins of the CPU reference's router against things other than itself.

Router definition: "Kimi K2 · Affinities" gate-forward excerpt (MoEGate.forward,
noaux_tc) and "DeepSeek-V3.2-Exp · Affinities" gate-forward excerpt
(Gate.forward).  Pins used here:
  * exact rational arithmetic for the gate logits and the sigmoid;
  * brute-force enumeration of every group subset and every expert subset on
    tiny shapes (the chosen set must maximise the score sum and every chosen
    member must rank before every unchosen one);
  * special cases that reduce to a plain sort or to closed forms;
  * invariants of the weights.
"""
import itertools
import zlib

import numpy as np
import pytest

import oracle
from tests.helpers import (decimal_sigmoid, exact_f32_dot, fraction_to_f32, near_midpoint)

# --------------------------------------------------------------- logits
def test_gate_logits_exact_rounding():
    """Each logit is the correctly rounded fp32 of the exact dot product."""
    rng = np.random.default_rng(7)
    N, d, E = 6, 256, 16
    x = (rng.standard_normal((N, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    W = (rng.standard_normal((E, d)) * 0.02).astype(np.float32)
    L = oracle.gate_logits(x, W)
    checked = 0
    for t in range(N):
        for e in range(E):
            q = exact_f32_dot(x[t], W[e])
            if near_midpoint(q, 24, 1e-12):
                continue
            assert L[t, e] == fraction_to_f32(q), (t, e)
            checked += 1
    assert checked >= N * E - 2


def test_gate_logits_zero_and_sign():
    x = np.zeros((2, 64), np.uint16)
    W = np.ones((3, 64), np.float32)
    assert (oracle.gate_logits(x, W) == 0).all()
    x1 = np.full((1, 64), 0x3F80, np.uint16)  # bf16 1.0
    W1 = np.stack([np.full(64, 0.5, np.float32), np.full(64, -0.25, np.float32)])
    assert oracle.gate_logits(x1, W1).tolist() == [[32.0, -16.0]]


# --------------------------------------------------------------- sigmoid
@pytest.mark.parametrize("L", [0.0, 1.0, -1.0, 0.5, -3.25, 7.0, 12.5, -20.0, 1e-3, 2.0 ** -20])
def test_sigmoid_correctly_rounded(L):
    q = decimal_sigmoid(L)
    if not near_midpoint(q, 24, 1e-12):
        assert np.float32(oracle.sigmoid(L)) == fraction_to_f32(q)


def test_sigmoid_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.sigmoid(200.0) == 1.0
    assert oracle.sigmoid(-200.0) == 0.0
    xs = np.linspace(-6, 6, 2001).astype(np.float32)
    s = np.array([oracle.sigmoid(float(v)) for v in xs], np.float32)
    assert (np.diff(s) >= 0).all()
    # sigmoid(-L) = 1 - sigmoid(L) up to one fp32 rounding of each side
    for v in xs[::97]:
        a, b = oracle.sigmoid(float(v)), oracle.sigmoid(float(-v))
        assert abs((a + b) - 1.0) <= 2 ** -23


# ----------------------------------------------------------- brute force
def _random_logits(N, E, mode, rng):
    if mode == "ties":
        # few distinct values: exact ties inside and across groups are common
        return rng.choice(np.array([-1.0, -0.5, 0.0, 0.25, 0.5, 1.0], np.float32), size=(N, E))
    return rng.standard_normal((N, E)).astype(np.float32)


def _random_bias(E, mode, rng):
    if mode == "none":
        return None
    if mode == "ties":
        return rng.choice(np.array([0.0, 0.125, -0.125], np.float32), size=E)
    return rng.uniform(-0.01, 0.01, E).astype(np.float32)


def _sigmoid_f32(L):
    f = np.vectorize(lambda v: oracle.sigmoid(float(v)), otypes=[np.float32])
    return f(L)


SHAPES = [  # (E, G, TG, K)
    (16, 4, 2, 4),   # the tiny workload's routing shape
    (16, 1, 1, 4),
    (12, 3, 2, 3),
    (8, 2, 1, 2),
    (16, 8, 3, 5),
    (6, 1, 1, 6),
    (10, 5, 5, 3),
]


def _rank(vals):
    """Position of each entry in the order (value descending, index ascending)."""
    N, M = vals.shape
    order = np.lexsort((np.broadcast_to(np.arange(M), (N, M)), -vals.astype(np.float64)), axis=1)
    r = np.empty_like(order)
    np.put_along_axis(r, order, np.broadcast_to(np.arange(M), (N, M)), axis=1)
    return r


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("lmode,bmode", [("normal", "unif"), ("ties", "ties"), ("ties", "none"),
                                         ("normal", "none")])
def test_selection_brute_force(shape, lmode, bmode):
    """Enumerate every group subset and every expert subset (2500 tokens per
    case, 10^4 per shape): the reference's kept groups and chosen experts must
    reach the largest score sum, and rank before every member left out."""
    E, G, TG, K = shape
    rng = np.random.default_rng(zlib.crc32(repr((shape, lmode, bmode)).encode()))
    N = 2500
    L = _random_logits(N, E, lmode, rng)
    b = _random_bias(E, bmode, rng)
    idx, w, _ = oracle.route_from_logits(L, b, G, TG, K, 1.0)
    s = _sigmoid_f32(L)
    c = s + (b if b is not None else np.float32(0))
    assert c.dtype == np.float32
    gsz = E // G
    rows = np.arange(N)[:, None]
    if G > 1:
        pairs = np.array(list(itertools.combinations(range(gsz), 2)))
        cg = c.reshape(N, G, gsz)
        gs = (cg[:, :, pairs[:, 0]] + cg[:, :, pairs[:, 1]]).max(axis=2)  # fp32 pair sums
        assert np.array_equal(gs, oracle.group_scores(c, G))
        kept_mask = np.isfinite(oracle.choice_scores(L, b, G, TG)).reshape(N, G, gsz).all(axis=2)
        assert (kept_mask.sum(axis=1) == TG).all()
        subs = np.array(list(itertools.combinations(range(G), TG)))
        sums = gs.astype(np.float64)[:, subs].sum(axis=2)              # [N, C]
        kept_sum = np.where(kept_mask, gs.astype(np.float64), 0.0).sum(axis=1)
        assert np.array_equal(kept_sum, sums.max(axis=1))
        rg = _rank(gs)
        max_kept = np.where(kept_mask, rg, -1).max(axis=1)
        min_drop = np.where(~kept_mask, rg, G).min(axis=1)
        assert (max_kept < min_drop).all()
        cand = np.repeat(kept_mask, gsz, axis=1)
    else:
        cand = np.ones((N, E), bool)
    chosen = np.zeros((N, E), bool)
    chosen[rows, idx] = True
    assert (chosen.sum(axis=1) == K).all(), "indices must be distinct"
    assert not (chosen & ~cand).any(), "an index outside the kept groups"
    cm = np.where(cand, c.astype(np.float64), -np.inf)
    subs = np.array(list(itertools.combinations(range(E), K)))
    best = cm[:, subs].sum(axis=2).max(axis=1)
    got = np.where(chosen, cm, 0.0).sum(axis=1)
    assert np.array_equal(got, best)
    rc = _rank(np.where(cand, c, -np.inf))
    assert (np.where(chosen, rc, -1).max(axis=1) < np.where(cand & ~chosen, rc, E).min(axis=1)).all()
    # emitted in (c desc, index asc) order
    assert (np.diff(rc[rows, idx], axis=1) > 0).all()


@pytest.mark.parametrize("E,G", [(16, 4), (12, 3), (32, 8), (8, 4)])
def test_group_scores_best_pair(E, G):
    rng = np.random.default_rng(E * 31 + G)
    c = rng.choice(np.array([0.1, 0.2, 0.3, 0.3, 0.9], np.float32), size=(400, E))
    gs = oracle.group_scores(c, G)
    gsz = E // G
    for t in range(c.shape[0]):
        for g in range(G):
            blk = c[t, g * gsz:(g + 1) * gsz]
            ref = max(np.float32(blk[i] + blk[j]) for i in range(gsz) for j in range(i + 1, gsz))
            assert gs[t, g] == ref


# ----------------------------------------------------------- special cases
def test_no_groups_no_bias_is_plain_topk_of_logits():
    rng = np.random.default_rng(5)
    N, E, K = 300, 64, 8
    # distinct logits spaced well apart, inside the range where fp32 sigmoid is strictly increasing
    L = np.stack([rng.permutation(E) for _ in range(N)]).astype(np.float32) * np.float32(0.05) - 1.5
    idx, _, _ = oracle.route_from_logits(L, None, 1, 1, K, 1.0)
    ref = np.argsort(-L, axis=1, kind="stable")[:, :K]
    assert (idx == ref).all()


def test_all_experts_chosen_weights_are_normalised_scores():
    rng = np.random.default_rng(6)
    N, E = 50, 8
    L = rng.standard_normal((N, E)).astype(np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 1, 1, E, 2.5)
    s = _sigmoid_f32(L).astype(np.float64)
    for t in range(N):
        assert sorted(idx[t].tolist()) == list(range(E))
        ref = 2.5 * s[t, idx[t]] / s[t].sum()
        assert np.allclose(w[t], ref, rtol=4e-7, atol=0)


def test_all_equal_logits_pick_lowest_indices():
    L = np.full((4, 16), 0.3, np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 4, 2, 4, 2.5)
    assert (idx == np.array([0, 1, 2, 3])).all()
    assert (w == np.float32(2.5) * (np.float32(1) / np.float32(4))).all() or np.allclose(w, 0.625)


def test_large_bias_forces_expert():
    rng = np.random.default_rng(8)
    L = rng.standard_normal((200, 16)).astype(np.float32)
    b = np.zeros(16, np.float32)
    b[11] = 2.0
    idx, _, _ = oracle.route_from_logits(L, b, 4, 2, 4, 1.0)
    assert (idx[:, 0] == 11).all()


def test_bias_steers_choice_not_weights():
    """Weights are the unbiased scores of the chosen experts."""
    rng = np.random.default_rng(9)
    L = rng.standard_normal((100, 16)).astype(np.float32)
    b = rng.uniform(-0.3, 0.3, 16).astype(np.float32)
    idx, w, _ = oracle.route_from_logits(L, b, 1, 1, 1, 1.0)  # K=1: no renormalisation
    s = _sigmoid_f32(L)
    assert (w[:, 0] == s[np.arange(100), idx[:, 0]]).all()


def test_single_expert_not_renormalised_but_scaled():
    L = np.array([[0.0, 3.0, -1.0, 0.5]], np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 1, 1, 1, 2.827)
    assert idx[0, 0] == 1
    assert w[0, 0] == np.float32(np.float32(oracle.sigmoid(3.0)) * np.float32(2.827))


def test_no_norm_flag():
    L = np.array([[0.0, 3.0, -1.0, 0.5]], np.float32)
    _, w, _ = oracle.route_from_logits(L, None, 1, 1, 2, 1.0, norm=False)
    assert w[0].tolist() == [np.float32(oracle.sigmoid(3.0)), np.float32(oracle.sigmoid(0.5))]


# --------------------------------------------------------------- invariants
@pytest.mark.parametrize("E,G,TG,K,rs", [(16, 4, 2, 4, 2.5), (256, 8, 4, 8, 2.5),
                                          (384, 1, 1, 8, 2.827), (896, 1, 1, 8, 2.827)])
def test_weight_invariants(E, G, TG, K, rs):
    rng = np.random.default_rng(E)
    N = 64
    L = (rng.standard_normal((N, E)) * 1.7).astype(np.float32)
    b = rng.uniform(-0.01, 0.01, E).astype(np.float32)
    idx, w, margin = oracle.route_from_logits(L, b, G, TG, K, rs)
    s = _sigmoid_f32(L)
    for t in range(N):
        assert len(set(idx[t].tolist())) == K
        # sum of weights is the route scale up to K roundings
        assert abs(float(w[t].astype(np.float64).sum()) - rs) <= K * rs * 2 ** -22
        # ratios are the ratios of the unbiased scores
        st = s[t, idx[t]].astype(np.float64)
        r = (w[t].astype(np.float64) / w[t, 0]) / (st / st[0])
        assert np.allclose(r, 1.0, rtol=2 * 2 ** -23 * 3, atol=0)
        if G > 1:
            gsz = E // G
            assert len({int(e) // gsz for e in idx[t]}) <= TG
    assert (margin >= 0).all()


def test_margin_is_gap_at_the_boundary():
    rng = np.random.default_rng(10)
    N, E, K = 100, 32, 4
    L = rng.standard_normal((N, E)).astype(np.float32)
    idx, _, margin = oracle.route_from_logits(L, None, 1, 1, K, 1.0)
    c = np.sort(_sigmoid_f32(L).astype(np.float64), axis=1)[:, ::-1]
    assert np.array_equal(margin, c[:, K - 1] - c[:, K])


def test_gate_logits_accumulation_is_exact():
    """2^24 + 63 * 0.5 = 2^24 + 31.5 rounds to 2^24 + 32 in fp32; an fp32 running
    sum would lose every 0.5 and return 2^24."""
    d = 64
    x = np.full((1, d), 0x3F80, np.uint16)     # bf16 1.0
    x[0, 0] = 0x4580                          # bf16 4096
    W = np.full((1, d), 0.5, np.float32)
    W[0, 0] = 4096.0
    assert oracle.gate_logits(x, W)[0, 0] == np.float32(2.0 ** 24 + 32)
