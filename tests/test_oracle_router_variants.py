"""Pins of the CPU reference's router variants against things other than itself.

Variants: "DeepSeek-V3.2-Exp · Affinities" gate-forward excerpt (Gate.forward):
softmax scoring over all experts in place of the sigmoid, and the group score
taken as the group's largest choice score (amax, the form used there without a
correction bias) in place of the sum of its two largest.  Pins used here:
  * softmax values against a 60-digit decimal evaluation (no libm), including
    logits large enough that exp() without the row maximum would overflow;
  * closed forms: two experts reduce to the logistic of the difference, equal
    logits give 1/E, an exact shift of every logit changes nothing;
  * brute-force enumeration of every group subset and every expert subset
    under both group scores;
  * group maxima against numpy's max.
"""
import itertools
import zlib
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import GROUP_MAX, GROUP_TOP2_SUM, SCORE_SIGMOID, SCORE_SOFTMAX
from tests.helpers import decimal_sigmoid, fraction_to_f32, near_midpoint


def _softmax_scores(L):
    """Scores of the reference with no bias and no groups (the softmax itself)."""
    L = np.asarray(L, np.float32)
    if L.ndim == 1:
        L = L[None]
    return oracle.choice_scores(L, None, 1, 1, score=SCORE_SOFTMAX)


def _decimal_softmax(row, prec=60):
    getcontext().prec = prec
    ex = [Decimal(float(v)).exp() for v in row]
    tot = sum(ex, Decimal(0))
    return [Fraction(e / tot) for e in ex]


# ------------------------------------------------------------- softmax values
@pytest.mark.parametrize("E,scale,shift", [(4, 1.0, 0.0), (16, 2.0, 0.0), (64, 1.0, 0.0),
                                           (256, 1.0, 0.0), (8, 30.0, 0.0), (32, 1.0, 500.0),
                                           (16, 1.0, -800.0)])
def test_softmax_matches_decimal(E, scale, shift):
    """fp32 rounding of the exact softmax (60 digits), except within 1e-13 of a
    rounding midpoint (the double evaluation errs by ~1e-15); shift=500 would
    overflow exp() in double without the row maximum subtracted."""
    rng = np.random.default_rng(zlib.crc32(repr((E, scale, shift)).encode()))
    L = (rng.standard_normal((6, E)) * scale + shift).astype(np.float32)
    s = _softmax_scores(L)
    assert np.isfinite(s).all()
    checked = 0
    for t in range(L.shape[0]):
        for e, q in enumerate(_decimal_softmax(L[t])):
            if near_midpoint(q, 24, 1e-13):
                continue
            assert s[t, e] == fraction_to_f32(q), (t, e)
            checked += 1
    assert checked >= L.size - 2


@pytest.mark.parametrize("a,b", [(0.0, 0.0), (1.0, 0.0), (0.5, -0.25), (3.0, 3.5), (-2.0, 5.0),
                                 (10.0, -10.0), (0.125, 0.0625)])
def test_softmax_of_two_is_logistic_of_difference(a, b):
    """softmax([a, b])[0] = 1 / (1 + exp(b - a)): the correctly rounded logistic
    of the (exact) difference a - b."""
    s = _softmax_scores([a, b])[0]
    for v, d in ((s[0], a - b), (s[1], b - a)):
        q = decimal_sigmoid(d)
        if not near_midpoint(q, 24, 1e-12):
            assert v == fraction_to_f32(q)


@pytest.mark.parametrize("E", [1, 3, 16, 256, 896, 1024])
def test_softmax_equal_logits_is_one_over_e(E):
    s = _softmax_scores(np.full(E, 0.7, np.float32))
    assert (s == fraction_to_f32(Fraction(1, E))).all()


def test_softmax_exact_shift_changes_nothing():
    rng = np.random.default_rng(11)
    # logits on a 2^-10 grid in [-8, 8): adding 1.5 or 64 stays exact in fp32
    L = (rng.integers(-8192, 8192, (50, 64)) / 1024.0).astype(np.float32)
    s = _softmax_scores(L)
    for c in (1.5, 64.0, -3.0):
        Ls = (L.astype(np.float64) + c).astype(np.float32)
        assert np.array_equal(Ls.astype(np.float64) - c, L.astype(np.float64))
        assert np.array_equal(_softmax_scores(Ls), s)


def test_softmax_sums_to_one():
    rng = np.random.default_rng(12)
    L = (rng.standard_normal((200, 256)) * 3).astype(np.float32)
    tot = _softmax_scores(L).astype(np.float64).sum(axis=1)
    # each score carries at most half an fp32 ulp (<= 2^-25 relative) of rounding error
    assert np.abs(tot - 1.0).max() <= 2.0 ** -24


def test_softmax_order_follows_logits():
    """Without bias or groups the chosen experts are the top-K logits (distinct
    logits spaced far enough apart that their fp32 scores stay distinct)."""
    rng = np.random.default_rng(13)
    N, E, K = 300, 64, 8
    L = np.stack([rng.permutation(E) for _ in range(N)]).astype(np.float32) * np.float32(0.05)
    idx, w, _ = oracle.route_from_logits(L, None, 1, 1, K, 1.0, norm=False, score=SCORE_SOFTMAX)
    assert (idx == np.argsort(-L, axis=1, kind="stable")[:, :K]).all()
    s = _softmax_scores(L)
    assert np.array_equal(w, np.take_along_axis(s, idx, axis=1))


def test_softmax_weights_not_renormalised_are_scaled_scores():
    rng = np.random.default_rng(14)
    N, E, K = 100, 32, 6
    L = rng.standard_normal((N, E)).astype(np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 1, 1, K, 2.5, norm=False, score=SCORE_SOFTMAX)
    s = _softmax_scores(L)
    ref = np.take_along_axis(s, idx, axis=1) * np.float32(2.5)
    assert np.array_equal(w, ref)


def test_softmax_all_experts_renormalised_sum_to_route_scale():
    rng = np.random.default_rng(15)
    N, E = 60, 16
    L = rng.standard_normal((N, E)).astype(np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 1, 1, E, 2.5, norm=True, score=SCORE_SOFTMAX)
    assert (np.sort(idx, axis=1) == np.arange(E)).all()
    assert np.allclose(w.astype(np.float64).sum(axis=1), 2.5, rtol=2e-6, atol=0)


def test_softmax_equal_logits_pick_lowest_indices():
    L = np.full((3, 32), -1.25, np.float32)
    idx, w, _ = oracle.route_from_logits(L, None, 4, 2, 6, 1.0, norm=False, score=SCORE_SOFTMAX,
                                         group=GROUP_MAX)
    assert (idx == np.arange(6)).all()
    assert (w == fraction_to_f32(Fraction(1, 32))).all()


# ----------------------------------------------------------- group maxima
@pytest.mark.parametrize("E,G", [(16, 4), (12, 3), (32, 8), (8, 4), (256, 8)])
def test_group_max_is_numpy_max(E, G):
    rng = np.random.default_rng(E * 7 + G)
    c = rng.choice(np.array([-0.5, 0.1, 0.2, 0.3, 0.3, 0.9], np.float32), size=(300, E))
    c[:5] = rng.standard_normal((5, E)).astype(np.float32)
    assert np.array_equal(oracle.group_scores(c, G, GROUP_MAX), c.reshape(-1, G, E // G).max(axis=2))


# ------------------------------------------------------------- brute force
SHAPES = [  # (E, G, TG, K)
    (16, 4, 2, 4),
    (12, 3, 2, 3),
    (8, 2, 1, 2),
    (16, 8, 3, 5),
    (10, 5, 5, 3),
    (8, 1, 1, 3),
]


def _rank(vals):
    N, M = vals.shape
    order = np.lexsort((np.broadcast_to(np.arange(M), (N, M)), -vals.astype(np.float64)), axis=1)
    r = np.empty_like(order)
    np.put_along_axis(r, order, np.broadcast_to(np.arange(M), (N, M)), axis=1)
    return r


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("score,group", [(SCORE_SOFTMAX, GROUP_TOP2_SUM),
                                         (SCORE_SIGMOID, GROUP_MAX),
                                         (SCORE_SOFTMAX, GROUP_MAX)])
@pytest.mark.parametrize("ties", [False, True])
def test_variant_selection_brute_force(shape, score, group, ties):
    """Every group subset and expert subset enumerated (2000 tokens per case):
    kept groups and chosen experts reach the largest score sum and rank before
    everything left out; weights are the chosen scores, renormalised."""
    E, G, TG, K = shape
    rng = np.random.default_rng(zlib.crc32(repr((shape, score, group, ties)).encode()))
    N = 2000
    if ties:
        L = rng.choice(np.array([-1.0, -0.5, 0.0, 0.25, 0.5, 1.0], np.float32), size=(N, E))
        b = rng.choice(np.array([0.0, 0.125, -0.125], np.float32), size=E)
    else:
        L = rng.standard_normal((N, E)).astype(np.float32)
        b = rng.uniform(-0.01, 0.01, E).astype(np.float32)
    idx, w, _ = oracle.route_from_logits(L, b, G, TG, K, 1.0, norm=True, score=score, group=group)
    # unbiased scores, pinned on their own by the softmax and sigmoid tests
    s = oracle.choice_scores(L, None, 1, 1, score=score)
    c = s + b
    gsz = E // G
    rows = np.arange(N)[:, None]
    if G > 1:
        cg = c.reshape(N, G, gsz)
        if group == GROUP_MAX:
            gs = cg.max(axis=2)
        else:
            pairs = np.array(list(itertools.combinations(range(gsz), 2)))
            gs = (cg[:, :, pairs[:, 0]] + cg[:, :, pairs[:, 1]]).max(axis=2)
        cs = oracle.choice_scores(L, b, G, TG, score=score, group=group)
        kept = np.isfinite(cs).reshape(N, G, gsz).all(axis=2)
        assert (kept.sum(axis=1) == TG).all()
        subs = np.array(list(itertools.combinations(range(G), TG)))
        best = gs.astype(np.float64)[:, subs].sum(axis=2).max(axis=1)
        assert np.array_equal(np.where(kept, gs.astype(np.float64), 0.0).sum(axis=1), best)
        rg = _rank(gs)
        assert (np.where(kept, rg, -1).max(axis=1) < np.where(~kept, rg, G).min(axis=1)).all()
        cand = np.repeat(kept, gsz, axis=1)
    else:
        cand = np.ones((N, E), bool)
    chosen = np.zeros((N, E), bool)
    chosen[rows, idx] = True
    assert (chosen.sum(axis=1) == K).all()
    assert not (chosen & ~cand).any()
    cm = np.where(cand, c.astype(np.float64), -np.inf)
    subs = np.array(list(itertools.combinations(range(E), K)))
    assert np.array_equal(np.where(chosen, cm, 0.0).sum(axis=1), cm[:, subs].sum(axis=2).max(axis=1))
    rc = _rank(np.where(cand, c, -np.inf))
    assert (np.diff(rc[rows, idx], axis=1) > 0).all()
    assert (np.where(chosen, rc, -1).max(axis=1) < np.where(cand & ~chosen, rc, E).min(axis=1)).all()
    sw = np.take_along_axis(s, idx, axis=1).astype(np.float64)
    ref = sw / (sw.sum(axis=1, keepdims=True) + 1e-20)
    assert np.allclose(w, ref, rtol=1e-6, atol=0)
