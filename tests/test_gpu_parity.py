"""Parity of every C-ABI entry point with the CPU reference, on the GPU.

Both sides get the same seeded inputs (host twin -> reference, device twin or a
copy of the host array -> CUDA library).  Bars:
  * selection from supplied logits: indices and weights bit-exact;
  * end-to-end routing: index sets equal for tokens whose biased-score margin
    exceeds 1e-5, weights within 1e-5 relative;
  * dispatch: counts, offsets, perm, pos exact; gathered rows bitwise;
  * combine: bitwise;
  * expert MLP and layer output: relative L2 <= 2e-2 in bf16.
Full-size workloads are checked on sampled tokens / experts the reference can
compute in seconds; the kernels always run at the full size.
"""
import numpy as np
import pytest

import oracle
import synth
from synth.workloads import WORKLOADS, host_inputs, host_expert, scaled
from tests.gpu_util import (MARGIN, REL_L2_OUT, W_REL, check_bf16_outputs, dev_bf16, host_bf16,
                            oracle_layer_tokens, random_topk, rel_l2, ulp_diff, ulp_stats)

pytestmark = pytest.mark.gpu

ALL = list(WORKLOADS)


@pytest.fixture(scope="module")
def moe():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import moe_routing_expert_fp32_b200 as m
    m.lib()
    oracle.set_threads(0)
    return m


def rcfg(m, wl):
    return m.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)


def acfg(m, wl):
    return m.ActConfig(wl.act, wl.beta, wl.lbeta)


# ------------------------------------------------------ selection from logits
def _logits(wl, N, mode):
    if mode == "normal":
        return synth.host_normal_f32(11, 9, (N, wl.E), 1.7)
    # exact ties: few distinct logits
    raw = synth.host_raw(11, 9, N * wl.E).reshape(N, wl.E)
    return (np.float32(-1.0) + np.float32(0.25) * (raw % 9).astype(np.float32)).astype(np.float32)


@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("mode", ["normal", "ties"])
def test_route_from_logits_bit_exact(moe, name, mode):
    import torch
    wl = WORKLOADS[name]
    N = wl.N
    L = _logits(wl, N, mode)
    b = host_inputs(scaled(wl, N=1))["bias"]
    if mode == "ties":
        b = np.round(b * 200).astype(np.float32) / np.float32(200)  # few distinct bias values
    idx_r, w_r, _ = oracle.route_from_logits(L, b, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    idx_g, w_g = moe.route_from_logits(torch.from_numpy(L).cuda(), torch.from_numpy(b).cuda(),
                                       rcfg(moe, wl))
    assert np.array_equal(idx_g.cpu().numpy(), idx_r)
    assert np.array_equal(w_g.cpu().numpy().view(np.uint32), w_r.view(np.uint32))


@pytest.mark.parametrize("E,G,TG,K,norm", [(16, 4, 2, 4, True), (8, 1, 1, 1, True),
                                           (64, 8, 8, 16, True), (1024, 32, 3, 16, True),
                                           (12, 3, 2, 6, False), (6, 1, 1, 6, True)])
def test_route_from_logits_shapes(moe, E, G, TG, K, norm):
    import torch
    rng = np.random.default_rng(E * 100 + K)
    N = 777
    L = rng.choice(np.array([-0.5, 0.0, 0.5, 1.0], np.float32), size=(N, E))
    L[: N // 2] = rng.standard_normal((N // 2, E)).astype(np.float32)
    b = rng.choice(np.array([0.0, 0.01, -0.01], np.float32), size=E)
    idx_r, w_r, _ = oracle.route_from_logits(L, b, G, TG, K, 2.0, norm)
    cfg = moe.RouteConfig(E, G, TG, K, 2.0, norm)
    idx_g, w_g = moe.route_from_logits(torch.from_numpy(L).cuda(), torch.from_numpy(b).cuda(), cfg)
    assert np.array_equal(idx_g.cpu().numpy(), idx_r)
    assert np.array_equal(w_g.cpu().numpy().view(np.uint32), w_r.view(np.uint32))
    # no bias
    idx_r, w_r, _ = oracle.route_from_logits(L, None, G, TG, K, 2.0, norm)
    idx_g, w_g = moe.route_from_logits(torch.from_numpy(L).cuda(), None, cfg)
    assert np.array_equal(idx_g.cpu().numpy(), idx_r)
    assert np.array_equal(w_g.cpu().numpy().view(np.uint32), w_r.view(np.uint32))


_SCORE = {"sigmoid": oracle.SCORE_SIGMOID, "softmax": oracle.SCORE_SOFTMAX}
_GROUP = {"top2_sum": oracle.GROUP_TOP2_SUM, "max": oracle.GROUP_MAX}


@pytest.mark.parametrize("score,group", [("softmax", "top2_sum"), ("sigmoid", "max"),
                                         ("softmax", "max")])
@pytest.mark.parametrize("E,G,TG,K,norm", [(256, 8, 4, 8, False), (256, 8, 4, 8, True),
                                           (1024, 32, 3, 16, True), (896, 1, 1, 8, True),
                                           (16, 4, 2, 4, False), (6, 1, 1, 6, True)])
def test_route_variants_bit_exact(moe, score, group, E, G, TG, K, norm):
    """Softmax scoring and group-max scores: indices and weights bit-exact from
    the same logits, with and without bias, ties included."""
    import torch
    rng = np.random.default_rng(E * 1000 + K + 7 * len(score + group))
    N = 777
    L = rng.choice(np.array([-0.5, 0.0, 0.5, 1.0], np.float32), size=(N, E))
    L[: N // 2] = (rng.standard_normal((N // 2, E)) * 2).astype(np.float32)
    L[: 8] += np.float32(300.0)  # large logits: softmax must subtract the row maximum
    b = rng.choice(np.array([0.0, 0.001, -0.001], np.float32), size=E)
    cfg = moe.RouteConfig(E, G, TG, K, 2.0, norm, score_func=score, group_score=group)
    for bias in (b, None):
        idx_r, w_r, _ = oracle.route_from_logits(L, bias, G, TG, K, 2.0, norm, score=_SCORE[score],
                                                 group=_GROUP[group])
        idx_g, w_g = moe.route_from_logits(torch.from_numpy(L).cuda(),
                                           None if bias is None else torch.from_numpy(bias).cuda(),
                                           cfg)
        assert np.array_equal(idx_g.cpu().numpy(), idx_r)
        assert np.array_equal(w_g.cpu().numpy().view(np.uint32), w_r.view(np.uint32))


# ----------------------------------------------------------- routing end to end
def _check_routing(idx_g, w_g, idx_r, w_r, margin):
    ok = margin > MARGIN
    assert ok.mean() > 0.5
    for t in np.nonzero(ok)[0]:
        assert set(idx_g[t].tolist()) == set(idx_r[t].tolist()), t
        og = dict(zip(idx_g[t].tolist(), w_g[t].tolist()))
        for e, wr in zip(idx_r[t].tolist(), w_r[t].tolist()):
            assert abs(og[e] - wr) <= W_REL * abs(wr), (t, e, og[e], wr)
    return int((~ok).sum())


@pytest.mark.parametrize("name", ALL)
def test_route_end_to_end(moe, name):
    import torch
    wl = WORKLOADS[name]
    inp = host_inputs(wl)
    x, W, b = inp["x"], inp["W"], inp["bias"]
    idx_g, w_g = moe.route(dev_bf16(x), torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda(),
                           rcfg(moe, wl))
    idx_g, w_g = idx_g.cpu().numpy(), w_g.cpu().numpy()
    rows = np.arange(wl.N)
    if wl.N > 1024:  # the reference routes a sample of the batch
        rows = np.unique(np.concatenate([np.arange(256), np.arange(wl.N - 256, wl.N),
                                         np.random.default_rng(0).choice(wl.N, 512, False)]))
    idx_r, w_r, margin = oracle.route(np.ascontiguousarray(x[rows]), W, b, wl.G, wl.TG, wl.K,
                                      wl.route_scale, wl.norm)
    n_low = _check_routing(idx_g[rows], w_g[rows], idx_r, w_r, margin)
    print(f"{name}: {len(rows)} tokens checked, {n_low} at or below the margin")


@pytest.mark.parametrize("score,group", [("softmax", "max"), ("sigmoid", "max")])
def test_route_variants_end_to_end(moe, score, group):
    """The gate GEMM followed by a variant selection, at the 256-expert decode shape."""
    import torch
    wl = WORKLOADS["dsv32_decode"]
    inp = host_inputs(wl)
    x, W = inp["x"], inp["W"]
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, score == "sigmoid",
                          score_func=score, group_score=group)
    idx_g, w_g = moe.route(dev_bf16(x), torch.from_numpy(W).cuda(), None, cfg)
    idx_r, w_r, margin = oracle.route(x, W, None, wl.G, wl.TG, wl.K, wl.route_scale,
                                      score == "sigmoid", score=_SCORE[score], group=_GROUP[group])
    n_low = _check_routing(idx_g.cpu().numpy(), w_g.cpu().numpy(), idx_r, w_r, margin)
    print(f"{score}/{group}: {wl.N} tokens checked, {n_low} at or below the margin")


# ------------------------------------------------------------------ dispatch
def _dispatch_case(moe, N, K, E, d, idx):
    import torch
    x = synth.host_normal_bf16(3, 1, (N, d), 1.0)
    c_g, o_g, p_g, q_g, xs_g = moe.dispatch(torch.from_numpy(idx).cuda(), dev_bf16(x), E)
    c_r, o_r, p_r, q_r = oracle.dispatch(idx, E)
    assert np.array_equal(c_g.cpu().numpy(), c_r)
    assert np.array_equal(o_g.cpu().numpy(), o_r)
    assert np.array_equal(p_g.cpu().numpy(), p_r)
    assert np.array_equal(q_g.cpu().numpy(), q_r)
    S = N * K
    rows = np.arange(S) if S <= 4096 else np.unique(
        np.concatenate([np.arange(1024), np.arange(S - 1024, S),
                        np.random.default_rng(1).choice(S, 2048, False)]))
    xs_rows = host_bf16(xs_g[torch.from_numpy(rows).cuda()])
    assert np.array_equal(xs_rows, x[p_r[rows] // K])


@pytest.mark.parametrize("name", ALL)
def test_dispatch(moe, name):
    wl = WORKLOADS[name]
    rng = np.random.default_rng(21)
    idx = random_topk(wl.N, wl.K, wl.E, rng, skew=1.2 if wl.skew else 0.0)
    _dispatch_case(moe, wl.N, wl.K, wl.E, wl.d_e, idx)


# (40000, 8, 64): 320 000 slots make 313 chunks of 1024, more than the 256
# that the scan keeps in registers, so its looping form runs.  Up to 4096
# slots the one-block sort runs: (1024, 4, 1024) is its largest case,
# (4097, 1, 256) just outside it
@pytest.mark.parametrize("N,K,E", [(1, 8, 384), (1000, 1, 16), (333, 3, 7), (5000, 16, 1024),
                                   (40000, 8, 64), (1024, 4, 256), (1024, 4, 1024),
                                   (4097, 1, 256), (512, 1, 1), (1, 1, 1)])
def test_dispatch_edge_shapes(moe, N, K, E):
    rng = np.random.default_rng(N + K + E)
    _dispatch_case(moe, N, K, E, 128, random_topk(N, K, E, rng, skew=1.5))


def test_dispatch_all_slots_one_expert(moe):
    N, K, E = 3000, 1, 64
    _dispatch_case(moe, N, K, E, 256, np.full((N, K), 17, np.int32))


def test_dispatch_out_of_range_index_is_reported_not_faulted(moe):
    import torch
    N, K, E, d = 64, 4, 16, 128
    idx = random_topk(N, K, E, np.random.default_rng(5))
    idx[3, 1] = E + 5
    idx[40, 0] = -2
    ws = moe.workspace(1 << 16)
    c, o, p, q, xs = moe.dispatch(torch.from_numpy(idx).cuda(), dev_bf16(
        synth.host_normal_bf16(0, 1, (N, d), 1.0)), E, ws=ws)
    assert moe.get_status(ws) == -7
    assert int(o[-1].item()) == N * K - 2
    assert q[3 * K + 1].item() == -1 and q[40 * K].item() == -1


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("name", ALL)
def test_combine_bitwise(moe, name):
    import torch
    wl = WORKLOADS[name]
    N, K, d = wl.N, wl.K, wl.d_e
    S = N * K
    y = synth.host_normal_bf16(4, 10, (S, d), 0.05)
    pos = np.random.default_rng(2).permutation(S).astype(np.int32)
    w = synth.host_uniform_f32(4, 11, (N, K), 0.0, 0.7)
    out_g = host_bf16(moe.combine(dev_bf16(y), torch.from_numpy(pos).cuda(),
                                  torch.from_numpy(w).cuda()))
    out_r = oracle.combine(y, pos, w, K)
    assert np.array_equal(out_g, out_r)


# ------------------------------------------- slot-order scatter + combine
@pytest.mark.parametrize("name", ALL)
def test_slot_order_scatter_and_combine(moe, name):
    """moe_expert_ffn_to_slots writes the MLP output of sorted row j to row
    perm[j] (the page's new_x[idxs] = outs): it must equal moe_expert_ffn's
    sorted output scattered by perm, bit for bit; moe_combine reading it in
    slot order (pos NULL) must equal the combine through pos bit for bit, and
    the reference combine of the same rows bit for bit (all tokens, or 2048
    sampled ones of the large batches)."""
    import torch
    wl = WORKLOADS[name]
    dev = synth.workloads.dev_inputs(wl)
    act = acfg(moe, wl)
    x_e = dev["x_e"] if wl.latent else dev["x"]
    idx, w = moe.route(dev["x"], dev["W"], dev["bias"], rcfg(moe, wl))
    counts, offsets, perm, pos, xs = moe.dispatch(idx, x_e, wl.E)
    y = moe.expert_ffn(xs, offsets, dev["w1"], dev["w3"], dev["w2"], act)
    ys = moe.expert_ffn_to_slots(xs, offsets, perm, dev["w1"], dev["w3"], dev["w2"], act)
    assert torch.equal(ys[perm.long()].view(torch.int16), y.view(torch.int16))
    out_s = moe.combine(ys, None, w)
    out_p = moe.combine(y, pos, w)
    assert torch.equal(out_s.view(torch.int16), out_p.view(torch.int16))
    toks = np.arange(wl.N) if wl.N <= 4096 else np.sort(
        np.random.default_rng(11).choice(wl.N, 2048, replace=False))
    rows = (toks[:, None] * wl.K + np.arange(wl.K)[None, :]).ravel()
    y_rows = host_bf16(ys[torch.from_numpy(rows).cuda()])
    w_rows = np.ascontiguousarray(w.cpu().numpy()[toks])
    ref = oracle.combine(y_rows, np.arange(rows.size, dtype=np.int32), w_rows, wl.K)
    assert np.array_equal(host_bf16(out_s)[toks], ref)


# ------------------------------------------------------------- expert MLP
def _expert_case(moe, wl, counts, sample_experts, rows_per_expert=48, seed=5):
    """Run moe_expert_ffn on all segments; check sampled experts' rows."""
    import torch
    E, F, d = wl.E, wl.F, wl.d_e
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    S = int(offsets[-1])
    xs_d = synth.dev_normal_bf16(torch.empty((S, d), dtype=torch.bfloat16, device="cuda"),
                                 seed, 12, 1.0)
    dev = synth.workloads.dev_inputs(wl, experts=True)
    y_d = moe.expert_ffn(xs_d, torch.from_numpy(offsets).cuda(), dev["w1"], dev["w3"], dev["w2"],
                         acfg(moe, wl))
    torch.cuda.synchronize()
    worst = 0.0
    got_all, ref_all = [], []
    for e in sample_experts:
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        n = b - a
        if n <= rows_per_expert:
            rows = np.arange(a, b)
        else:  # first tile, a tile boundary, the ragged tail
            cand = [a, a + 1, a + 127, a + 128, a + 129, b - 2, b - 1]
            cand += list(np.random.default_rng(e).choice(np.arange(a, b), rows_per_expert - 7))
            rows = np.unique(np.clip(cand, a, b - 1))
        xs_rows = np.stack([synth.host_normal_bf16(seed, 12, (d,), 1.0, start=int(r) * d)
                            for r in rows])
        w1, w3, w2 = host_expert(wl, e)
        y_r = oracle.expert_ffn(xs_rows, w1, w3, w2, wl.act, wl.beta, wl.lbeta)
        y_g = host_bf16(y_d[torch.from_numpy(rows).cuda()])
        err = rel_l2(y_g, y_r)
        print(f"expert {wl.name} {e}: rows {len(rows)}/{n} rel_l2 {err:.2e} "
              f"ulp {ulp_stats(y_g, y_r)}")
        assert err <= REL_L2_OUT
        worst = max(worst, err)
        got_all.append(y_g)
        ref_all.append(y_r)
    if got_all:
        check_bf16_outputs(np.concatenate(got_all), np.concatenate(ref_all),
                           long_dots=max(d, F) > 512, what=f"expert MLP {wl.name}")
    return worst


@pytest.mark.parametrize("name", ALL)
def test_expert_ffn(moe, name):
    wl = WORKLOADS[name]
    rng = np.random.default_rng(31)
    idx = random_topk(wl.N, wl.K, wl.E, rng, skew=1.2 if wl.skew else 0.0)
    counts = np.bincount(idx.ravel(), minlength=wl.E)
    order = np.argsort(-counts, kind="stable")
    nz = order[counts[order] > 0]
    sample = sorted({int(nz[0]), int(nz[len(nz) // 2]), int(nz[-1])})
    if wl.E <= 16:
        sample = list(range(wl.E))
    _expert_case(moe, wl, counts, sample)


def test_expert_ffn_one_long_segment_and_empty_experts(moe):
    """All rows on one expert: a segment many tiles long with a ragged tail."""
    wl = scaled(WORKLOADS["tiny"], E=8)
    counts = np.zeros(8, np.int64)
    counts[5] = 1000
    _expert_case(moe, wl, counts, [5], rows_per_expert=64)


def test_expert_ffn_situ_shapes(moe):
    wl = scaled(WORKLOADS["k3_latent_decode"], E=24, d_e=256, F=384, N=200)
    counts = np.random.default_rng(3).integers(0, 140, 24)
    counts[[2, 7]] = 0
    _expert_case(moe, wl, counts, list(range(24)), rows_per_expert=200)


# ------------------------------------------------------------ whole layer
def _forward(moe, wl, dev):
    import torch
    N = wl.N
    idx = torch.empty((N, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((N, wl.K), dtype=torch.float32, device="cuda")
    out = moe.forward(dev["x"], dev["W"], dev["bias"], rcfg(moe, wl), dev["w1"], dev["w3"],
                      dev["w2"], acfg(moe, wl), x_e=dev["x_e"] if wl.latent else None,
                      topk_idx=idx, topk_w=w)
    return host_bf16(out), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", ALL)
def test_forward_end_to_end(moe, name):
    """The whole layer against the reference's per-token loop (the reference's
    own routing), on every token of the small batches and on 128 sampled
    tokens (first, last and 126 random) of the larger ones."""
    wl = WORKLOADS[name]
    dev = synth.workloads.dev_inputs(wl)
    out_g, idx_g, w_g = _forward(moe, wl, dev)
    inp = host_inputs(wl)
    n_tok = wl.N if wl.N <= 128 else 128
    toks = np.arange(wl.N) if n_tok == wl.N else np.unique(
        np.concatenate([[0, wl.N - 1], np.random.default_rng(7).choice(wl.N, n_tok - 2, False)]))
    x = np.ascontiguousarray(inp["x"][toks])
    xe = np.ascontiguousarray(inp["x_e"][toks])
    idx_r, w_r, margin = oracle.route(x, inp["W"], inp["bias"], wl.G, wl.TG, wl.K,
                                      wl.route_scale, wl.norm)
    _check_routing(idx_g[toks], w_g[toks], idx_r, w_r, margin)
    keep = margin > MARGIN
    out_r = oracle_layer_tokens(wl, xe, idx_r, w_r)
    print(f"forward {name}: {keep.sum()}/{len(toks)} tokens")
    check_bf16_outputs(out_g[toks][keep], out_r[keep], long_dots=max(wl.d_e, wl.F) > 512,
                       what=f"layer {name}", layer=True)


@pytest.mark.parametrize("N", [512, 9216])
def test_forward_max_experts_and_top_k(moe, N):
    """The largest expert count and top-k the ABI accepts (E = 1024, K = 16)
    through the whole layer: 512 tokens take the decode kernels (8 rows per
    expert), 9216 tokens the CTA-pair kernels (144 rows per expert, one-tile
    experts spread among larger ones); both take the int8 gate.  128 sampled
    tokens against the reference's per-token loop."""
    wl = scaled(WORKLOADS["tiny"], N=N, E=1024, K=16, name=f"e1024_k16_n{N}")
    assert (N * wl.K) / wl.E > 128 or N == 512
    dev = synth.workloads.dev_inputs(wl)
    out_g, idx_g, w_g = _forward(moe, wl, dev)
    inp = host_inputs(wl)
    toks = np.unique(np.concatenate(
        [[0, N - 1], np.random.default_rng(11).choice(N, 126, False)]))
    x = np.ascontiguousarray(inp["x"][toks])
    xe = np.ascontiguousarray(inp["x_e"][toks])
    idx_r, w_r, margin = oracle.route(x, inp["W"], inp["bias"], wl.G, wl.TG, wl.K,
                                      wl.route_scale, wl.norm)
    _check_routing(idx_g[toks], w_g[toks], idx_r, w_r, margin)
    keep = margin > MARGIN
    out_r = oracle_layer_tokens(wl, xe, idx_r, w_r)
    print(f"forward E=1024 K=16 N={N}: {keep.sum()}/{len(toks)} tokens")
    check_bf16_outputs(out_g[toks][keep], out_r[keep], long_dots=False,
                       what=f"layer E=1024 K=16 N={N}", layer=True)


def test_forward_tiny_matches_reference_moe_infer_exactly_where_routing_agrees(moe):
    """At the tiny size the whole batch goes through the reference's sorted
    moe_infer; compare every token with margin > 1e-5."""
    wl = WORKLOADS["tiny"]
    dev = synth.workloads.dev_inputs(wl)
    out_g, idx_g, w_g = _forward(moe, wl, dev)
    inp = host_inputs(wl)
    from synth.workloads import host_experts_all
    w1, w3, w2 = host_experts_all(wl)
    idx_r, w_r, margin = oracle.route(inp["x"], inp["W"], inp["bias"], wl.G, wl.TG, wl.K,
                                      wl.route_scale)
    out_r = oracle.moe_infer(inp["x_e"], idx_r, w_r, w1, w3, w2, wl.act)
    keep = margin > MARGIN
    check_bf16_outputs(out_g[keep], out_r[keep], long_dots=False, what="tiny sorted moe_infer",
                       layer=True)


def test_forward_deterministic_and_empty(moe):
    import torch
    wl = WORKLOADS["dsv32_decode"]
    dev = synth.workloads.dev_inputs(wl)
    a, _, _ = _forward(moe, wl, dev)
    b, _, _ = _forward(moe, wl, dev)
    assert np.array_equal(a, b)
    # N = 0 is a valid empty call
    x0 = torch.empty((0, wl.d_r), dtype=torch.bfloat16, device="cuda")
    out = moe.forward(x0, dev["W"], dev["bias"], rcfg(moe, wl), dev["w1"], dev["w3"], dev["w2"],
                      acfg(moe, wl))
    assert out.shape == (0, wl.d_e)


def test_forward_single_token(moe):
    wl = scaled(WORKLOADS["k2_prefill"], N=1)
    dev = synth.workloads.dev_inputs(wl)
    out_g, idx_g, w_g = _forward(moe, wl, dev)
    inp = host_inputs(wl)
    idx_r, w_r, margin = oracle.route(inp["x"], inp["W"], inp["bias"], 1, 1, wl.K,
                                      wl.route_scale)
    assert set(idx_g[0]) == set(idx_r[0])
    ys = [oracle.expert_ffn(inp["x_e"], *host_expert(wl, int(e)))[0] for e in idx_r[0]]
    out_r = oracle.combine(np.stack(ys), np.arange(wl.K, dtype=np.int32), w_r, wl.K)
    assert rel_l2(out_g, out_r) <= REL_L2_OUT


@pytest.mark.parametrize("counts", [[1500, 700, 37, 0, 1763], [900, 5, 300, 800, 2000]])
def test_expert_ffn_large_tiles_ragged(moe, counts):
    """> 128 rows per expert on average selects the 256-row tile variant; the
    segments end mid-tile, below 32 rows and on a 64-row box boundary."""
    wl = scaled(WORKLOADS["tiny"], E=5, d_e=256, F=384)
    _expert_case(moe, wl, np.array(counts), list(range(5)), rows_per_expert=96)


@pytest.mark.parametrize("act", ["silu", "situ"])
def test_expert_ffn_pair_tile_order_all_rows(moe, act):
    """The CTA-pair variant takes the tiles of one-tile experts (1 to 256 rows)
    spread among the tiles of larger ones; with 8 one-tile experts (1, 2, 3,
    17, 40, 64, 255 and 256 rows), an empty one and three of 3-4 tiles, every
    output row is checked against the oracle: a tile taken twice or never
    would leave rows wrong.  SiTU takes the same epilogue with its own
    activation."""
    wl = scaled(WORKLOADS["tiny"], E=12, d_e=256, F=384, act=act,
                beta=4.0 if act == "situ" else WORKLOADS["tiny"].beta,
                lbeta=8.0 if act == "situ" else WORKLOADS["tiny"].lbeta)
    counts = np.array([700, 3, 40, 256, 1, 0, 900, 17, 255, 64, 520, 2])
    assert counts.sum() > 128 * wl.E  # the 256-row tile variant
    _expert_case(moe, wl, counts, list(range(12)), rows_per_expert=10 ** 6)


@pytest.mark.parametrize("act", ["silu", "situ"])
def test_expert_ffn_mid_tiles(moe, act):
    """17..128 rows per expert on average selects the 128-row tile variant."""
    wl = scaled(WORKLOADS["k3_latent_decode"], E=12, d_e=384, F=256, act=act)
    counts = np.random.default_rng(9).integers(20, 200, 12)
    counts[4] = 0
    _expert_case(moe, wl, counts, list(range(12)), rows_per_expert=64)


@pytest.mark.parametrize("name,N,E", [("dsv32_decode", 128, 256), ("tiny", 64, 16),
                                      ("k2_prefill", 1024, 96), ("k3_latent_decode", 64, 896),
                                      ("k2_prefill", 5, 384)])
def test_expert_ffn_gathered_equals_the_separate_gather(moe, name, N, E):
    """moe_expert_ffn_gathered (rows gathered inside the w1/w3 kernel by
    tile::gather4) equals moe_expert_ffn on moe_dispatch's gathered copy, bit
    for bit: the MMAs see the same rows in the same order."""
    import torch
    wl = scaled(WORKLOADS[name], N=N, E=E)
    dev = synth.workloads.dev_inputs(wl)
    act = acfg(moe, wl)
    x_e = dev["x_e"] if wl.latent else dev["x"]
    idx, w = moe.route(dev["x"], dev["W"], dev["bias"], rcfg(moe, wl))
    counts, offsets, perm, pos, xs = moe.dispatch(idx, x_e, wl.E)
    y_sep = moe.expert_ffn(xs, offsets, dev["w1"], dev["w3"], dev["w2"], act)
    y_g = moe.expert_ffn_gathered(x_e, wl.K, perm, offsets, dev["w1"], dev["w3"], dev["w2"], act)
    assert torch.equal(y_g.view(torch.int16), y_sep.view(torch.int16))
    # and sampled rows against the reference directly: row j is expert e's
    # MLP on token perm[j] / K
    offs = offsets.cpu().numpy()
    perm_h = perm.cpu().numpy()
    S = int(offs[-1])
    rows = np.unique(np.concatenate([[0, S - 1], np.random.default_rng(3).choice(S, 22)]))
    xe_h = host_inputs(wl)["x_e"]
    got, ref = [], []
    for j in rows:
        e = int(np.searchsorted(offs, j, side="right") - 1)
        x1 = np.ascontiguousarray(xe_h[perm_h[j] // wl.K][None, :])
        ref.append(oracle.expert_ffn(x1, *host_expert(wl, e), wl.act, wl.beta, wl.lbeta)[0])
        got.append(host_bf16(y_g[int(j)]))
    check_bf16_outputs(np.stack(got), np.stack(ref), long_dots=max(wl.d_e, wl.F) > 512,
                       what=f"gathered {name}")
