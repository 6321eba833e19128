"""Expert parallelism on one GPU: P ranks emulated in one process.

Every emulated rank routes and sorts its own tokens (moe_route,
moe_dispatch); the all-to-alls of the expert-parallel step are emulated by
slicing (rank q receives, from every source p, the rows of its experts
q*E_local .. +E_local-1, which are contiguous in p's sorted rows); rank q runs
moe_ep_expert_ffn on what it received with its own slice of the expert
weights; the outputs go back to their sources in the same slices and each
source combines them.  The result must match the single-GPU layer
(moe_forward) on the same tokens: same routing, outputs within 1e-3 relative
L2 (the rows meet the same MMAs in the same k order; tile shapes may differ);
and sampled tokens of every rank must meet the reference (the CPU oracle's
expert MLP and combine, fed with the GPU's routing) under the layer's output
bars.
A real multi-GPU run of this exchange (NCCL all-to-all over NVLink) needs
more than one GPU; its host logic is tested with gloo on CPU.
"""
import numpy as np
import pytest

import synth
from synth.workloads import WORKLOADS, host_inputs, scaled
from tests.gpu_util import check_bf16_outputs, host_bf16, oracle_layer_tokens, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import moe_routing_expert_fp32_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("name,P,N", [("tiny", 2, 64), ("dsv32_decode", 4, 32),
                                      ("k3_latent_decode", 8, 16), ("k2_prefill", 4, 256)])
def test_ep_emulated_equals_one_gpu(moe, name, P, N):
    import torch
    wl = scaled(WORKLOADS[name], N=N)
    E_l = wl.E // P
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    shared = synth.workloads.dev_inputs(wl, rank=0)
    W, b, w1, w3, w2 = shared["W"], shared["bias"], shared["w1"], shared["w3"], shared["w2"]
    ranks = []
    for p in range(P):
        d = synth.workloads.dev_inputs(wl, rank=p, experts=False)
        x_e = d["x_e"] if wl.latent else d["x"]
        idx, w = moe.route(d["x"], W, b, cfg)
        counts, offs, perm, pos, xs = moe.dispatch(idx, x_e, wl.E)
        ref = moe.forward(d["x"], W, b, cfg, w1, w3, w2, act, x_e=d["x_e"] if wl.latent else None)
        ranks.append(dict(idx=idx, w=w, counts=counts, offs=offs.cpu().numpy(), pos=pos, xs=xs,
                          ref=ref))
    # the exchange, emulated: rank q's received rows and counts
    y_back = [torch.empty_like(r["xs"]) for r in ranks]
    for q in range(P):
        lo, hi = q * E_l, (q + 1) * E_l
        parts = [r["xs"][r["offs"][lo]:r["offs"][hi]] for r in ranks]
        recv = torch.cat(parts).contiguous()
        rc = torch.stack([r["counts"][lo:hi] for r in ranks]).contiguous()
        yq = moe.ep_expert_ffn(recv, rc, w1[lo:hi], w3[lo:hi], w2[lo:hi], act)
        o = 0
        for p, r in enumerate(ranks):
            n = int(r["offs"][hi] - r["offs"][lo])
            y_back[p][r["offs"][lo]:r["offs"][hi]] = yq[o:o + n]
            o += n
        assert o == recv.shape[0]
    outs = []
    for p, r in enumerate(ranks):
        out = moe.combine(y_back[p], r["pos"], r["w"])
        outs.append(out)
        got, ref = host_bf16(out), host_bf16(r["ref"])
        err = rel_l2(got, ref)
        print(f"{name} rank {p}/{P}: rel_l2 {err:.2e}, bit-exact {np.mean(got == ref):.4f}")
        assert err <= 1e-3
    _check_against_reference(wl, P, outs, ranks)


def _check_against_reference(wl, P, outs, ranks, per_rank=16):
    """Sampled tokens of every emulated rank against the reference's
    per-token loop (its expert MLP and combine), fed with the routing the
    GPU computed for them, so that only the expert-parallel step is checked."""
    xe, idx, w, got = [], [], [], []
    for p, r in enumerate(ranks):
        n = wl.N
        toks = np.arange(n) if n <= per_rank else np.unique(
            np.concatenate([[0, n - 1], np.random.default_rng(p).choice(n, per_rank - 2, False)]))
        xe.append(host_inputs(wl, rank=p)["x_e"][toks])
        idx.append(r["idx"].cpu().numpy()[toks])
        w.append(r["w"].cpu().numpy()[toks])
        got.append(host_bf16(outs[p])[toks])
    ref = oracle_layer_tokens(wl, np.concatenate(xe), np.concatenate(idx), np.concatenate(w))
    check_bf16_outputs(np.concatenate(got), ref, long_dots=max(wl.d_e, wl.F) > 512,
                       what=f"expert-parallel {wl.name} P={P}", layer=True)


def test_ep_expert_ffn_reports_inconsistent_counts(moe):
    """recv_counts that do not add up to the rows: reported, nothing read out
    of range."""
    import torch
    wl = scaled(WORKLOADS["tiny"], N=16)
    d = synth.workloads.dev_inputs(wl)
    xr = d["x"][:10].contiguous()
    rc = torch.tensor([[3, 4], [5, 6]], dtype=torch.int32, device="cuda")  # 18 != 10
    ws = moe.workspace(moe.lib().moe_ep_expert_ffn_workspace_size(10, wl.d_e, 2, 2, wl.F))
    moe.ep_expert_ffn(xr, rc, d["w1"][:2], d["w3"][:2], d["w2"][:2], moe.ActConfig(), ws=ws)
    assert moe.get_status(ws) == -7


@pytest.mark.parametrize("name,P,N", [("tiny", 2, 64), ("dsv32_decode", 4, 32),
                                      ("k3_latent_decode", 8, 16), ("k2_prefill", 4, 256)])
def test_ep_peer_rows_emulated(moe, name, P, N):
    """The exchange through peer memory (moe_ep_dispatch_rows,
    moe_ep_combine_rows) with P ranks emulated on one GPU: every rank's
    buffers are ordinary allocations of this GPU, addressed exactly as peer
    mappings would be.  Each rank's received rows must equal, bit for bit,
    the rows the all-to-all delivers (slices of the senders' sorted rows); the
    combine loading outputs from the ranks' buffers must equal, bit for bit,
    moe_combine on the same outputs brought home; the layer output matches
    moe_forward within 1e-3 relative L2."""
    import torch
    from moe_routing_expert_fp32_b200.ep import p2p_plan
    wl = scaled(WORKLOADS[name], N=N)
    E_l = wl.E // P
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    shared = synth.workloads.dev_inputs(wl, rank=0)
    W, b, w1, w3, w2 = shared["W"], shared["bias"], shared["w1"], shared["w3"], shared["w2"]
    ranks = []
    for p in range(P):
        d = synth.workloads.dev_inputs(wl, rank=p, experts=False)
        x_e = d["x_e"] if wl.latent else d["x"]
        idx, w = moe.route(d["x"], W, b, cfg)
        counts, offs, perm, pos, xs_none = moe.dispatch(idx, x_e, wl.E, gather=False)
        assert xs_none is None
        counts2, offs2, perm2, pos2, xs = moe.dispatch(idx, x_e, wl.E)
        for a, b2 in ((counts, counts2), (offs, offs2), (perm, perm2), (pos, pos2)):
            assert torch.equal(a, b2)
        ref = moe.forward(d["x"], W, b, cfg, w1, w3, w2, act, x_e=d["x_e"] if wl.latent else None)
        ranks.append(dict(x_e=x_e, idx=idx, w=w, counts=counts, offs=offs, pos=pos, xs=xs,
                          ref=ref))
    all_counts = torch.stack([r["counts"] for r in ranks]).cpu().numpy()
    plans = [p2p_plan(all_counts, p, P) for p in range(P)]
    cap = [max(1, plans[q][2]) for q in range(P)]
    # each rank's receive and output buffers, with a guard row past the end
    xr = [torch.full((cap[q] + 1, wl.d_e), 7.0, dtype=torch.bfloat16, device="cuda")
          for q in range(P)]
    yb = [torch.empty((cap[q] + 1, wl.d_e), dtype=torch.bfloat16, device="cuda")
          for q in range(P)]
    for p, r in enumerate(ranks):
        table = moe.peer_rows(xr, plans[p][0], cap)
        ws = moe.workspace(256)
        moe.ep_dispatch_rows(r["x_e"], r["pos"], r["offs"], wl.E, table, wl.K, ws=ws)
        assert moe.get_status(ws) == 0
    offs_h = [r["offs"].cpu().numpy() for r in ranks]
    for q in range(P):
        lo, hi = q * E_l, (q + 1) * E_l
        want = torch.cat([r["xs"][offs_h[p][lo]:offs_h[p][hi]] for p, r in enumerate(ranks)])
        R = plans[q][2]
        assert torch.equal(xr[q][:R], want), f"rank {q}: received rows differ"
        assert bool((xr[q][cap[q]] == 7.0).all()), "guard row overwritten"
        rc = torch.from_numpy(plans[q][1]).cuda()
        moe.ep_expert_ffn(xr[q][:R], rc, w1[lo:hi], w3[lo:hi], w2[lo:hi], act, y=yb[q][:R])
    outs = []
    for p, r in enumerate(ranks):
        table = moe.peer_rows(yb, plans[p][0], cap)
        ws = moe.workspace(256)
        out = moe.ep_combine_rows(table, r["pos"], r["offs"], wl.E, r["w"], wl.d_e, ws=ws)
        outs.append(out)
        assert moe.get_status(ws) == 0
        # the same outputs brought home in sorted order, then moe_combine
        home = torch.empty_like(r["xs"])
        for q in range(P):
            lo, hi = offs_h[p][q * E_l], offs_h[p][(q + 1) * E_l]
            f = plans[p][0][q]
            home[lo:hi] = yb[q][f:f + (hi - lo)]
        assert torch.equal(out, moe.combine(home, r["pos"], r["w"]))
        got, ref = host_bf16(out), host_bf16(r["ref"])
        err = rel_l2(got, ref)
        print(f"{name} rank {p}/{P} (peer rows): rel_l2 {err:.2e}")
        assert err <= 1e-3
    _check_against_reference(wl, P, outs, ranks)


def test_ep_peer_rows_out_of_capacity_is_reported(moe):
    """A buffer too small for the rows sent to it: the rows past its capacity
    are not stored (a guard region past it stays intact) and the status word
    says MOE_ERR_DEVICE_BOUNDS; the same for the combine's loads."""
    import torch
    wl = scaled(WORKLOADS["tiny"], N=32)
    P = 2
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    d = synth.workloads.dev_inputs(wl)
    idx, w = moe.route(d["x"], d["W"], d["bias"], cfg)
    counts, offs, _, pos, _ = moe.dispatch(idx, d["x"], wl.E, gather=False)
    plan = __import__("moe_routing_expert_fp32_b200.ep", fromlist=["p2p_plan"]).p2p_plan(
        counts.cpu().numpy()[None, :].repeat(P, 0), 0, P)
    sent = [int(offs[(q + 1) * (wl.E // P)] - offs[q * (wl.E // P)]) for q in range(P)]
    assert min(sent) > 2
    cap = [s - 2 for s in sent]  # two rows short on each rank
    bufs = [torch.full((s + 8, wl.d_e), 3.0, dtype=torch.bfloat16, device="cuda") for s in sent]
    ws = moe.workspace(256)
    moe.ep_dispatch_rows(d["x"], pos, offs, wl.E, moe.peer_rows(bufs, plan[0], cap), wl.K, ws=ws)
    assert moe.get_status(ws) == -7
    for q in range(P):
        assert bool((bufs[q][cap[q]:] == 3.0).all())
    ws = moe.workspace(256)
    moe.ep_combine_rows(moe.peer_rows(bufs, plan[0], cap), pos, offs, wl.E, w, wl.d_e, ws=ws)
    assert moe.get_status(ws) == -7
