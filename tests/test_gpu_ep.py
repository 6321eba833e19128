"""Expert parallelism on one GPU: P ranks emulated in one process.

Every emulated rank routes and sorts its own tokens (moe_route,
moe_dispatch); the all-to-alls of the expert-parallel step are emulated by
slicing (rank q receives, from every source p, the rows of its experts
q*E_local .. +E_local-1, which are contiguous in p's sorted rows); rank q runs
moe_ep_expert_ffn on what it received with its own slice of the expert
weights; the outputs go back to their sources in the same slices and each
source combines them.  The result must match the single-GPU layer
(moe_forward) on the same tokens: same routing, outputs within 1e-3 relative
L2 (the rows meet the same MMAs in the same k order; tile shapes may differ).
A real multi-GPU run of this exchange (NCCL all-to-all over NVLink) needs
more than one GPU; its host logic is tested with gloo on CPU.
"""
import numpy as np
import pytest

import synth
from synth.workloads import WORKLOADS, scaled
from tests.gpu_util import host_bf16, rel_l2

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
    for p, r in enumerate(ranks):
        out = moe.combine(y_back[p], r["pos"], r["w"])
        got, ref = host_bf16(out), host_bf16(r["ref"])
        err = rel_l2(got, ref)
        print(f"{name} rank {p}/{P}: rel_l2 {err:.2e}, bit-exact {np.mean(got == ref):.4f}")
        assert err <= 1e-3


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
