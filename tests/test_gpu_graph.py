"""moe_forward captured in a CUDA graph: the layer makes no host
synchronisation and allocates nothing on the device (the caller's workspace
and output), so one forward can be captured and replayed.  A replay must give
the eager call's output bit for bit, also after new input values are written
into the captured buffers."""
import numpy as np
import pytest

from synth.workloads import WORKLOADS, dev_inputs, scaled

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],                                  # decode variant, launch-bound
    "dsv32_decode": WORKLOADS["dsv32_decode"],                  # decode variant, split-K gate
    "pair_16x512": scaled(WORKLOADS["k2_prefill"], E=16, N=512),  # CTA-pair GEMMs, int8 gate
}


@pytest.fixture(scope="module")
def moe():
    import moe_routing_expert_fp32_b200 as m
    m.lib()
    return m


@pytest.mark.parametrize("name", list(CASES))
def test_forward_graph_replay_matches_eager(moe, name):
    import torch
    wl = CASES[name]
    dev = dev_inputs(wl)
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    ws = moe.workspace(moe.workspace_size(wl.N, wl.d_r, wl.d_e, cfg, wl.F))
    x = dev["x"].clone()
    out = torch.empty((wl.N, wl.d_e), dtype=torch.bfloat16, device="cuda")

    def fwd(inp, o):
        return moe.forward(inp, dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"], act,
                           ws=ws, out=o)

    # eager result (also makes every one-time set-up call before the capture)
    ref = fwd(x, torch.empty_like(out)).clone()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fwd(x, out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    n0 = moe.launch_count()
    with torch.cuda.graph(g):
        fwd(x, out)
    captured = moe.launch_count() - n0
    assert captured > 0
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.get_status(ws) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))

    # new values in the captured input buffer: the replay follows them
    x.copy_(-dev["x"])
    g.replay()
    torch.cuda.synchronize()
    ref2 = fwd(-dev["x"], torch.empty_like(out))
    torch.cuda.synchronize()
    assert moe.get_status(ws) == 0
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
    assert not torch.equal(ref2.view(torch.int16), ref.view(torch.int16))
    print(f"{name}: {captured} kernels in the graph")


@pytest.mark.parametrize("name", ["tiny_block", "k3_block_decode"])
def test_block_graph_replay_matches_eager(moe, name):
    """The whole MoE block (latent projections, norm, shared experts, split-K
    dense layers) captured and replayed."""
    import torch
    import synth
    from synth.workloads import BLOCKS
    wl = BLOCKS[name]
    dev = dev_inputs(wl)
    blk = synth.workloads.dev_block(wl)
    W = moe.BlockWeights(
        gate_weight=dev["W"], gate_bias=dev["bias"], w1=dev["w1"], w3=dev["w3"], w2=dev["w2"],
        down_proj=blk["down_proj"], norm_weight=blk["norm_w"], up_proj=blk["up_proj"],
        shared_w1=None if blk["shared"] is None else blk["shared"][0],
        shared_w3=None if blk["shared"] is None else blk["shared"][1],
        shared_w2=None if blk["shared"] is None else blk["shared"][2])
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    x = dev["x"].clone()
    ref = moe.block_forward(x, W, cfg, act, norm_eps=wl.norm_eps).clone()
    torch.cuda.synchronize()
    ws = moe.workspace(moe.lib().moe_block_workspace_size(
        wl.N, *_block_args(moe, wl, W, cfg)))
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.block_forward(x, W, cfg, act, norm_eps=wl.norm_eps, ws=ws, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.block_forward(x, W, cfg, act, norm_eps=wl.norm_eps, ws=ws, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.get_status(ws) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    x.copy_(-dev["x"])
    g.replay()
    ref2 = moe.block_forward(-dev["x"], W, cfg, act, norm_eps=wl.norm_eps)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))


def _block_args(moe, wl, W, cfg):
    import ctypes
    F_sh = 0 if W.shared_w1 is None else W.shared_w1.shape[0]
    dims = moe._BlockDims(wl.d_r, wl.d_e, wl.F, F_sh, float(wl.norm_eps))
    return ctypes.byref(dims), ctypes.byref(W._c()), ctypes.byref(cfg._c())
