"""moe_launch_count counts the kernels the library actually launched: one per
combine; for a dispatch that copies rows four (histogram, scan, scatter,
gather), or two for a small one (the one-block sort, gather); three or one
per sort-only dispatch; and the same number for every repetition of one
moe_forward."""
import numpy as np
import pytest

import synth
from tests.gpu_util import dev_bf16, random_topk

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,E,want", [(300, 40, (2, 1, 1)),      # 1200 slots: the one-block sort
                                      (300, 1000, (2, 1, 1)),    # up to 1024 experts: the same
                                      (2000, 40, (4, 3, 1))])    # more than 4096 slots
def test_launch_count_per_entry_point(N, E, want):
    import torch
    import moe_routing_expert_fp32_b200 as moe
    K, d = 4, 256
    idx = torch.from_numpy(random_topk(N, K, E, np.random.default_rng(5))).cuda()
    x = dev_bf16(synth.host_normal_bf16(3, 1, (N, d), 1.0))
    moe.dispatch(idx, x, E)  # first call: kernel attributes set up
    n0 = moe.launch_count()
    counts, offsets, perm, pos, xs = moe.dispatch(idx, x, E)
    n1 = moe.launch_count()
    moe.dispatch(idx, x, E, gather=False)
    n2 = moe.launch_count()
    w = torch.rand((N, K), dtype=torch.float32, device="cuda")
    moe.combine(xs, pos, w)
    n3 = moe.launch_count()
    torch.cuda.synchronize()
    assert (n1 - n0, n2 - n1, n3 - n2) == want


def test_launch_count_of_forward_is_stable():
    import torch
    import moe_routing_expert_fp32_b200 as moe
    from synth.workloads import WORKLOADS, dev_inputs
    wl = WORKLOADS["tiny"]
    dev = dev_inputs(wl)
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    ws = moe.workspace(moe.workspace_size(wl.N, wl.d_r, wl.d_e, cfg, wl.F))
    deltas = []
    for _ in range(3):
        n0 = moe.launch_count()
        moe.forward(dev["x"], dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"], act,
                    ws=ws)
        deltas.append(moe.launch_count() - n0)
    torch.cuda.synchronize()
    # route (gate GEMM + selection), dispatch (one-block sort + gather at
    # 256 slots), tile list, two expert GEMMs, combine
    assert deltas[0] == deltas[1] == deltas[2] and 8 <= deltas[0] <= 13


def test_launch_count_of_route_on_both_gate_paths():
    """moe_route launches: the fp32 gate GEMM and the selection for a decode
    batch (the split-K partials are summed by the selection, no reduce
    kernel); the two slicers, the int8 gate GEMM and the selection once the
    batch fills the int8 tiles (here 25 tiles of 128 experts x 96 tokens)."""
    import torch
    import moe_routing_expert_fp32_b200 as moe
    for (N, E, d, want) in [(128, 256, 7168, 2), (2400, 128, 64, 4)]:
        x = synth.dev_normal_bf16(torch.empty((N, d), dtype=torch.bfloat16, device="cuda"), 1, 1,
                                  1.0)
        W = synth.dev_normal_f32(torch.empty((E, d), dtype=torch.float32, device="cuda"), 1, 2,
                                 0.02)
        cfg = moe.RouteConfig(E, 1, 1, 8, 1.0, True)
        moe.route(x, W, None, cfg)  # kernel attributes set up
        n0 = moe.launch_count()
        moe.route(x, W, None, cfg)
        assert moe.launch_count() - n0 == want, (N, E, d)
    torch.cuda.synchronize()
