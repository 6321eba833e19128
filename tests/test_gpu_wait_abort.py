"""The bounded-wait abort path of the grouped expert GEMM kernels, made to run
by the diagnostics hook (moe_set_wait_probe): each CTA's producer waits on a
barrier that nothing arrives on before it issues any copy, gives up after
1 ms, records MOE_ERR_DEVICE_TIMEOUT and the kernel stops (other roles
stopped, tensor memory freed).  Nothing faults or hangs: the status word
reads -6, the outputs are untouched, and the next call (hook off) on the same
context gives exactly the result it gave before."""
import numpy as np
import pytest

import synth
from synth.workloads import WORKLOADS, scaled

pytestmark = pytest.mark.gpu


def _case(moe, wl, counts, seed=3):
    import torch
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    S = int(offsets[-1])
    xs = synth.dev_normal_bf16(torch.empty((S, wl.d_e), dtype=torch.bfloat16, device="cuda"),
                               seed, 12, 1.0)
    dev = synth.workloads.dev_inputs(wl, experts=True)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    return xs, torch.from_numpy(offsets).cuda(), dev, act


# decode (<= 16 rows per expert), mid (<= 128) and CTA-pair (> 128) variants
@pytest.mark.parametrize("counts", [[3, 0, 5, 1, 2, 7, 0, 4], [60, 90, 0, 130, 44, 100, 70, 25],
                                    [1500, 700, 37, 0, 1763]])
def test_wait_probe_aborts_cleanly_and_the_context_stays_usable(counts):
    import torch
    import moe_routing_expert_fp32_b200 as moe
    wl = scaled(WORKLOADS["tiny"], E=len(counts), d_e=256, F=384)
    xs, offsets, dev, act = _case(moe, wl, np.array(counts))
    ws = moe.workspace(moe.lib().moe_expert_ffn_workspace_size(xs.shape[0], wl.d_e, wl.E, wl.F))
    y_ref = moe.expert_ffn(xs, offsets, dev["w1"], dev["w3"], dev["w2"], act, ws=ws)
    torch.cuda.synchronize()
    assert moe.get_status(ws) == 0
    sentinel = torch.full_like(y_ref, 7.0)
    prev = moe.set_wait_probe(True)
    try:
        y = moe.expert_ffn(xs, offsets, dev["w1"], dev["w3"], dev["w2"], act, ws=ws,
                           y=sentinel.clone())
        torch.cuda.synchronize()
        assert moe.get_status(ws) == -6          # MOE_ERR_DEVICE_TIMEOUT, read from the device
        assert torch.equal(y.view(torch.int16), sentinel.view(torch.int16))  # nothing written
    finally:
        moe.set_wait_probe(prev)
    y2 = moe.expert_ffn(xs, offsets, dev["w1"], dev["w3"], dev["w2"], act, ws=ws)
    torch.cuda.synchronize()
    assert moe.get_status(ws) == 0
    assert torch.equal(y2.view(torch.int16), y_ref.view(torch.int16))


def test_wait_probe_reaches_the_whole_layer():
    """moe_forward runs the same kernels: with the hook on its status reads -6,
    with the hook off the layer gives its usual output again."""
    import torch
    import moe_routing_expert_fp32_b200 as moe
    from synth.workloads import dev_inputs
    wl = WORKLOADS["tiny"]
    dev = dev_inputs(wl)
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    ws = moe.workspace(moe.workspace_size(wl.N, wl.d_r, wl.d_e, cfg, wl.F))

    def fwd():
        out = moe.forward(dev["x"], dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"],
                          act, ws=ws)
        torch.cuda.synchronize()
        return out, moe.get_status(ws)

    ref, st = fwd()
    assert st == 0
    prev = moe.set_wait_probe(True)
    try:
        _, st = fwd()
        assert st == -6
    finally:
        moe.set_wait_probe(prev)
    out, st = fwd()
    assert st == 0 and torch.equal(out.view(torch.int16), ref.view(torch.int16))
