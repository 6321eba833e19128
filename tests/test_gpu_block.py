"""Parity of the block entry points (moe_linear, moe_rms_norm,
moe_block_forward) with the CPU reference, on the GPU, through the C ABI.

Bars:
  * moe_linear: relative L2 <= 2e-2 in bf16 and at most a few bf16 ulps
    anywhere (tensor-core fp32 accumulation against a double sum); the
    residual add is checked bit for bit against the reference add of the
    kernel's own Linear output;
  * moe_rms_norm and the fused combine + RMSNorm: bit-exact (both sides take
    the mean in double and round once from double), allowing a handful of
    one-ulp flips where the two sum orders straddle a rounding midpoint;
  * moe_block_forward: routing as moe_route; over the tokens whose
    biased-score margin exceeds 1e-5, output relative L2 <= 2e-2 and the
    per-row and per-element bars of the layer output (tests/gpu_util.py);
    the shared experts' MLP meets the expert MLP's bars.
"""
import numpy as np
import pytest

import oracle
import synth
from synth.workloads import BLOCKS, host_block, host_expert, host_inputs, scaled
from tests.gpu_util import (MARGIN, REL_L2_OUT, check_bf16_outputs, dev_bf16, host_bf16, rel_l2,
                            ulp_diff)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import moe_routing_expert_fp32_b200 as m
    m.lib()
    oracle.set_threads(0)
    return m


def _rand_bf16(rng, shape, scale=1.0):
    v = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = v.view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


# ------------------------------------------------------------------- linear
@pytest.mark.parametrize("M,K,N_out", [(1, 7168, 2048), (7, 256, 128), (64, 7168, 2048),
                                       (64, 2048, 7168), (100, 512, 384), (300, 1024, 256),
                                       (1000, 256, 640), (16, 7168, 2048), (128, 2048, 7168)])
def test_linear(moe, M, K, N_out):
    rng = np.random.default_rng(M * 7 + K + N_out)
    x = _rand_bf16(rng, (M, K))
    W = _rand_bf16(rng, (N_out, K), 0.02)
    res = _rand_bf16(rng, (M, N_out))
    y_g = host_bf16(moe.linear(dev_bf16(x), dev_bf16(W)))
    y_r = oracle.linear(x, W)
    err = rel_l2(y_g, y_r)
    ud = ulp_diff(y_g, y_r)
    print(f"M={M} K={K} N={N_out}: rel_l2 {err:.2e}, max ulp {ud.max()}, "
          f"exact {np.mean(ud == 0):.4f}")
    assert err <= REL_L2_OUT
    assert np.mean(ud <= 1) >= 0.99
    # residual: bf16(bf16(x.W^T) + res), checked against the kernel's own product
    z_g = host_bf16(moe.linear(dev_bf16(x), dev_bf16(W), residual=dev_bf16(res)))
    assert np.array_equal(z_g, oracle.add(y_g, res))


def test_linear_residual_in_place(moe):
    rng = np.random.default_rng(5)
    x = _rand_bf16(rng, (40, 256))
    W = _rand_bf16(rng, (256, 256), 0.05)
    r = _rand_bf16(rng, (40, 256))
    y = host_bf16(moe.linear(dev_bf16(x), dev_bf16(W)))
    buf = dev_bf16(r)
    moe.linear(dev_bf16(x), dev_bf16(W), residual=buf, out=buf)
    assert np.array_equal(host_bf16(buf), oracle.add(y, r))


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("N,d,eps", [(1, 2048, 1e-6), (300, 2048, 1e-6), (77, 128, 1e-2),
                                     (50, 1024, 0.0), (33, 4096, 1e-6), (9, 8192, 1e-5),
                                     (5, 136, 1e-6)])
def test_rms_norm_bit_exact(moe, N, d, eps):
    rng = np.random.default_rng(N + d)
    x = _rand_bf16(rng, (N, d), 1.7)
    w = _rand_bf16(rng, (d,), 0.3)
    out_g = host_bf16(moe.rms_norm(dev_bf16(x), dev_bf16(w), eps))
    out_r = oracle.rms_norm(x, w, eps)
    ud = ulp_diff(out_g, out_r)
    assert ud.max() <= 1 and (ud > 0).sum() <= max(2, out_r.size // 100000), (ud > 0).sum()


# ------------------------------------------------------------------- block
def _block_dev(moe, wl, dev, blk):
    W = moe.BlockWeights(
        gate_weight=dev["W"], gate_bias=dev["bias"], w1=dev["w1"], w3=dev["w3"], w2=dev["w2"],
        down_proj=blk["down_proj"], norm_weight=blk["norm_w"], up_proj=blk["up_proj"],
        shared_w1=None if blk["shared"] is None else blk["shared"][0],
        shared_w3=None if blk["shared"] is None else blk["shared"][1],
        shared_w2=None if blk["shared"] is None else blk["shared"][2])
    return W


def _run_block(moe, wl, norm=True, shared=True):
    import torch
    dev = synth.workloads.dev_inputs(wl)
    blk = synth.workloads.dev_block(wl)
    if not norm:
        blk["norm_w"] = None
    if not shared:
        blk["shared"] = None
    W = _block_dev(moe, wl, dev, blk)
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    idx = torch.empty((wl.N, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.N, wl.K), dtype=torch.float32, device="cuda")
    out = moe.block_forward(dev["x"], W, cfg, act, norm_eps=wl.norm_eps, topk_idx=idx,
                            topk_w=w)
    return host_bf16(out), idx.cpu().numpy(), w.cpu().numpy()


def _ref_tokens(wl, toks, norm=True, shared=True):
    """The reference block for the given tokens, expert weights regenerated
    one expert at a time (per-token loop of the pinned parts)."""
    inp = host_inputs(wl)
    hb = host_block(wl)
    x = np.ascontiguousarray(inp["x"][toks])
    idx_r, w_r, margin = oracle.route(x, inp["W"], inp["bias"], wl.G, wl.TG, wl.K,
                                      wl.route_scale, wl.norm)
    xe = oracle.linear(x, hb["down_proj"]) if wl.latent else x
    cache = {}
    out = np.zeros((len(toks), wl.d_r), np.uint16)
    for i in range(len(toks)):
        ys = []
        for e in idx_r[i]:
            e = int(e)
            if e not in cache:
                cache[e] = host_expert(wl, e)
            ys.append(oracle.expert_ffn(xe[i:i + 1], *cache[e], wl.act, wl.beta, wl.lbeta)[0])
        y = oracle.combine(np.stack(ys), np.arange(wl.K, dtype=np.int32),
                           np.ascontiguousarray(w_r[i:i + 1]), wl.K)
        if wl.latent:
            if norm:
                y = oracle.rms_norm(y, hb["norm_w"], wl.norm_eps)
            y = oracle.linear(y, hb["up_proj"])
        if shared and hb["shared"] is not None:
            y = oracle.add(y, oracle.expert_ffn(x[i:i + 1], *hb["shared"], wl.act, wl.beta,
                                                wl.lbeta))
        out[i] = y[0]
    return out, idx_r, w_r, margin


def _check_block(wl, out_g, idx_g, toks, norm=True, shared=True):
    out_r, idx_r, w_r, margin = _ref_tokens(wl, toks, norm, shared)
    keep = margin > MARGIN
    assert keep.mean() > 0.5
    for i in np.nonzero(keep)[0]:
        assert set(idx_g[toks[i]].tolist()) == set(idx_r[i].tolist())
    print(f"{wl.name}: {keep.sum()}/{len(toks)} tokens")
    check_bf16_outputs(out_g[toks][keep], out_r[keep],
                       long_dots=max(wl.d_r, wl.d_e, wl.F, wl.F_shared) > 512,
                       what=f"block {wl.name}", layer=True, ulp_bars=False)


@pytest.mark.parametrize("norm,shared", [(True, True), (False, True), (True, False)])
def test_block_tiny(moe, norm, shared):
    wl = BLOCKS["tiny_block"]
    out_g, idx_g, _ = _run_block(moe, wl, norm, shared)
    _check_block(wl, out_g, idx_g, np.arange(wl.N), norm, shared)


def test_block_not_latent_with_shared(moe):
    """d_e = d_r: no projections; the combine adds the shared output."""
    wl = scaled(BLOCKS["tiny_block"], name="tiny_dense_block", d_e=256, latent=False, act="silu")
    out_g, idx_g, _ = _run_block(moe, wl)
    _check_block(wl, out_g, idx_g, np.arange(wl.N))


def test_block_k3_decode(moe):
    wl = BLOCKS["k3_block_decode"]
    out_g, idx_g, _ = _run_block(moe, wl)
    toks = np.array([0, 3, 5, 9, 17, 22, 28, 31, 36, 40, 44, 49, 53, 58, 61, 63])
    _check_block(wl, out_g, idx_g, toks)


def test_block_prefill_sizes(moe):
    """A batch that takes the CTA-pair GEMMs for the dense layers."""
    wl = scaled(BLOCKS["k3_block_decode"], name="k3_block_prefill", N=1024, E=64, F=512)
    out_g, idx_g, _ = _run_block(moe, wl)
    toks = np.array([0, 1, 300, 777, 1023])
    _check_block(wl, out_g, idx_g, toks)


def test_block_edge_sizes(moe):
    for n in (0, 1, 3):
        wl = scaled(BLOCKS["tiny_block"], N=n)
        out_g, idx_g, _ = _run_block(moe, wl)
        assert out_g.shape == (n, wl.d_r)
        if n:
            _check_block(wl, out_g, idx_g, np.arange(n))


def test_block_equals_its_entry_points_bitwise(moe):
    """moe_block_forward (fused combine + RMSNorm, residual in the up
    projection's epilogue) equals the same block built from the separate entry
    points, bit for bit."""
    import torch
    wl = scaled(BLOCKS["k3_block_decode"], name="k3_block_small", N=200, E=32)
    dev = synth.workloads.dev_inputs(wl)
    blk = synth.workloads.dev_block(wl)
    cfg = moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    out_b = moe.block_forward(dev["x"], _block_dev(moe, wl, dev, blk), cfg, act,
                              norm_eps=wl.norm_eps)
    x_e = moe.linear(dev["x"], blk["down_proj"])
    y = moe.forward(dev["x"], dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"], act,
                    x_e=x_e)
    y = moe.rms_norm(y, blk["norm_w"], wl.norm_eps)
    sh = moe.shared_experts(dev["x"], *blk["shared"], act)
    out_p = moe.linear(y, blk["up_proj"], residual=sh)
    assert torch.equal(out_b.view(torch.int16), out_p.view(torch.int16))


@pytest.mark.parametrize("M,d,F,act", [(64, 7168, 3072, "situ"), (1, 7168, 3072, "silu"),
                                       (100, 512, 256, "silu"), (600, 256, 384, "situ")])
def test_shared_experts(moe, M, d, F, act):
    """The shared experts' MLP (split over K at small M) against the reference
    expert MLP, with and without a residual."""
    rng = np.random.default_rng(M + d + F)
    x = _rand_bf16(rng, (M, d))
    w1, w3 = _rand_bf16(rng, (F, d), 0.02), _rand_bf16(rng, (F, d), 0.02)
    w2 = _rand_bf16(rng, (d, F), 0.02)
    res = _rand_bf16(rng, (M, d))
    a = moe.ActConfig(act, 4.0, 8.0) if act == "situ" else moe.ActConfig("silu")
    y_g = host_bf16(moe.shared_experts(dev_bf16(x), dev_bf16(w1), dev_bf16(w3), dev_bf16(w2), a))
    rows = np.arange(M) if M <= 100 else np.array([0, 1, 255, 256, M - 1])
    y_r = oracle.expert_ffn(np.ascontiguousarray(x[rows]), w1, w3, w2, a.kind, a.beta,
                            a.linear_beta)
    print(f"M={M} d={d} F={F}")
    check_bf16_outputs(y_g[rows], y_r, long_dots=max(d, F) > 512, what=f"shared M={M}")
    z_g = host_bf16(moe.shared_experts(dev_bf16(x), dev_bf16(w1), dev_bf16(w3), dev_bf16(w2), a,
                                       residual=dev_bf16(res)))
    assert np.array_equal(z_g, oracle.add(y_g, res))

