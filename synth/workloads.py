"""The five synthetic MoE-layer workloads and how their inputs are drawn.

Shapes, distributions and routing parameters follow the workload list of the
project (tiny, DeepSeek-V3.2-shaped decode, Kimi-K2-shaped prefill, Kimi-K3-
shaped latent decode, skewed Kimi-K2 stress).  Every tensor comes from the
counter-based generator in ``synth.h`` with its own tensor id, so any slice can
be regenerated on either side.

Recipe (seed 0 unless stated):
  x    [N, d_r]  bf16  ~ N(0, 1)          tensor id 1 (rank r uses rows r*N .. r*N+N-1)
  W    [E, d_r]  fp32  ~ N(0, 0.02)       tensor id 2
  b    [E]       fp32  ~ U(-0.01, 0.01)   tensor id 3 (skewed workload: calibrated file)
  w1   [E, F, d_e] bf16 ~ N(0, 0.02)      tensor id 4
  w3   [E, F, d_e] bf16 ~ N(0, 0.02)      tensor id 5
  w2   [E, d_e, F] bf16 ~ N(0, 0.02)      tensor id 6
  x_e  [N, d_e]  bf16  = bf16(x . P^T)    latent workload only (else x_e = x): the
                                           down-projected x, P [d_e, d_r] fp32 ~
                                           N(0, 1/d_r), tensor id 7, so x_e ~ N(0, 1)

The whole-block workload (routed layer inside KimiSparseMoeBlock) adds:
  down_proj [d_e, d_r] bf16 ~ N(0, 0.02)          tensor id 9
  norm_w    [d_e]      bf16 = bf16(U(0.5, 1.5))   tensor id 10
  up_proj   [d_r, d_e] bf16 ~ N(0, 0.02)          tensor id 11
  shared w1, w3 [F_sh, d_r], w2 [d_r, F_sh] bf16 ~ N(0, 0.02)   tensor ids 12, 13, 14
"""
from __future__ import annotations

import os
from dataclasses import dataclass, asdict

import numpy as np

TID_X, TID_W, TID_BIAS, TID_W1, TID_W3, TID_W2, TID_XE, TID_POP = 1, 2, 3, 4, 5, 6, 7, 8
TID_DOWN, TID_NORM, TID_UP, TID_SW1, TID_SW3, TID_SW2 = 9, 10, 11, 12, 13, 14
NORM_LO, NORM_HI = 0.5, 1.5

SIGMA_X = 1.0
SIGMA_W = 0.02
SIGMA_EXPERT = 0.02
BIAS_LO, BIAS_HI = -0.01, 0.01

_REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SKEW_BIAS_FILE = os.path.join(_REPO, "tests", "golden", "k2_skew_bias.txt")


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d_r: int
    d_e: int
    E: int
    G: int
    TG: int
    K: int
    F: int
    act: str            # "silu" or "situ"
    route_scale: float
    beta: float = 1.0   # SiTU beta
    lbeta: float = 0.0  # SiTU linear_beta; 0 means "not set"
    norm: bool = True   # norm_topk_prob
    latent: bool = False
    skew: bool = False
    seed: int = 0
    F_shared: int = 0       # whole-block workloads: shared experts' hidden width
    norm_eps: float = 1e-6  # whole-block workloads: routed_expert_norm epsilon

    @property
    def S(self) -> int:
        return self.N * self.K

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    "tiny": Workload("tiny", N=64, d_r=256, d_e=256, E=16, G=4, TG=2, K=4, F=128,
                     act="silu", route_scale=2.5),
    "dsv32_decode": Workload("dsv32_decode", N=128, d_r=7168, d_e=7168, E=256, G=8, TG=4, K=8,
                             F=2048, act="silu", route_scale=2.5),
    "k2_prefill": Workload("k2_prefill", N=4096, d_r=7168, d_e=7168, E=384, G=1, TG=1, K=8,
                           F=2048, act="silu", route_scale=2.827),
    "k3_latent_decode": Workload("k3_latent_decode", N=64, d_r=7168, d_e=2048, E=896, G=1, TG=1,
                                 K=8, F=3072, act="situ", route_scale=2.827, beta=4.0, lbeta=8.0,
                                 latent=True),
    "k2_skew": Workload("k2_skew", N=16384, d_r=7168, d_e=7168, E=384, G=1, TG=1, K=8, F=2048,
                        act="silu", route_scale=2.827, skew=True),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (e.g. fewer tokens)."""
    d = wl.as_dict()
    d.update(kw)
    return Workload(**d)


# The whole KimiSparseMoeBlock at the Kimi-K3 latent decode shape: x_e is the
# down projection of x (not a tensor of its own), then RMSNorm, up projection
# and one shared expert of width 3072 on the full 7168 width.
BLOCKS = {
    "k3_block_decode": scaled(WORKLOADS["k3_latent_decode"], name="k3_block_decode",
                              F_shared=3072),
    "tiny_block": Workload("tiny_block", N=64, d_r=256, d_e=128, E=16, G=4, TG=2, K=4, F=128,
                           act="situ", route_scale=2.5, beta=4.0, lbeta=8.0, latent=True,
                           F_shared=256),
}


# ------------------------------------------------------------------ host side
def skew_bias() -> np.ndarray:
    """Calibrated correction bias of the skewed workload (384 fp32 values)."""
    vals = []
    with open(SKEW_BIAS_FILE) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float.fromhex(line))
    return np.asarray(vals, dtype=np.float32)


def latent_x_e(wl: Workload, x: np.ndarray) -> np.ndarray:
    """x_e = bf16(x . P^T) for the latent workload: the routed experts see a
    down projection of the router's input (the workload's "down-projected
    x"); the projection P [d_e, d_r] is synthetic, fp32 ~ N(0, 1/d_r) with
    tensor id 7, so x_e ~ N(0, 1).  Input preparation, not the layer: the dot
    products are taken in double, rounded to fp32 and then to bf16 (nearest
    even).  x: bf16 bit patterns [n, d_r]; returns bf16 bit patterns."""
    from . import bf16_bits_to_f32, host_normal_f32
    P = host_normal_f32(wl.seed, TID_XE, (wl.d_e, wl.d_r), 1.0 / np.sqrt(wl.d_r))
    xf = bf16_bits_to_f32(x).astype(np.float64)
    y = (xf @ P.astype(np.float64).T).astype(np.float32)
    return _bf16_bits_rne(y).reshape(x.shape[0], wl.d_e)


def host_inputs(wl: Workload, rank: int = 0, n_tokens: int | None = None) -> dict:
    """Router-side inputs and x_e on the host (expert weights: ``host_expert``).
    n_tokens: only the first n_tokens rows of the rank's batch."""
    from . import host_normal_bf16, host_normal_f32, host_uniform_f32
    n = wl.N if n_tokens is None else min(int(n_tokens), wl.N)
    x = host_normal_bf16(wl.seed, TID_X, (n, wl.d_r), SIGMA_X, start=rank * wl.N * wl.d_r)
    W = host_normal_f32(wl.seed, TID_W, (wl.E, wl.d_r), SIGMA_W)
    if wl.skew:
        b = skew_bias()
        assert b.shape == (wl.E,)
    else:
        b = host_uniform_f32(wl.seed, TID_BIAS, (wl.E,), BIAS_LO, BIAS_HI)
    xe = latent_x_e(wl, x) if wl.latent else x
    return {"x": x, "W": W, "bias": b, "x_e": xe}


def host_expert(wl: Workload, e: int):
    """(w1 [F, d_e], w3 [F, d_e], w2 [d_e, F]) of expert e as bf16 bit patterns."""
    from . import host_normal_bf16
    n = wl.F * wl.d_e
    w1 = host_normal_bf16(wl.seed, TID_W1, (wl.F, wl.d_e), SIGMA_EXPERT, start=e * n)
    w3 = host_normal_bf16(wl.seed, TID_W3, (wl.F, wl.d_e), SIGMA_EXPERT, start=e * n)
    w2 = host_normal_bf16(wl.seed, TID_W2, (wl.d_e, wl.F), SIGMA_EXPERT, start=e * n)
    return w1, w3, w2


def host_experts_all(wl: Workload):
    """All experts stacked: w1, w3 [E, F, d_e], w2 [E, d_e, F] (small workloads only)."""
    from . import host_normal_bf16
    w1 = host_normal_bf16(wl.seed, TID_W1, (wl.E, wl.F, wl.d_e), SIGMA_EXPERT)
    w3 = host_normal_bf16(wl.seed, TID_W3, (wl.E, wl.F, wl.d_e), SIGMA_EXPERT)
    w2 = host_normal_bf16(wl.seed, TID_W2, (wl.E, wl.d_e, wl.F), SIGMA_EXPERT)
    return w1, w3, w2


# ---------------------------------------------------------------- device side
def dev_inputs(wl: Workload, rank: int = 0, device="cuda", experts: bool = True) -> dict:
    """All inputs as torch CUDA tensors, drawn by the device twin."""
    import torch
    from . import dev_normal_bf16, dev_normal_f32, dev_uniform_f32
    bf, f32 = torch.bfloat16, torch.float32
    x = dev_normal_bf16(torch.empty((wl.N, wl.d_r), dtype=bf, device=device), wl.seed, TID_X,
                        SIGMA_X, start=rank * wl.N * wl.d_r)
    W = dev_normal_f32(torch.empty((wl.E, wl.d_r), dtype=f32, device=device), wl.seed, TID_W,
                       SIGMA_W)
    if wl.skew:
        b = torch.from_numpy(skew_bias()).to(device)
    else:
        b = dev_uniform_f32(torch.empty((wl.E,), dtype=f32, device=device), wl.seed, TID_BIAS,
                            BIAS_LO, BIAS_HI)
    if wl.latent:
        # the down projection is computed once on the host (from the host
        # twin's identical x) and uploaded, so both sides see the same bits
        from . import host_normal_bf16
        xh = host_normal_bf16(wl.seed, TID_X, (wl.N, wl.d_r), SIGMA_X, start=rank * wl.N * wl.d_r)
        xe = torch.from_numpy(latent_x_e(wl, xh).view(np.int16)).to(device).view(bf)
    else:
        xe = x
    out = {"x": x, "W": W, "bias": b, "x_e": xe}
    if experts:
        out["w1"] = dev_normal_bf16(torch.empty((wl.E, wl.F, wl.d_e), dtype=bf, device=device),
                                    wl.seed, TID_W1, SIGMA_EXPERT)
        out["w3"] = dev_normal_bf16(torch.empty((wl.E, wl.F, wl.d_e), dtype=bf, device=device),
                                    wl.seed, TID_W3, SIGMA_EXPERT)
        out["w2"] = dev_normal_bf16(torch.empty((wl.E, wl.d_e, wl.F), dtype=bf, device=device),
                                    wl.seed, TID_W2, SIGMA_EXPERT)
    return out


# ------------------------------------------------------- the block around it
def _bf16_bits_rne(a: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def host_block(wl: Workload) -> dict:
    """Block weights on the host as bf16 bit patterns (down/up/norm absent
    unless latent, shared absent unless F_shared)."""
    from . import host_normal_bf16, host_uniform_f32
    out = {"down_proj": None, "norm_w": None, "up_proj": None, "shared": None}
    if wl.latent:
        out["down_proj"] = host_normal_bf16(wl.seed, TID_DOWN, (wl.d_e, wl.d_r), SIGMA_EXPERT)
        out["norm_w"] = _bf16_bits_rne(host_uniform_f32(wl.seed, TID_NORM, (wl.d_e,), NORM_LO,
                                                        NORM_HI))
        out["up_proj"] = host_normal_bf16(wl.seed, TID_UP, (wl.d_r, wl.d_e), SIGMA_EXPERT)
    if wl.F_shared:
        out["shared"] = (
            host_normal_bf16(wl.seed, TID_SW1, (wl.F_shared, wl.d_r), SIGMA_EXPERT),
            host_normal_bf16(wl.seed, TID_SW3, (wl.F_shared, wl.d_r), SIGMA_EXPERT),
            host_normal_bf16(wl.seed, TID_SW2, (wl.d_r, wl.F_shared), SIGMA_EXPERT))
    return out


def dev_block(wl: Workload, device="cuda") -> dict:
    """The same block weights drawn by the device twin (torch CUDA tensors)."""
    import torch
    from . import dev_normal_bf16, dev_uniform_f32
    bf = torch.bfloat16
    out = {"down_proj": None, "norm_w": None, "up_proj": None, "shared": None}

    def nrm(tid, shape):
        return dev_normal_bf16(torch.empty(shape, dtype=bf, device=device), wl.seed, tid,
                               SIGMA_EXPERT)
    if wl.latent:
        out["down_proj"] = nrm(TID_DOWN, (wl.d_e, wl.d_r))
        u = dev_uniform_f32(torch.empty((wl.d_e,), dtype=torch.float32, device=device), wl.seed,
                            TID_NORM, NORM_LO, NORM_HI)
        out["norm_w"] = u.to(bf)  # round to nearest even, as the host twin
        out["up_proj"] = nrm(TID_UP, (wl.d_r, wl.d_e))
    if wl.F_shared:
        out["shared"] = (nrm(TID_SW1, (wl.F_shared, wl.d_r)), nrm(TID_SW3, (wl.F_shared, wl.d_r)),
                         nrm(TID_SW2, (wl.d_r, wl.F_shared)))
    return out
