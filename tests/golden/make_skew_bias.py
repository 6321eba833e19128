"""Write ``k2_skew_bias.txt``: the correction bias of the skewed Kimi-K2-shaped
stress workload (N=16384, d=7168, 384 experts, top-8).

The workload asks for Zipf(s=1.2) expert popularity with at least 20 experts
that receive no token.  The bias is calibrated once, with the CPU reference
only (gate logits and routing), and stored; both the CUDA path and the
reference then read the stored values as an input.

Recipe:
  1. Popularity ranks: experts sorted by a seeded 64-bit draw (tensor id 8).
  2. Target slot shares q_r proportional to r^-1.2 for ranks 1..364, capped at
     1/K (an expert is picked at most once per token) by water-filling; the 20
     experts of ranks 365..384 get share 0.
  3. Calibration batch: 8192 tokens drawn with seed 1, the workload's gate
     weight W (seed 0); logits computed once.
  4. 2000 sign steps: route top-8 of (sigmoid + b) and move
     b_e += 1e-3 * sign(q_e - load_e).
  5. The 20 zero-share experts get min(b) - 2, so they can never be chosen.
  6. Validation on the workload's own batch (seed 0, 16384 tokens): count of
     experts with no token and the slot share of the top 10% of experts,
     written into the file header.

Zipf(1.2) over 364 experts with the 1/K cap gives the top 10% of experts about
three quarters of the slots, not one half: the two numbers in the workload
description cannot both hold, and the named exponent is the one kept.

Run: python -m tests.golden.make_skew_bias   (a few minutes on 8 cores)
"""
from __future__ import annotations

import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402
from synth.workloads import WORKLOADS, SIGMA_W, SIGMA_X, TID_POP, TID_W, TID_X  # noqa: E402

OUT = os.path.join(HERE, "k2_skew_bias.txt")
ZIPF_S = 1.2
N_ZERO = 20
N_CAL = 8192
ITERS = 2000
STEP = 1e-3


def target_shares(E: int, K: int) -> np.ndarray:
    """Share of slots per popularity rank (index 0 = rank 1)."""
    n_pos = E - N_ZERO
    q = np.arange(1, n_pos + 1, dtype=np.float64) ** -ZIPF_S
    q /= q.sum()
    cap = 1.0 / K
    fixed = np.zeros(n_pos, bool)
    for _ in range(n_pos):
        over = (q > cap) & ~fixed
        if not over.any():
            break
        fixed |= over
        q[fixed] = cap
        rest = ~fixed
        q[rest] *= (1.0 - cap * fixed.sum()) / q[rest].sum()
    return np.concatenate([q, np.zeros(N_ZERO)])


def main() -> None:
    wl = WORKLOADS["k2_skew"]
    E, K, d = wl.E, wl.K, wl.d_r
    oracle.set_threads(os.cpu_count() or 1)
    raw = synth.host_raw(wl.seed, TID_POP, E)
    by_rank = np.argsort(raw, kind="stable")           # by_rank[r] = expert of rank r+1
    q_rank = target_shares(E, K)
    q = np.empty(E)
    q[by_rank] = q_rank
    W = synth.host_normal_f32(wl.seed, TID_W, (E, d), SIGMA_W)
    x_cal = synth.host_normal_bf16(1, TID_X, (N_CAL, d), SIGMA_X)
    L_cal = oracle.gate_logits(x_cal, W)
    b = np.zeros(E, np.float32)
    for it in range(ITERS):
        idx, _, _ = oracle.route_from_logits(L_cal, b, 1, 1, K, wl.route_scale)
        load = np.bincount(idx.ravel(), minlength=E) / float(N_CAL * K)
        b = (b + np.float32(STEP) * np.sign(q - load).astype(np.float32)).astype(np.float32)
        if it % 250 == 0:
            print(f"iter {it}: max |q-load| = {np.abs(q - load).max():.4f}", flush=True)
    zero = by_rank[E - N_ZERO:]
    b[zero] = np.float32(b.min() - np.float32(2.0))
    # validation on the workload's own batch
    x0 = synth.host_normal_bf16(wl.seed, TID_X, (wl.N, d), SIGMA_X)
    idx0, _, _ = oracle.route(x0, W, b, 1, 1, K, wl.route_scale)
    cnt = np.bincount(idx0.ravel(), minlength=E)
    n_zero = int((cnt == 0).sum())
    top10 = float(np.sort(cnt)[::-1][: int(round(0.1 * E))].sum() / cnt.sum())
    body = "".join(f"{float(v).hex()}\n" for v in b)
    sha = hashlib.sha256(body.encode()).hexdigest()
    with open(OUT, "w") as f:
        f.write("# correction bias of the skewed K2-shaped workload (384 fp32, hex)\n")
        f.write(f"# Zipf s={ZIPF_S}, {N_ZERO} forced zero experts, {ITERS} sign steps of {STEP}\n")
        f.write(f"# validation on seed-0 batch (N={wl.N}): experts with no token = {n_zero}, "
                f"top-10% slot share = {top10:.4f}, max expert load = {int(cnt.max())}\n")
        f.write(f"# sha256 of the value lines: {sha}\n")
        f.write(body)
    print(f"wrote {OUT}: zero={n_zero} top10={top10:.4f} max={cnt.max()} sha256={sha}")


if __name__ == "__main__":
    main()
