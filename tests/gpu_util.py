"""Helpers for the GPU parity tests: moving bf16 bit patterns between numpy and
torch, comparison metrics, and the parity tolerances."""
from __future__ import annotations

import numpy as np

# Tolerances of the parity contract.
REL_L2_OUT = 2e-2     # layer / expert outputs, relative L2 in bf16
W_REL = 1e-5          # routing weights (end to end, aligned by expert id)
MARGIN = 1e-5         # biased-score margin above which end-to-end indices must match


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(a_bits: np.ndarray) -> np.ndarray:
    return (a_bits.astype(np.uint32) << 16).view(np.float32)


def rel_l2(got_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    g = f32(got_bits).astype(np.float64)
    r = f32(ref_bits).astype(np.float64)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / (den if den > 0 else 1.0))


def ulp_diff(got_bits: np.ndarray, ref_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place (sign-magnitude aware)."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), b + 0x8000)
    return np.abs(ordered(got_bits) - ordered(ref_bits))


def random_topk(N: int, K: int, E: int, rng, skew: float = 0.0) -> np.ndarray:
    """Distinct expert ids per token; skew > 0 draws with Zipf-like popularity."""
    if skew > 0:
        p = np.arange(1, E + 1, dtype=np.float64) ** -skew
        p /= p.sum()
        keys = rng.random((N, E)) ** (1.0 / p)[None, :]  # weighted sampling w/o replacement
        return np.argsort(-keys, axis=1)[:, :K].astype(np.int32)
    keys = rng.random((N, E))
    return np.argsort(keys, axis=1)[:, :K].astype(np.int32)


def oracle_layer_tokens(wl, xe_rows: np.ndarray, idx: np.ndarray, w: np.ndarray,
                        workers: int | None = None) -> np.ndarray:
    """The reference layer output of a few tokens: out[i] = combine over k of
    expert_ffn(idx[i, k]) on xe_rows[i], weighted by w[i, k] -- the per-token
    loop of moe_infer.  Tokens are grouped by expert so that each expert's
    weights are drawn once; experts run in a thread pool (the reference's C
    calls release the GIL), each call single-threaded.  Bit-identical to the
    same loop run serially: every row's arithmetic is independent."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from synth.workloads import host_expert

    n, K = idx.shape
    by_e: dict[int, list[tuple[int, int]]] = {}
    for i in range(n):
        for k in range(K):
            by_e.setdefault(int(idx[i, k]), []).append((i, k))
    ys = np.zeros((n, K, xe_rows.shape[1]), np.uint16)

    def run(e):
        oracle.set_threads(1)  # this thread's OpenMP team (the generator's too)
        slots = by_e[e]
        w1, w3, w2 = host_expert(wl, e)
        rows = np.ascontiguousarray(xe_rows[[i for i, _ in slots]])
        y = oracle.expert_ffn(rows, w1, w3, w2, wl.act, wl.beta, wl.lbeta)
        for (i, k), r in zip(slots, y):
            ys[i, k] = r

    with ThreadPoolExecutor(max_workers=workers or os.cpu_count() or 1) as ex:
        list(ex.map(run, sorted(by_e)))
    out = np.zeros((n, xe_rows.shape[1]), np.uint16)
    for i in range(n):
        out[i] = oracle.combine(ys[i], np.arange(K, dtype=np.int32),
                                np.ascontiguousarray(w[i:i + 1]), K)[0]
    return out


def ulp_stats(got_bits: np.ndarray, ref_bits: np.ndarray) -> dict:
    """Fraction of outputs within 0, 1 and 2 bf16 ulp of the reference, and the
    largest distance."""
    u = ulp_diff(got_bits, ref_bits)
    return {"n": int(u.size), "eq": float((u == 0).mean()), "le1": float((u <= 1).mean()),
            "le2": float((u <= 2).mean()), "max": int(u.max()) if u.size else 0}


# Bars on the bf16 outputs of the expert MLP and of the layer, beside the
# contract's 2e-2 relative L2 over the whole sample.  They are set from what
# the kernels reach against the double-accumulated reference (fp32 tensor-core
# accumulation flips the bf16 rounding of g, u and y now and then, more often
# the longer the dot products) and are tight enough that a corrupted row, a
# tile's tail, one 128-column weight block or a single wrong column fails:
ROW_REL_L2 = 1e-2       # every sampled row: ||y - y_ref|| / ||y_ref||
ELEM_OF_RMS = 0.125     # every element: |y - y_ref| <= 0.125 * rms(y_ref row)
ULP1_SHORT, ULP1_LONG = 0.995, 0.95   # fraction within 1 bf16 ulp (d, F <= 512 / longer)
ULP2_LONG = 0.97                      # fraction within 2 ulp, longer dot products
# the layer output sums K such expert rows, so its figures sit a little lower
ULP1_LAYER_LONG, ULP2_LAYER_LONG = 0.94, 0.96


def row_errors(got_bits: np.ndarray, ref_bits: np.ndarray):
    """Per-row relative L2 and per-row largest |error| / rms(reference row)."""
    g = f32(got_bits).astype(np.float64).reshape(-1, got_bits.shape[-1])
    r = f32(ref_bits).astype(np.float64).reshape(-1, ref_bits.shape[-1])
    nr = np.linalg.norm(r, axis=1)
    rms = nr / np.sqrt(r.shape[1])
    rel = np.linalg.norm(g - r, axis=1) / np.where(nr > 0, nr, 1.0)
    emax = np.abs(g - r).max(axis=1) / np.where(rms > 0, rms, 1.0)
    return rel, emax


def check_bf16_outputs(got_bits: np.ndarray, ref_bits: np.ndarray, long_dots: bool,
                       what: str = "", layer: bool = False, ulp_bars: bool = True) -> dict:
    """Asserts the output bars above (relative L2 over the sample, per row,
    per element, ulp fractions) and returns the measured figures.
    ulp_bars=False leaves the ulp fractions out: for the whole block, whose
    output is a Linear over inputs that already carry the routed layer's
    rounding, the per-row and per-element bars are the meaningful ones."""
    rel, emax = row_errors(got_bits, ref_bits)
    st = ulp_stats(got_bits, ref_bits)
    st.update({"rel_l2": rel_l2(got_bits, ref_bits), "row_rel_max": float(rel.max()),
               "elem_of_rms_max": float(emax.max())})
    print(f"bars {what}: {st}")
    assert st["rel_l2"] <= REL_L2_OUT, st
    assert st["row_rel_max"] <= ROW_REL_L2, st
    assert st["elem_of_rms_max"] <= ELEM_OF_RMS, st
    if not ulp_bars:
        pass
    elif long_dots and layer:
        assert st["le1"] >= ULP1_LAYER_LONG and st["le2"] >= ULP2_LAYER_LONG, st
    elif long_dots:
        assert st["le1"] >= ULP1_LONG and st["le2"] >= ULP2_LONG, st
    else:
        assert st["le1"] >= ULP1_SHORT, st
    return st
