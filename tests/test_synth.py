"""The seeded input generator: reproducible, sliceable, right distribution, and
the device twin bit-identical to the host twin."""
import numpy as np
import pytest

import synth
from synth.workloads import WORKLOADS, host_inputs


def test_reproducible_and_sliceable():
    a = synth.host_normal_f32(0, 4, (100_000,), 0.02)
    b = synth.host_normal_f32(0, 4, (100_000,), 0.02)
    assert np.array_equal(a, b)
    s = synth.host_normal_f32(0, 4, (1000,), 0.02, start=54_321)
    assert np.array_equal(s, a[54_321:55_321])
    c = synth.host_normal_f32(1, 4, (1000,), 0.02)
    assert not np.array_equal(c, a[:1000])
    d = synth.host_normal_f32(0, 5, (1000,), 0.02)
    assert not np.array_equal(d, a[:1000])


def test_normal_moments():
    z = synth.host_normal_f32(0, 1, (2_000_000,), 1.0).astype(np.float64)
    assert abs(z.mean()) < 3e-3
    assert abs(z.std() - 1.0) < 3e-3
    # Irwin-Hall(8): bounded, excess kurtosis -6/(5*8) = -0.15
    k = ((z - z.mean()) ** 4).mean() / z.var() ** 2 - 3.0
    assert abs(k + 0.15) < 0.02
    assert np.abs(z).max() < np.sqrt(24.0) + 1e-3


def test_uniform_range():
    u = synth.host_uniform_f32(0, 3, (1_000_000,), -0.01, 0.01).astype(np.float64)
    assert u.min() >= -0.01 and u.max() < 0.01
    assert abs(u.mean()) < 5e-5
    assert abs(u.std() - 0.02 / np.sqrt(12)) < 5e-5


def test_bf16_is_nearest_even_of_fp32():
    import torch
    f = synth.host_normal_f32(0, 6, (200_000,), 0.02)
    b = synth.host_normal_bf16(0, 6, (200_000,), 0.02)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(b, ref)


def test_workload_inputs_shapes():
    wl = WORKLOADS["tiny"]
    inp = host_inputs(wl)
    assert inp["x"].shape == (64, 256) and inp["x"].dtype == np.uint16
    assert inp["W"].shape == (16, 256) and inp["W"].dtype == np.float32
    assert inp["bias"].shape == (16,)
    assert inp["x_e"] is inp["x"]
    wl4 = WORKLOADS["k3_latent_decode"]
    assert wl4.latent and wl4.d_e == 2048 and wl4.d_r == 7168


def test_rank_slices_are_disjoint_rows_of_one_tensor():
    wl = WORKLOADS["tiny"]
    r0 = host_inputs(wl, rank=0)["x"]
    r1 = host_inputs(wl, rank=1)["x"]
    both = synth.host_normal_bf16(0, synth.TID_X, (2 * wl.N, wl.d_r), 1.0)
    assert np.array_equal(both[:wl.N], r0) and np.array_equal(both[wl.N:], r1)


@pytest.mark.gpu
def test_device_twin_bit_identical():
    import torch
    for (start, n) in [(0, 1 << 20), (123_456_789, 100_003)]:
        hb = synth.host_normal_bf16(7, 4, (n,), 0.02, start=start)
        db = synth.dev_normal_bf16(torch.empty(n, dtype=torch.bfloat16, device="cuda"), 7, 4,
                                   0.02, start=start)
        assert np.array_equal(db.view(torch.int16).cpu().numpy().astype(np.uint16), hb)
        hf = synth.host_normal_f32(7, 2, (n,), 0.02, start=start)
        df = synth.dev_normal_f32(torch.empty(n, dtype=torch.float32, device="cuda"), 7, 2, 0.02,
                                  start=start)
        assert np.array_equal(df.cpu().numpy().view(np.uint32), hf.view(np.uint32))
        hu = synth.host_uniform_f32(7, 3, (n,), -0.01, 0.01, start=start)
        du = synth.dev_uniform_f32(torch.empty(n, dtype=torch.float32, device="cuda"), 7, 3,
                                   -0.01, 0.01, start=start)
        assert np.array_equal(du.cpu().numpy().view(np.uint32), hu.view(np.uint32))


def test_latent_x_e_is_the_down_projection_of_x():
    """The latent workload's x_e is bf16(x . P^T) with P [d_e, d_r] drawn with
    tensor id 7 and sigma 1/sqrt(d_r): entries checked against the exact
    rational dot product (rounded to fp32, then to bf16), and the whole
    tensor is about N(0, 1)."""
    from fractions import Fraction
    wl = WORKLOADS["k3_latent_decode"]
    inp = host_inputs(wl)
    x, xe = inp["x"], inp["x_e"]
    assert xe.shape == (wl.N, wl.d_e) and xe.dtype == np.uint16
    P = synth.host_normal_f32(wl.seed, synth.TID_XE, (wl.d_e, wl.d_r), 1.0 / np.sqrt(wl.d_r))
    xf = synth.bf16_bits_to_f32(x)
    for t, j in [(0, 0), (3, 17), (63, 2047), (40, 1000)]:
        exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], P[j]))
        f32 = np.float32(float(exact))
        want = int(np.asarray([f32]).view(np.uint32)[0])
        want = (want + 0x7FFF + ((want >> 16) & 1)) >> 16
        assert int(xe[t, j]) == want, (t, j)
    v = synth.bf16_bits_to_f32(xe).astype(np.float64)
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1.0) < 0.03
    # the first rows alone are the first rows of the whole batch
    part = host_inputs(wl, n_tokens=5)
    assert np.array_equal(part["x_e"], xe[:5]) and np.array_equal(part["x"], x[:5])
