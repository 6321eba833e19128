"""The C-ABI library loads without a GPU, exports every entry point its header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    from moe_routing_expert_fp32_b200 import build as b
    b.build()
    import moe_routing_expert_fp32_b200 as m
    return m.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_forward",
              "moe_route_from_logits", "moe_workspace_size", "moe_get_status", "moe_strerror"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in moe.h but not exported"


def test_binding_names_match_the_header():
    import moe_routing_expert_fp32_b200 as m
    assert set(m.EXPORTS) <= set(declared_functions())


def _cfg(m, E=16, G=4, TG=2, K=4, rs=2.5):
    return m._RouteCfg(E, G, TG, K, 1, rs)


@pytest.mark.parametrize("E,G,TG,K,code", [
    (16, 4, 2, 4, -4),    # valid config; fails on the NULL workspace, not on the config
    (16, 3, 2, 4, -1),    # E not divisible by G
    (16, 4, 5, 4, -1),    # TG > G
    (16, 4, 1, 5, -1),    # K > TG * E / G
    (16, 16, 2, 2, -1),   # one expert per group with G > 1
    (2048, 1, 1, 8, -2),  # E > 1024
    (64, 64, 2, 2, -1),   # G > 32 is checked after E/G >= 2 ... E/G = 1 -> invalid
    (16, 1, 1, 17, -1),   # K > E
    (32, 1, 1, 17, -2),   # K > 16
    (0, 1, 1, 1, -1),
])
def test_route_config_validation(L, E, G, TG, K, code):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m, E, G, TG, K)
    rc = L.moe_route(None, 4, 256, None, None, ctypes.byref(c), None, None, None, 0, None)
    if code == -4:
        assert rc == -1  # NULL tensors with N > 0 are caught first
    else:
        assert rc == code


def test_route_rejects_before_cuda(L):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m)
    assert L.moe_route(None, -1, 256, None, None, ctypes.byref(c), None, None, None, 0, None) == -1
    assert L.moe_route(None, 4, 100, None, None, ctypes.byref(c), None, None, None, 0, None) == -2
    assert L.moe_route(None, 4, 256, None, None, None, None, None, None, 0, None) == -1
    # N = 0 with a NULL workspace: workspace error, no CUDA call
    assert L.moe_route(None, 0, 256, None, None, ctypes.byref(c), None, None, None, 0, None) == -4
    c.route_scale = float("inf")
    assert L.moe_route(None, 4, 256, None, None, ctypes.byref(c), None, None, None, 0, None) == -1


@pytest.mark.parametrize("field,value,code", [
    ("score_func", 1, -4), ("group_score", 1, -4),    # valid variants: NULL workspace next
    ("score_func", 2, -1), ("score_func", -1, -1), ("group_score", 2, -1),
])
def test_route_variant_validation(L, field, value, code):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m)
    setattr(c, field, value)
    assert L.moe_route(None, 0, 256, None, None, ctypes.byref(c), None, None, None, 0, None) == code
    assert L.moe_route_from_logits(None, 0, None, ctypes.byref(c), None, None, None, 0,
                                   None) == code


def test_route_config_binding_defaults():
    import moe_routing_expert_fp32_b200 as m
    c = m.RouteConfig(16, 4, 2, 4, 2.5)._c()
    assert (c.score_func, c.group_score, c.norm_topk_prob) == (0, 0, 1)
    c = m.RouteConfig(16, 4, 2, 4, 2.5, False, score_func="softmax", group_score="max")._c()
    assert (c.score_func, c.group_score, c.norm_topk_prob) == (1, 1, 0)


def test_workspace_checks(L):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m)
    need = L.moe_route_workspace_size(64, 256, ctypes.byref(c))
    assert need >= 256 + 64 * 16 * 4
    buf = (ctypes.c_uint8 * (need + 512))()
    base = ctypes.addressof(buf)
    aligned = (base + 255) // 256 * 256
    # too small
    rc = L.moe_route(ctypes.c_void_p(16), 64, 256, ctypes.c_void_p(16), None, ctypes.byref(c),
                     ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(aligned), need - 1,
                     None)
    assert rc == -4
    # misaligned
    rc = L.moe_route(ctypes.c_void_p(16), 64, 256, ctypes.c_void_p(16), None, ctypes.byref(c),
                     ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(aligned + 16),
                     need, None)
    assert rc == -4
    # misaligned tensor
    rc = L.moe_route(ctypes.c_void_p(18), 64, 256, ctypes.c_void_p(16), None, ctypes.byref(c),
                     ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(aligned), need,
                     None)
    assert rc == -3


def test_expert_ffn_shape_limits(L):
    import moe_routing_expert_fp32_b200 as m
    a = m._ActCfg(0, 1.0, 0.0)
    p = ctypes.c_void_p(256)
    # d_e not a multiple of 128
    assert L.moe_expert_ffn(p, p, 4, 16, 100, 128, p, p, p, ctypes.byref(a), p, p, 1 << 20,
                            None) == -2
    # F not a multiple of 128
    assert L.moe_expert_ffn(p, p, 4, 16, 128, 96, p, p, p, ctypes.byref(a), p, p, 1 << 20,
                            None) == -2
    bad = m._ActCfg(7, 1.0, 0.0)
    assert L.moe_expert_ffn(p, p, 4, 16, 128, 128, p, p, p, ctypes.byref(bad), p, p, 1 << 20,
                            None) == -1
    assert L.moe_expert_ffn(p, p, 4, 16, 128, 128, None, p, p, ctypes.byref(a), p, p, 1 << 20,
                            None) == -1


def test_dispatch_and_combine_validation(L):
    p = ctypes.c_void_p(256)
    assert L.moe_dispatch(p, 4, 0, 16, p, 256, p, p, p, p, p, p, 1 << 20, None) == -1
    assert L.moe_dispatch(p, 4, 17, 16, p, 256, p, p, p, p, p, p, 1 << 20, None) == -2
    assert L.moe_dispatch(p, 4, 4, 16, p, 250, p, p, p, p, p, p, 1 << 20, None) == -2
    assert L.moe_combine(p, p, p, 4, 4, 250, p, p, 256, None) == -2
    assert L.moe_combine(None, p, p, 4, 4, 256, p, p, 256, None) == -1


def test_forward_validation(L):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m)
    a = m._ActCfg(0, 1.0, 0.0)
    p = ctypes.c_void_p(256)
    # x_e NULL but d_e != d_r
    assert L.moe_forward(p, None, 4, 256, 128, p, None, ctypes.byref(c), p, p, p, 128,
                         ctypes.byref(a), p, None, None, p, 1 << 30, None, None) == -1
    sz = L.moe_workspace_size(64, 256, 256, ctypes.byref(c), 128)
    assert sz > 64 * 4 * 256 * 2 * 2  # holds xs and y


def test_strerror(L):
    for code in range(-8, 1):
        assert L.moe_strerror(code)
    assert L.moe_strerror(-99) == b"unknown moe_status"


def _block_args(m, d_r=256, d_e=128, F=128, F_sh=256, latent=True, shared=True, norm=True):
    dims = m._BlockDims(d_r, d_e, F, F_sh if shared else 0, 1e-6)
    p = ctypes.c_void_p(256)  # never dereferenced: validation only
    w = m._BlockWeights(p, None, p if latent else None, p if (latent and norm) else None,
                        p if latent else None, p, p, p, p if shared else None,
                        p if shared else None, p if shared else None)
    return dims, w


@pytest.mark.parametrize("kw,ok", [
    ({}, True),
    ({"shared": False}, True),
    ({"norm": False}, True),
    ({"latent": False, "d_e": 256, "norm": False}, True),
    ({"latent": False, "d_e": 128, "norm": False}, False),   # d_e != d_r without projections
    ({"d_r": 200}, False),                                    # d_r not a multiple of 128
    ({"F_sh": 100}, False),
    ({"d_e": 16384, "d_r": 16384}, False),                    # latent width above 8192
])
def test_block_workspace_validation(L, kw, ok):
    import moe_routing_expert_fp32_b200 as m
    dims, w = _block_args(m, **kw)
    c = _cfg(m)
    need = L.moe_block_workspace_size(64, ctypes.byref(dims), ctypes.byref(w), ctypes.byref(c))
    assert (need > 0) == ok


def test_block_rejects_inconsistent_parts(L):
    import moe_routing_expert_fp32_b200 as m
    c = _cfg(m)
    a = m._ActCfg(0, 1.0, 0.0)
    dims, w = _block_args(m)
    w.up_proj = None                       # down_proj without up_proj
    assert L.moe_block_forward(None, 0, ctypes.byref(dims), ctypes.byref(w), ctypes.byref(c),
                               ctypes.byref(a), None, None, None, None, 0, None) == -1
    dims, w = _block_args(m)
    w.shared_w2 = None                     # a partial shared expert
    assert L.moe_block_forward(None, 0, ctypes.byref(dims), ctypes.byref(w), ctypes.byref(c),
                               ctypes.byref(a), None, None, None, None, 0, None) == -1
    dims, w = _block_args(m)
    dims.norm_eps = float("nan")
    assert L.moe_block_forward(None, 0, ctypes.byref(dims), ctypes.byref(w), ctypes.byref(c),
                               ctypes.byref(a), None, None, None, None, 0, None) == -1
    dims, w = _block_args(m)               # valid: fails on the NULL workspace only
    assert L.moe_block_forward(None, 0, ctypes.byref(dims), ctypes.byref(w), ctypes.byref(c),
                               ctypes.byref(a), None, None, None, None, 0, None) == -4


def test_linear_and_norm_validation(L):
    assert L.moe_linear_workspace_size(64, 7168, 2048) > 512       # split-K partials
    assert L.moe_linear_workspace_size(4096, 7168, 2048) == 512    # fills the GPU: no split
    assert L.moe_linear_workspace_size(64, 100, 2048) == 0
    # K and N_out must be multiples of 128
    assert L.moe_linear(None, 0, 100, ctypes.c_void_p(256), 128, None, None, None, 0, None) == -2
    assert L.moe_linear(None, 0, 128, None, 128, None, None, None, 0, None) == -1
    assert L.moe_linear(None, 0, 128, ctypes.c_void_p(258), 128, None, None, None, 0, None) == -3
    assert L.moe_linear(None, 0, 128, ctypes.c_void_p(256), 128, None, None, None, 0, None) == -4
    # RMSNorm: negative or NaN eps, widths
    w = ctypes.c_void_p(256)
    assert L.moe_rms_norm(None, 0, 128, w, -1.0, None, None) == -1
    assert L.moe_rms_norm(None, 0, 128, w, float("nan"), None, None) == -1
    assert L.moe_rms_norm(None, 0, 100, w, 1e-6, None, None) == -2
    assert L.moe_rms_norm(None, 0, 16384, w, 1e-6, None, None) == -2
    assert L.moe_rms_norm(None, 4, 128, w, 1e-6, None, None) == -1


def test_ep_expert_ffn_validation(L):
    import moe_routing_expert_fp32_b200 as m
    a = m._ActCfg(0, 1.0, 0.0)
    p = ctypes.c_void_p(256)
    assert L.moe_ep_expert_ffn_workspace_size(100, 256, 2, 8, 128) > 256
    assert L.moe_ep_expert_ffn_workspace_size(100, 256, 0, 8, 128) == 0
    # P * E_local above 1024
    assert L.moe_ep_expert_ffn(None, 0, p, 64, 32, 256, 128, p, p, p, ctypes.byref(a), None, None,
                               0, None) == -2
    # missing counts, bad widths, NULL workspace
    assert L.moe_ep_expert_ffn(None, 0, None, 2, 8, 256, 128, p, p, p, ctypes.byref(a), None, None,
                               0, None) == -1
    assert L.moe_ep_expert_ffn(None, 0, p, 2, 8, 200, 128, p, p, p, ctypes.byref(a), None, None,
                               0, None) == -2
    assert L.moe_ep_expert_ffn(None, 0, p, 2, 8, 256, 128, p, p, p, ctypes.byref(a), None, None,
                               0, None) == -4


def test_launch_count_is_exported_and_starts_without_gpu_work(L):
    """moe_launch_count is the library's own tally of accepted kernel launches;
    calls rejected on the host add nothing to it."""
    before = L.moe_launch_count()
    assert L.moe_combine(None, None, None, 4, 0, 128, None, None, 0, None) == -1  # K = 0
    assert L.moe_launch_count() == before


def _dispatch_chunks(S):
    """Chunk count of the stable sort as moe_dispatch_static's comment in
    include/moe.h states it: chunk length clamp(S/256, 64, 1024) rounded up
    to a multiple of 32."""
    ch = min(max(S // 256, 64), 1024)
    ch = (ch + 31) // 32 * 32
    return (S + ch - 1) // ch


@pytest.mark.parametrize("N,K,E", [(1, 1, 1), (64, 4, 16), (128, 8, 256), (4096, 8, 384),
                                   (16384, 8, 384), (100000, 6, 1024), (3, 16, 1000)])
def test_dispatch_workspace_follows_the_documented_chunking(L, N, K, E):
    """The workspace holds the 256-byte status word and 4 * chunks * E bytes
    of per-chunk counts (256-byte aligned); the static entry point's 2 MiB
    limit is stated in the same terms."""
    counts = 4 * _dispatch_chunks(N * K) * E
    assert L.moe_dispatch_workspace_size(N, K, E) == 256 + (counts + 255) // 256 * 256
    if counts > (2 << 20):
        # rejected on the host, before any device work (the pointers are fake)
        p = ctypes.c_void_p(256)
        assert L.moe_dispatch_static(p, N, K, E, p, 128, p, p, p, p, p, None) == -2


def test_bench_roofline_picks_the_binding_peak():
    """The bench's w1/w3 roofline object is HBM-bound for the decode and
    prefill workloads and tensor-bound for the skewed one, with achieved /
    peak computed against the matching measured figure."""
    import bench
    from synth.workloads import WORKLOADS
    peaks = {"hbm_gbs": 6546.9, "bf16_tflops": 1676.5, "bf16_tflops_sustained": 1374.1,
             "source": "measured"}
    dec = bench.gate_up_roofline(WORKLOADS["dsv32_decode"], 252, 2.17, peaks)
    assert dec["bound"] == "hbm" and dec["unit"] == "GB/s"
    assert abs(dec["achieved"] - 14.82e9 / 2.17e-3 / 1e9) / dec["achieved"] < 0.01
    assert abs(dec["frac"] - dec["achieved"] / 6546.9) < 1e-12
    pre = bench.gate_up_roofline(WORKLOADS["k2_prefill"], 384, 3.5, peaks)
    assert pre["bound"] == "hbm"
    skew = WORKLOADS["k2_skew"]
    sk = bench.gate_up_roofline(skew, 364, 8.8, peaks)
    assert sk["bound"] == "tensor" and sk["unit"] == "TFLOP/s"
    assert sk["traffic"] is None or sk["traffic"] > 0
    flops = 4 * skew.N * skew.K * skew.F * skew.d_e
    assert abs(sk["achieved"] - flops / 8.8e-3 / 1e12) < 1e-9
    assert abs(sk["frac"] - sk["achieved"] / 1374.1) < 1e-12


def test_bench_traffic_records(tmp_path):
    """gate_up_traffic: an HBM-bound launch scales the decode-shaped record by
    touched experts; a tensor-bound one takes only the record of the same
    workload and sizes; a record whose kernel source hash no longer matches
    gives None."""
    import hashlib, json, bench
    from synth.workloads import WORKLOADS, scaled
    src = "bench.py"
    with open(os.path.join(bench.ROOT, src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    skew = WORKLOADS["k2_skew"]
    recs = [{"workload": "dsv32_decode", "source": src, "source_sha256": sha,
             "touched_experts": 10, "dram_bytes_read": 1000, "dram_bytes_write": 24,
             "scaling": "touched"},
            {"workload": "k2_skew", "N": skew.N, "E": skew.E, "source": src,
             "source_sha256": sha, "touched_experts": 364, "dram_bytes_read": 5000,
             "dram_bytes_write": 7, "scaling": "same-workload"}]
    p = tmp_path / "t.json"
    p.write_text(json.dumps({"records": recs}))
    assert bench.gate_up_traffic(WORKLOADS["dsv32_decode"], 30, "hbm", str(p)) == 3 * 1024
    assert bench.gate_up_traffic(skew, 364, "tensor", str(p)) == 5007
    assert bench.gate_up_traffic(scaled(skew, N=8192), 300, "tensor", str(p)) is None
    assert bench.gate_up_traffic(WORKLOADS["k2_prefill"], 384, "tensor", str(p)) is None
    recs[1]["source_sha256"] = "0" * 64
    p.write_text(json.dumps({"records": recs}))
    assert bench.gate_up_traffic(skew, 364, "tensor", str(p)) is None
    # several source files: the hash covers all of them, in order
    two = [src, "__graft_entry__.py"]
    recs[1]["source"] = two
    recs[1]["source_sha256"] = bench.source_sha256(two)
    p.write_text(json.dumps({"records": recs}))
    assert bench.gate_up_traffic(skew, 364, "tensor", str(p)) == 5007
    recs[1]["source"] = two[::-1]
    p.write_text(json.dumps({"records": recs}))
    assert bench.gate_up_traffic(skew, 364, "tensor", str(p)) is None


def test_ep_rows_validation(L):
    """moe_ep_dispatch_rows / moe_ep_combine_rows reject bad arguments on the
    host, before any device work (the pointers here are fake)."""
    import moe_routing_expert_fp32_b200 as m
    p = ctypes.c_void_p(256)
    ws = ctypes.c_void_p(1 << 20)

    def table(P, rows=256, cap=10, first=0):
        return m.peer_rows([rows] * P, [first] * P, [cap] * P)

    def disp(t, E=8, K=2, d=128, x=p, pos=p, offs=p, w=ws, wb=256):
        return L.moe_ep_dispatch_rows(x, 4, K, d, pos, offs, E, ctypes.byref(t), w, wb, None)

    def comb(t, E=8, K=2, d=128, out=p, tw=p, w=ws, wb=256):
        return L.moe_ep_combine_rows(ctypes.byref(t), p, p, E, tw, 4, K, d, out, w, wb, None)

    for f in (disp, comb):
        assert f(table(3)) == -1                    # 8 experts do not split over 3 ranks
        t = table(2)
        t.num_ranks = 0
        assert f(t) == -2                           # no ranks
        t.num_ranks = 65
        assert f(t) == -2                           # more than MOE_MAX_PEERS
        assert f(table(2, rows=None)) == -1         # capacity without a buffer
        assert f(table(2, rows=264)) == -3          # buffer not 16-byte aligned
        assert f(table(2, cap=-1)) == -1
        assert f(table(2, first=-1)) == -1
        assert f(table(2), K=17) == -2
        assert f(table(2), d=100) == -2
        assert f(table(2), w=None) == -4            # no workspace
        assert f(table(2), wb=8) == -4              # workspace too small
    assert disp(table(2), x=None) == -1
    assert disp(table(2), x=ctypes.c_void_p(264)) == -3
    assert disp(table(2), pos=None) == -1
    assert comb(table(2), out=None) == -1
    assert comb(table(2), tw=None) == -1
    with pytest.raises(ValueError):
        m.peer_rows([], [], [])
    with pytest.raises(ValueError):
        m.peer_rows([256] * 65, [0] * 65, [1] * 65)


def test_dispatch_without_the_copy_needs_no_rows(L):
    """moe_dispatch with xs NULL sorts only, so x_e may be NULL too; with xs
    given, x_e is required (host checks, fake pointers rejected before any
    device work)."""
    p = ctypes.c_void_p(256)
    # xs given without x_e: rejected on the host
    assert L.moe_dispatch(p, 4, 2, 8, None, 128, p, p, p, p, p, p, 1 << 20, None) == -1
    # an unaligned x_e matters only when the rows are copied
    assert L.moe_dispatch(p, 4, 2, 8, ctypes.c_void_p(264), 128, p, p, p, p, p, p, 1 << 20,
                          None) == -3




def test_expert_ffn_to_slots_validation(L):
    """moe_expert_ffn_to_slots rejects bad arguments on the host (fake
    pointers, nothing reaches a device): it needs perm whenever there are
    rows, the expert MLP's shape limits and 16-byte aligned rows."""
    import moe_routing_expert_fp32_b200 as m
    p = ctypes.c_void_p(256)
    a = m.ActConfig("silu")._c()
    ws = ctypes.c_void_p(1 << 20)
    big = 1 << 30
    # perm missing with rows present
    assert L.moe_expert_ffn_to_slots(p, p, None, 8, 64, 256, 128, p, p, p, ctypes.byref(a), p, ws,
                                     big, None) == -1
    # d_e not a multiple of 128
    assert L.moe_expert_ffn_to_slots(p, p, p, 8, 64, 200, 128, p, p, p, ctypes.byref(a), p, ws,
                                     big, None) == -2
    # y_slots not 16-byte aligned
    assert L.moe_expert_ffn_to_slots(p, p, p, 8, 64, 256, 128, p, p, p, ctypes.byref(a),
                                     ctypes.c_void_p(264), ws, big, None) == -3
    # workspace too small
    assert L.moe_expert_ffn_to_slots(p, p, p, 8, 64, 256, 128, p, p, p, ctypes.byref(a), p, ws,
                                     8, None) == -4


def test_wait_probe_switch_round_trips(L):
    """moe_set_wait_probe returns the previous setting; it launches nothing."""
    before = L.moe_launch_count()
    prev = L.moe_set_wait_probe(1)
    assert L.moe_set_wait_probe(prev) == 1
    assert L.moe_set_wait_probe(prev) == prev
    assert L.moe_launch_count() == before
