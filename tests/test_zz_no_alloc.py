"""moe_dispatch_static: the dispatch entry point for callers that cannot
allocate device memory (a plugin that its host framework hands only input and
output tensors, a process whose device memory another allocator has reserved,
a loop that must not call cudaMalloc).  It must give exactly what moe_dispatch
gives, call after call, while its scratch lives in a fixed array inside the
library.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest

import synth
from tests.gpu_util import dev_bf16, random_topk

pytestmark = pytest.mark.gpu


def _outputs(torch, N, K, E, d):
    S = N * K
    return (torch.empty(E, dtype=torch.int32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.empty(S, dtype=torch.int32, device="cuda"),
            torch.empty(S, dtype=torch.int32, device="cuda"),
            torch.empty((S, d), dtype=torch.bfloat16, device="cuda"))


def _call_static(L, torch, idx, x, E, outs):
    N, K = idx.shape
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    c, o, p, q, xs = outs
    return L.moe_dispatch_static(vp(idx), N, K, E, vp(x), x.shape[1], vp(c), vp(o), vp(p), vp(q),
                                 vp(xs), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(torch, a, b):
    for u, v in zip(a, b):
        if u.dtype == torch.bfloat16:
            u, v = u.view(torch.int16), v.view(torch.int16)
        assert torch.equal(u, v)


def test_static_dispatch_matches_dispatch_on_consecutive_calls():
    import torch
    import moe_routing_expert_fp32_b200 as moe
    L = moe.lib()
    cases = [  # (N, K, E, d, skew): decode-shaped, then a larger skewed batch, then tiny
        (128, 8, 256, 7168, 0.0),
        (4096, 8, 384, 1024, 1.2),
        (64, 4, 16, 256, 0.0),
    ]
    prepared = []
    for i, (N, K, E, d, skew) in enumerate(cases):
        idx = torch.from_numpy(random_topk(N, K, E, np.random.default_rng(40 + i), skew)).cuda()
        x = dev_bf16(synth.host_normal_bf16(9, 1, (N, d), 1.0, start=i * 10_000_000))
        ref = moe.dispatch(idx, x, E)  # the existing entry point, with its own workspace
        prepared.append((idx, x, E, ref, _outputs(torch, N, K, E, d)))
    torch.cuda.synchronize()
    # first call on this device: looks up the array's address
    idx, x, E, ref, outs = prepared[0]
    assert _call_static(L, torch, idx, x, E, outs) == 0
    torch.cuda.synchronize()
    _same(torch, outs, ref)
    free_before = torch.cuda.mem_get_info()[0]
    # two more calls in a row on the same array: no stale state, no allocation
    for idx, x, E, ref, outs in prepared[1:]:
        assert _call_static(L, torch, idx, x, E, outs) == 0
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    for idx, x, E, ref, outs in prepared[1:]:
        _same(torch, outs, ref)
    assert free_before - free_after < (1 << 20)


def test_static_dispatch_rejects_sizes_beyond_its_array():
    import torch
    import moe_routing_expert_fp32_b200 as moe
    L = moe.lib()
    p = ctypes.c_void_p(256)
    # 2^21 slots over 1024 experts would need 8 MiB of per-chunk counts
    rc = L.moe_dispatch_static(p, 1 << 18, 8, 1024, p, 128, p, p, p, p, p, None)
    assert rc == -2
    # the binding wrapper gives the same answer as moe_dispatch on a small case
    idx = torch.from_numpy(random_topk(50, 2, 7, np.random.default_rng(1))).cuda()
    x = dev_bf16(synth.host_normal_bf16(2, 1, (50, 128), 1.0))
    _same(torch, moe.dispatch_static(idx, x, 7), moe.dispatch(idx, x, 7))


def test_static_dispatch_sort_only_matches_dispatch():
    """xs = NULL: only counts, offsets, perm and pos, as moe_dispatch gives them
    with gather=False; x_e is not read, so a NULL x_e is accepted too."""
    import torch
    import moe_routing_expert_fp32_b200 as moe
    L = moe.lib()
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    for i, (N, K, E) in enumerate([(128, 8, 256), (4096, 8, 384), (1, 1, 3)]):
        idx = torch.from_numpy(random_topk(N, K, E, np.random.default_rng(70 + i),
                                           1.2 if N > 1000 else 0.0)).cuda()
        x = dev_bf16(synth.host_normal_bf16(4, 1, (N, 128), 1.0))
        ref = moe.dispatch(idx, x, E, gather=False)[:4]
        got = moe.dispatch_static(idx, x, E, gather=False)
        assert got[4] is None
        _same(torch, got[:4], ref)
        c, o, p, q = (torch.empty_like(t) for t in ref)
        rc = L.moe_dispatch_static(vp(idx), N, K, E, None, 128, vp(c), vp(o), vp(p), vp(q), None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        _same(torch, (c, o, p, q), ref)
