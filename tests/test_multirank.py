"""The multi-rank path on CPU (gloo, world size 2): token sharding gives each
rank disjoint rows of one batch, routing a shard equals routing those rows in
one batch, and the step time is the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from synth.workloads import WORKLOADS, host_inputs
        wl = WORKLOADS["tiny"]
        inp = host_inputs(wl, rank=rank)
        idx, w, _ = oracle.route(inp["x"], inp["W"], inp["bias"], wl.G, wl.TG, wl.K,
                                 wl.route_scale)
        got = [torch.zeros((wl.N, wl.K), dtype=torch.int32) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(idx))
        fake_ms = [1.0 + rank, 10.0 - rank]
        mx = bench.max_over_ranks(fake_ms, world)
        if rank == 0:
            q.put(("idx", np.concatenate([g.numpy() for g in got])))
            q.put(("max", mx))
            q.put(("tput", bench.aggregate_throughput(wl.N, world, mx[0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_tokens_and_take_max():
    import oracle
    import synth
    from synth.workloads import WORKLOADS, host_inputs
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = dict(q.get(timeout=10) for _ in range(3))
    wl = WORKLOADS["tiny"]
    inp = host_inputs(wl)
    x_all = synth.host_normal_bf16(wl.seed, synth.TID_X, (world * wl.N, wl.d_r), 1.0)
    idx_all, _, _ = oracle.route(x_all, inp["W"], inp["bias"], wl.G, wl.TG, wl.K, wl.route_scale)
    assert np.array_equal(out["idx"], idx_all)
    assert out["max"] == [2.0, 10.0]
    assert out["tput"] == pytest.approx(world * wl.N / 2.0e-3)
