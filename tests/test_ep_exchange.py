"""The expert-parallel exchange on CPU (gloo, world sizes 2 and 3).

`exchange_forward` (the product's exchange logic: counts all-to-all, rows
all-to-all-v, local experts on the received segments, the reverse
all-to-all-v, combine) runs here with the four compute steps taken by the CPU
reference, so the collectives and the bookkeeping are checked without a GPU.
Every rank's output must equal, bit for bit, the reference moe_infer of its
own tokens with all experts on one rank (the expert MLP and the combine are
row-wise, so only a wrong exchange can change a result).
"""
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


def _case(rank, E):
    """Rank-dependent token batches (uneven sizes) and shared weights."""
    rng = np.random.default_rng(100 + rank)
    N = 10 + 7 * rank
    d, F, K = 32, 16, 3
    x = (rng.standard_normal((N, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wr = np.random.default_rng(7)
    W = (wr.standard_normal((E, d)) * 0.2).astype(np.float32)
    b = wr.uniform(-0.01, 0.01, E).astype(np.float32)

    def bf(shape):
        return ((wr.standard_normal(shape) * 0.1).astype(np.float32).view(np.uint32)
                >> 16).astype(np.uint16)
    return x, W, b, bf((E, F, d)), bf((E, F, d)), bf((E, d, F)), K


def _worker(rank, world, port, E, q):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from moe_routing_expert_fp32_b200.ep import Steps, exchange_forward
        x, W, b, w1, w3, w2, K = _case(rank, E)
        E_local = E // world
        lo = rank * E_local

        def route(xr):
            idx, w, _ = oracle.route(xr.numpy().view(np.uint16), W, b, 1, 1, K, 1.5)
            return torch.from_numpy(idx), torch.from_numpy(w)

        def dispatch(idx, xe):
            counts, _, perm, pos = oracle.dispatch(idx.numpy(), E)
            xs = oracle.gather(xe.numpy().view(np.uint16), perm, K)
            return (torch.from_numpy(counts), torch.from_numpy(pos),
                    torch.from_numpy(xs.view(np.int16)))

        def experts(xr, recv_counts):
            rows = xr.numpy().view(np.uint16)
            y = np.zeros_like(rows)
            o = 0
            rc = recv_counts.numpy()
            for p in range(rc.shape[0]):
                for e in range(rc.shape[1]):
                    n = int(rc[p, e])
                    if n:
                        y[o:o + n] = oracle.expert_ffn(rows[o:o + n], w1[lo + e], w3[lo + e],
                                                       w2[lo + e], "silu")
                    o += n
            assert o == rows.shape[0]
            return torch.from_numpy(y.view(np.int16))

        def combine(y, pos, w):
            return torch.from_numpy(oracle.combine(y.numpy().view(np.uint16), pos.numpy(),
                                                   w.numpy(), K))

        xt = torch.from_numpy(x.view(np.int16))
        out, idx, w = exchange_forward(xt, xt, Steps(route, dispatch, experts, combine), E)
        ref = oracle.moe_infer(x, idx.numpy(), w.numpy(), w1, w3, w2, "silu")
        q.put((rank, bool(np.array_equal(out.numpy(), ref)), int(idx.numel())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (3, 12)])
def test_exchange_forward_equals_one_rank(world, E):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in res) == list(range(world))
    assert all(r[1] for r in res), res


@pytest.mark.parametrize("P,E_local", [(1, 4), (2, 3), (4, 2), (8, 16)])
def test_p2p_plan_places_rows_as_the_all_to_all_would(P, E_local):
    """Brute force: lay out every destination rank's buffer as the all-to-all
    delivers it (sources in rank order, each source's rows sorted by expert)
    and check that p2p_plan puts each source's rows exactly there."""
    from moe_routing_expert_fp32_b200.ep import p2p_plan
    rng = np.random.default_rng(P * 100 + E_local)
    E = P * E_local
    counts = rng.integers(0, 7, size=(P, E))
    counts[0, :] = 0                      # a rank that sends nothing
    buffers = [[] for _ in range(P)]      # rank q's rows: (source, expert, i)
    for p in range(P):
        for q in range(P):
            for e in range(q * E_local, (q + 1) * E_local):
                buffers[q] += [(p, e, i) for i in range(counts[p, e])]
    for rank in range(P):
        first_row, recv_counts, recv_rows = p2p_plan(counts, rank, P)
        assert recv_rows == len(buffers[rank])
        assert recv_counts.dtype == np.int32 and recv_counts.shape == (P, E_local)
        assert (recv_counts == counts[:, rank * E_local:(rank + 1) * E_local]).all()
        for q in range(P):
            # the sender's sorted positions for q's experts start at
            # offsets[q*E_local]; position j lands at first_row[q] + j - that
            sent = [(rank, e, i) for e in range(q * E_local, (q + 1) * E_local)
                    for i in range(counts[rank, e])]
            assert buffers[q][first_row[q]:first_row[q] + len(sent)] == sent


def test_p2p_plan_rejects_counts_that_do_not_split():
    from moe_routing_expert_fp32_b200.ep import p2p_plan
    with pytest.raises(ValueError):
        p2p_plan(np.zeros((2, 5), dtype=np.int64), 0, 2)
    with pytest.raises(ValueError):
        p2p_plan(np.zeros((3, 6), dtype=np.int64), 0, 2)


def _p2p_worker(rank, world, port, E, q, xr_bufs, y_bufs):
    """exchange_forward_p2p with the compute steps taken by the CPU reference
    and every rank's row buffers in shared memory, so a rank's send step
    writes straight into the other ranks' buffers and its combine reads from
    them, as the peer-memory kernels do on GPUs."""
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from moe_routing_expert_fp32_b200.ep import P2PSteps, exchange_forward_p2p
        x, W, b, w1, w3, w2, K = _case(rank, E)
        E_local = E // world
        lo = rank * E_local
        d = x.shape[1]

        def route(xr):
            idx, w, _ = oracle.route(xr.numpy().view(np.uint16), W, b, 1, 1, K, 1.5)
            return torch.from_numpy(idx), torch.from_numpy(w)

        def dispatch(idx, xe):
            counts, offsets, _, pos = oracle.dispatch(idx.numpy(), E)
            return torch.from_numpy(counts), torch.from_numpy(offsets), torch.from_numpy(pos)

        def buffers(cap, d_e, like):
            assert d_e == d and cap <= xr_bufs[0].shape[0]
            return xr_bufs[rank], y_bufs[rank], xr_bufs, y_bufs

        def owner(offs, j):
            return next(r for r in range(world) if j < offs[(r + 1) * E_local])

        def send_rows(xe, pos, offsets, xr_at, first_row, cap):
            offs = offsets.numpy()
            for s, j in enumerate(pos.numpy()):
                if j < 0:
                    continue
                r = owner(offs, j)
                row = first_row[r] + j - offs[r * E_local]
                assert row < cap
                xr_at[r][row] = xe[s // K]

        def experts(xr, recv_counts, y):
            rows = xr.numpy().view(np.uint16)
            out = y.numpy().view(np.uint16)
            o = 0
            for p in range(recv_counts.shape[0]):
                for e in range(recv_counts.shape[1]):
                    n = int(recv_counts[p, e])
                    if n:
                        out[o:o + n] = oracle.expert_ffn(rows[o:o + n], w1[lo + e], w3[lo + e],
                                                         w2[lo + e], "silu")
                    o += n
            assert o == rows.shape[0]

        def combine_rows(y_at, first_row, cap, pos, offsets, w):
            offs = offsets.numpy()
            home = np.zeros((pos.numel(), d), np.uint16)  # outputs in sorted order
            for r in range(world):
                a, z = offs[r * E_local], offs[(r + 1) * E_local]
                f = first_row[r]
                home[a:z] = y_at[r][f:f + (z - a)].numpy().view(np.uint16)
            return torch.from_numpy(oracle.combine(home, pos.numpy(), w.numpy(), K))

        steps = P2PSteps(route, dispatch, buffers, send_rows, experts, combine_rows,
                         lambda: dist.barrier())
        xt = torch.from_numpy(x.view(np.int16))
        out, idx, w = exchange_forward_p2p(xt, xt, steps, E)
        ref = oracle.moe_infer(x, idx.numpy(), w.numpy(), w1, w3, w2, "silu")
        q.put((rank, bool(np.array_equal(out.numpy(), ref)), int(idx.numel())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (3, 12)])
def test_exchange_forward_p2p_equals_one_rank(world, E):
    import torch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    cap = 256  # more rows than any rank receives here (all ranks: 81 or 153 slots)
    xr_bufs = [torch.zeros((cap, 32), dtype=torch.int16).share_memory_() for _ in range(world)]
    y_bufs = [torch.zeros((cap, 32), dtype=torch.int16).share_memory_() for _ in range(world)]
    procs = [ctx.Process(target=_p2p_worker, args=(r, world, port, E, q, xr_bufs, y_bufs))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in res) == list(range(world))
    assert all(r[1] for r in res), res


def test_growing_buffer_reallocates_only_when_needed():
    """The peer-memory step's row buffer is kept across steps and grows to
    the next power of two only when a step needs more rows; the same row
    counts give the same decisions on every rank."""
    from moe_routing_expert_fp32_b200.ep import GrowingBuffer
    made = []
    g = GrowingBuffer(lambda rows: made.append(rows) or f"buf{rows}")
    assert g.get(100) == ("buf128", 128)
    assert g.get(128) == ("buf128", 128) and g.get(1) == ("buf128", 128)
    assert g.get(129) == ("buf256", 256)
    assert g.get(200) == ("buf256", 256)
    assert made == [128, 256]
    h = GrowingBuffer(lambda rows: rows)
    assert h.get(1) == (1, 1) and h.get(3) == (4, 4)
