"""Expert parallelism: the routed layer with its experts split over the ranks
of a process group ("Kimi K3 · Add shared output", moe-forward excerpt: the
experts a rank runs are self.experts[i + ep_rank * experts_per_rank]).

Rank q holds the E_local = E / P consecutive experts q*E_local .. +E_local-1.
One step on every rank:

  1. route its own tokens and sort its slots by expert (moe_route,
     moe_dispatch): the sorted rows xs are grouped by destination rank, rank
     q's slice being rows offsets[q*E_local] .. offsets[(q+1)*E_local];
  2. exchange the per-(rank, local expert) row counts (all-to-all of P x
     E_local int32), then the rows themselves (all-to-all-v);
  3. run the local experts on the received rows, which arrive grouped by
     source rank and sorted by local expert within a source
     (moe_ep_expert_ffn: segment (p, e) uses local expert e);
  4. send the outputs back (the reverse all-to-all-v) into the slots the rows
     came from, and combine them with the routing weights (moe_combine).

`ep_forward_p2p` is the same step without a collective moving the rows: the
send kernel (moe_ep_dispatch_rows) stores each token row straight into the
receiving ranks' buffers through peer addresses of a symmetric-memory
allocation, and the combine (moe_ep_combine_rows) loads the outputs straight
from the ranks that computed them; `p2p_plan` places every rank's rows and
`exchange_forward_p2p` holds that step's logic, its compute and memory steps
passed in as callables (`P2PSteps`).

The collectives are torch.distributed all-to-alls (NCCL over NVLink on GPUs);
their split sizes need the counts on the host, the one synchronisation of the
step (the page's tokens_per_expert.cpu()).  Rows travel as int32 views of
their bf16 bits (two values per word; d_e is even), a type every backend
exchanges.  `exchange_forward` holds the exchange logic and takes the four
compute steps as callables, so the same code drives the CUDA kernels
(`ep_forward`) and any other implementation of the steps.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable


@dataclass
class Steps:
    """The compute steps around the exchange.

    route(x_r) -> (idx [N, K] int32, w [N, K] fp32)
    dispatch(idx, x_e) -> (counts [E] int32, pos [S] int32, xs [S, d_e] bf16)
    experts(xr [R, d_e], recv_counts [P, E_local] int32) -> y [R, d_e]
    combine(y [S, d_e], pos, w) -> out [N, d_e]
    """
    route: Callable
    dispatch: Callable
    experts: Callable
    combine: Callable


def exchange_forward(x_r, x_e, steps: Steps, num_experts: int, group=None):
    """One expert-parallel step on this rank (see the module docstring)."""
    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group)
    if num_experts % P != 0:
        raise ValueError(f"{num_experts} experts do not split over {P} ranks")
    E_local = num_experts // P
    idx, w = steps.route(x_r)
    counts, pos, xs = steps.dispatch(idx, x_e)
    d_e = xs.shape[1]
    send_counts = counts.reshape(P, E_local).contiguous()
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    # split sizes on the host: the step's one synchronisation
    send_split = send_counts.sum(dim=1).tolist()
    recv_split = recv_counts.sum(dim=1).tolist()
    xs_bits = xs.contiguous().view(torch.int32)
    xr_bits = torch.empty((sum(recv_split), d_e // 2), dtype=torch.int32, device=xs.device)
    dist.all_to_all_single(xr_bits, xs_bits, recv_split, send_split, group=group)
    yr = steps.experts(xr_bits.view(xs.dtype), recv_counts)
    y_bits = torch.empty_like(xs_bits)
    dist.all_to_all_single(y_bits, yr.contiguous().view(torch.int32), send_split, recv_split,
                           group=group)
    return steps.combine(y_bits.view(xs.dtype), pos, w), idx, w


def ep_forward(x_r, W, bias, cfg, w1_local, w3_local, w2_local, act, x_e=None, group=None):
    """The routed layer with this rank's experts w1_local, w3_local
    [E_local, F, d_e] and w2_local [E_local, d_e, F]; every rank passes its
    own tokens.  Returns (out [N, d_e] bf16, topk_idx, topk_w)."""
    from . import combine, dispatch, ep_expert_ffn, route

    x_e = x_r if x_e is None else x_e

    def _dispatch(idx, xe):
        counts, _, _, pos, xs = dispatch(idx, xe, cfg.num_experts)
        return counts, pos, xs

    steps = Steps(
        route=lambda xr: route(xr, W, bias, cfg),
        dispatch=_dispatch,
        experts=lambda xr, rc: ep_expert_ffn(xr, rc, w1_local, w3_local, w2_local, act),
        combine=lambda y, pos, w: combine(y, pos, w),
    )
    return exchange_forward(x_r, x_e, steps, cfg.num_experts, group)


def p2p_plan(all_counts, rank: int, P: int):
    """Where this rank's rows go and what it receives, from every rank's
    per-expert counts all_counts [P, E] (host integers, identical on all ranks):

      first_row[q]  this rank's first row in rank q's buffer: the rows ranks
                    0 .. rank-1 send to q, so q receives its rows grouped by
                    source rank and, within a source, sorted by local expert;
      recv_counts   [P, E_local] int32: the rows each source sends to this
                    rank's experts (the segments moe_ep_expert_ffn runs);
      recv_rows     the rows this rank receives.
    """
    import numpy as np

    c = np.asarray(all_counts, dtype=np.int64)
    if c.ndim != 2 or c.shape[0] != P or c.shape[1] % P != 0:
        raise ValueError(f"counts of shape {c.shape} do not split over {P} ranks")
    E_local = c.shape[1] // P
    rows_to = c.reshape(P, P, E_local).sum(axis=2)  # [source rank, destination rank]
    first_row = [int(rows_to[:rank, q].sum()) for q in range(P)]
    recv_counts = np.ascontiguousarray(c[:, rank * E_local:(rank + 1) * E_local], dtype=np.int32)
    return first_row, recv_counts, int(rows_to[:, rank].sum())


@dataclass
class P2PSteps:
    """The steps of the exchange through peer memory (`exchange_forward_p2p`).

    route(x_r) -> (idx [N, K] int32, w [N, K] fp32)
    dispatch(idx, x_e) -> (counts [E] int32, offsets [E+1] int32, pos [S] int32)
    buffers(cap, d_e, like) -> (xr, y, xr_at, y_at): this rank's receive and
        output buffers of `cap` rows and every rank's, as the send and combine
        steps address them (the same `cap` on every rank)
    send_rows(x_e, pos, offsets, xr_at, first_row, cap): store each slot's row
        into its rank's receive buffer
    experts(xr [R, d_e], recv_counts [P, E_local] int32, y [R, d_e]): the
        local experts on the received rows, outputs into y
    combine_rows(y_at, first_row, cap, pos, offsets, w) -> out [N, d_e]
    barrier(): every rank's previous step has finished
    """
    route: Callable
    dispatch: Callable
    buffers: Callable
    send_rows: Callable
    experts: Callable
    combine_rows: Callable
    barrier: Callable


def exchange_forward_p2p(x_r, x_e, steps: P2PSteps, num_experts: int, group=None):
    """One expert-parallel step through peer memory on this rank:

      1. route and sort its slots;
      2. all-gather the per-expert counts (the step's one host
         synchronisation) and place the rows with p2p_plan;
      3. store its rows into the receiving ranks' buffers; barrier;
      4. run the local experts on the received rows; barrier;
      5. combine, loading each slot's output from the rank that computed it;
         barrier (no rank reuses its buffers while a peer still reads them).

    Returns (out, topk_idx, topk_w)."""
    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if num_experts % P != 0:
        raise ValueError(f"{num_experts} experts do not split over {P} ranks")
    idx, w = steps.route(x_r)
    counts, offsets, pos = steps.dispatch(idx, x_e)
    got = [torch.empty_like(counts) for _ in range(P)]
    dist.all_gather(got, counts.contiguous(), group=group)
    all_counts = torch.stack(got).cpu().numpy()
    first_row, recv_counts, R = p2p_plan(all_counts, rank, P)
    cap = max(1, max(p2p_plan(all_counts, q, P)[2] for q in range(P)))
    xr, y, xr_at, y_at = steps.buffers(cap, x_e.shape[1], x_e)
    steps.send_rows(x_e, pos, offsets, xr_at, first_row, cap)
    steps.barrier()
    steps.experts(xr[:R], recv_counts, y[:R])
    steps.barrier()
    out = steps.combine_rows(y_at, first_row, cap, pos, offsets, w)
    steps.barrier()
    return out, idx, w


class GrowingBuffer:
    """A buffer of at least `rows` rows kept from one step to the next: it is
    (re)allocated only when a step needs more rows than it holds, rounded up
    to a power of two.  With symmetric memory the allocation is collective;
    every rank asks for the same row count (the largest receive count, from
    the all-gathered counts), so every rank reallocates at the same steps."""

    def __init__(self, alloc):
        self._alloc = alloc
        self.rows = 0
        self.obj = None

    def get(self, rows: int):
        if rows > self.rows:
            self.rows = 1 << max(0, int(rows) - 1).bit_length()
            self.obj = None  # the old buffer goes before the new one is made
            self.obj = self._alloc(self.rows)
        return self.obj, self.rows


# symmetric row buffers of ep_forward_p2p, one per (group, device, width)
_P2P_BUFFERS: dict = {}


def ep_forward_p2p(x_r, W, bias, cfg, w1_local, w3_local, w2_local, act, x_e=None, group=None):
    """The routed layer with this rank's experts (w1_local, w3_local
    [E_local, F, d_e], w2_local [E_local, d_e, F]), the rows moved through
    peer memory by this library's kernels: moe_ep_dispatch_rows stores them
    into the receiving ranks' halves of a torch symmetric-memory buffer (the
    same size on every rank: the largest receive count), the experts write
    their outputs to the other half, and moe_ep_combine_rows loads them back.
    The barriers are a stream synchronisation and a process-group barrier.
    The buffer is kept for the next step (GrowingBuffer) and grows only when a
    step receives more rows than it holds.
    Returns (out [N, d_e] bf16, topk_idx, topk_w)."""
    import torch
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm

    from . import dispatch, ep_combine_rows, ep_dispatch_rows, ep_expert_ffn, peer_rows, route

    group = group or dist.group.WORLD
    P = dist.get_world_size(group)
    rank = dist.get_rank(group)
    E = cfg.num_experts
    x_e = x_r if x_e is None else x_e

    def _dispatch(idx, xe):
        counts, offsets, _, pos, _ = dispatch(idx, xe, E, gather=False)
        return counts, offsets, pos

    def _alloc(d_e, device):
        def make(rows):
            buf = symm.empty(2 * rows, d_e, dtype=torch.bfloat16, device=device)
            return buf, symm.rendezvous(buf, group)
        return make

    def _buffers(cap, d_e, like):
        key = (group.group_name, like.device.index, d_e)
        if key not in _P2P_BUFFERS:
            _P2P_BUFFERS[key] = GrowingBuffer(_alloc(d_e, like.device))
        (buf, handle), rows = _P2P_BUFFERS[key].get(cap)
        offset = buf.data_ptr() - handle.buffer_ptrs[rank]
        xr_at = [handle.buffer_ptrs[q] + offset for q in range(P)]
        y_at = [a + rows * d_e * buf.element_size() for a in xr_at]
        return buf[:cap], buf[rows:rows + cap], xr_at, y_at

    def _send(xe, pos, offsets, xr_at, first_row, cap):
        ep_dispatch_rows(xe, pos, offsets, E, peer_rows(xr_at, first_row, [cap] * P), cfg.top_k)

    def _experts(xr, recv_counts, y):
        rc = torch.from_numpy(recv_counts).to(xr.device)
        ep_expert_ffn(xr, rc, w1_local, w3_local, w2_local, act, y=y)

    def _combine(y_at, first_row, cap, pos, offsets, w):
        return ep_combine_rows(peer_rows(y_at, first_row, [cap] * P), pos, offsets, E, w,
                               x_e.shape[1])

    def _barrier():
        torch.cuda.current_stream().synchronize()
        dist.barrier(group=group)

    steps = P2PSteps(route=lambda xr: route(xr, W, bias, cfg), dispatch=_dispatch,
                     buffers=_buffers, send_rows=_send, experts=_experts,
                     combine_rows=_combine, barrier=_barrier)
    return exchange_forward_p2p(x_r, x_e, steps, E, group)
