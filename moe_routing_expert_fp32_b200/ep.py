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
