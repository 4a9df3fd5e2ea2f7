"""Context parallelism: sequences split over the ranks of a process group, one state exchange.

Rank r of a group of W holds the r-th contiguous span of every sequence: the same B, heads and
layout on every rank, the same local length S on every rank (BNSD or BSND, every local sequence
full, so rank r holds tokens [r S, (r + 1) S)).  Per chunk the state update is affine in the
start state (the FlashKDA README's chunk equations, 功能说明, rearranged), so a whole span maps
its start state to  S_end = S_start M_r + R_r.  Then, per (sequence, value head):

  1. ranks 0 .. W-2 compute (M_r, R_r) over their span (``kda_forward_summary``); the last
     rank's would never be used, it contributes zeros;
  2. one all-gather of the [M_r; R_r] pairs (NCCL over NVLink: 2 D^2 fp32 per unit and rank);
  3. rank r folds its start state from the true initial state through the maps of ranks
     0 .. r-1 (``kda_state_chain``);
  4. rank r runs its span from that state (``kda_forward``): its rows of the output and the
     state at the end of its span, which on the last rank is the sequences' final state.

Work per rank: one summary pass (two runs of the span, no outputs), a fold of r steps and one
forward, against one forward over all W spans on a single GPU.  The only collective is the
all-gather.  Every step runs in libkda.so; this module only orders the calls.

Every rank makes the same calls in the same order.  If a rank fails before the exchange, the
others leave the all-gather with the backend's error (the peer's connection closing, or the
process group's timeout), so give the group a short timeout to bound how long they wait.
"""
from __future__ import annotations

import torch

from . import api


class LibraryOps:
    """The library calls the schedule is made of (the default; tests may substitute their own
    to check the rank bookkeeping without a GPU)."""

    summary = staticmethod(api.forward_summary)
    chain = staticmethod(api.state_chain)
    forward = staticmethod(api.flash_kda)


def _group_info(group):
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def _all_gather(local: torch.Tensor, world: int, group) -> torch.Tensor:
    # the concatenated form ([W * 2, ...], viewed as [W, 2, ...]) is the one every backend takes
    import torch.distributed as dist
    out = torch.empty((world * local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    dist.all_gather_into_tensor(out, local, group=group)
    return out.view((world,) + tuple(local.shape))


def flash_kda_context_parallel(q, k, v, g, beta, scale: float, initial_state, A_log, dt_bias,
                               lower_bound: float, layout: str, plan, group=None, ops=None,
                               exchange=None, rank: int | None = None,
                               world: int | None = None):
    """The forward pass of this rank's span (see the module docstring).

    q, k, v, g, beta, plan: this rank's span, as for ``flash_kda`` (BNSD or BSND, every local
    sequence full length).  initial_state: the sequences' initial state (fp32 [B, Nv, D, D] or
    None), the same on every rank.  Returns (out, state): this span's output rows and the state
    at the end of the span (the final state of the whole sequences on the last rank).

    ``exchange(local) -> gathered`` overrides the all-gather ([2, B, Nv, D, D] in, [W, 2, B, Nv,
    D, D] out, in rank order); ``ops`` overrides the library calls; ``rank`` and ``world``
    override the group's (with ``exchange``, spans can be run one after another in one process).
    """
    if layout not in ("BNSD", "BSND"):
        raise ValueError("context parallelism splits BNSD or BSND sequences")
    ops = ops or LibraryOps
    g_rank, g_world = _group_info(group)
    rank = g_rank if rank is None else int(rank)
    world = g_world if world is None else int(world)
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if world == 1:
        return ops.forward(q, k, v, g, beta, scale, initial_state, A_log, dt_bias, lower_bound,
                           layout, plan)
    sh = plan.shape
    cu = plan.cu_seqlens
    if cu is not None and any(int(cu[i + 1] - cu[i]) != sh.S for i in range(len(cu) - 1)):
        raise ValueError("every local sequence must be full length (the spans are contiguous)")
    # 1. this span's affine maps, written straight into the exchange buffer
    local = torch.empty((2, sh.B, sh.Nv, sh.D, sh.D), dtype=torch.float32, device=q.device)
    if rank < world - 1:
        ops.summary(q, k, v, g, beta, A_log, dt_bias, lower_bound, layout, plan, M=local[0],
                    R=local[1])
    else:
        local.zero_()
    # 2. the one exchange
    gathered = exchange(local) if exchange is not None else _all_gather(local, world, group)
    # 3. the start state of this span
    start = initial_state
    if rank > 0:
        start = ops.chain(initial_state, gathered[:rank, 0], gathered[:rank, 1])
    # 4. this span from its true start state
    return ops.forward(q, k, v, g, beta, scale, start, A_log, dt_bias, lower_bound, layout, plan)
