"""Expert parallelism for the routed MoE feed-forward layer over torch.distributed.

The 256 routed experts of a layer are split into contiguous ranges, one per
rank (one GPU per rank); every rank sees all tokens and their routing, runs
its own experts' pairs (``stq1_moe_ffn_local``: pairs routed to other ranks
contribute zero) and the partial outputs are summed with one all-reduce
(NCCL over NVLink / NVSwitch between GPUs).  This is the B200 counterpart of
the pages' deployment on eight GPUs ("Tencent's 200GB Hy4-preview ...", "The
catch: not a drop-in GGUF"), whose split the pages do not describe.
"""

from __future__ import annotations

from typing import Callable


def expert_range(n_experts: int, world: int, rank: int) -> tuple[int, int]:
    """(first expert, count) of rank's contiguous share; counts differ by at most one."""
    if world <= 0 or not 0 <= rank < world or n_experts < world:
        raise ValueError("need 0 <= rank < world <= n_experts")
    base, extra = divmod(n_experts, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def expert_parallel(local_fn: Callable[[int, int], "torch.Tensor"], n_experts: int, group=None):
    """Runs ``local_fn(begin, count)`` for this rank's expert range and sums the
    partial outputs of all ranks in place (one all-reduce); returns the sum."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    begin, count = expert_range(n_experts, world, rank)
    out = local_fn(begin, count)
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def moe_ffn_expert_parallel(gateup_local, down_local, x, topk_ids, topk_weights, n: int, hidden: int,
                            n_experts: int, flags: int = 0, group=None):
    """The layer's output [T, hidden] on every rank; gateup_local / down_local hold
    this rank's expert range (see expert_range) back to back."""
    from . import moe_ffn_local
    return expert_parallel(
        lambda begin, count: moe_ffn_local(gateup_local, down_local, x, topk_ids, topk_weights, n, hidden, count,
                                           begin, flags=flags),
        n_experts, group)
