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


# ---------------------------------------------------------------------------
# Row-sharded GEMV: each rank holds a contiguous range of the weight rows and
# computes its part of y; the parts are all-gathered (no reduction is needed,
# every output row lives on one rank).
# ---------------------------------------------------------------------------


def row_range(n_rows: int, world: int, rank: int) -> tuple[int, int]:
    """(first row, count) of rank's contiguous share of n_rows; counts differ by at most one."""
    if world <= 0 or not 0 <= rank < world or n_rows < world:
        raise ValueError("need 0 <= rank < world <= n_rows")
    base, extra = divmod(n_rows, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def gemv_row_sharded(w_local, x, n: int, k: int, group=None, gemv_fn=None):
    """y [b, n] on every rank from this rank's rows ``w_local`` (its row_range of
    the [n, k] matrix, packed) and the shared activations x [b, k]: a local
    GEMV, then an all-gather of the equal-size (padded) parts."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    begin, count = row_range(n, world, rank)
    if gemv_fn is None:
        from . import gemv as gemv_fn
    part = gemv_fn(w_local, x, count, k)                     # [b, count]
    b = part.shape[0]
    width = -(-n // world)                                   # the largest share
    padded = part.new_zeros((b, width))
    padded[:, :count] = part
    gathered = part.new_empty((world * b, width))            # the parts stacked along rows
    dist.all_gather_into_tensor(gathered, padded.contiguous(), group=group)
    gathered = gathered.view(world, b, width)
    y = part.new_empty((b, n))
    for r in range(world):
        rb, rc = row_range(n, world, r)
        y[:, rb:rb + rc] = gathered[r, :, :rc]
    return y


# ---------------------------------------------------------------------------
# Expert parallelism with token dispatch (prefill): tokens are spread over the
# ranks too; every (token, slot) pair travels to the rank that holds its
# expert, is computed there, and its result travels back (two all-to-alls).
# ---------------------------------------------------------------------------


class LibraryExchangeKernels:
    """The device steps of moe_ffn_all_to_all, from the library."""

    out_dtype = "float32"                                    # dtype of the rows ffn_rows returns

    @staticmethod
    def dispatch(topk_ids, x, topk_weights, n_experts, world):
        from . import ep_dispatch
        return ep_dispatch(topk_ids, x, topk_weights, n_experts, world)

    @staticmethod
    def ffn_rows(gateup_local, down_local, x_rows, local_ids, w_rows, n, hidden, n_local, flags):
        from . import moe_ffn_local
        return moe_ffn_local(gateup_local, down_local, x_rows, local_ids.view(-1, 1),
                             None if w_rows is None else w_rows.view(-1, 1), n, hidden, n_local, 0, flags=flags)

    @staticmethod
    def combine(rows, inv, t, topk):
        from . import ep_combine
        return ep_combine(rows, inv, t, topk)


def moe_ffn_all_to_all(gateup_local, down_local, x, topk_ids, topk_weights, n: int, hidden: int, n_experts: int,
                       flags: int = 0, group=None, kernels=LibraryExchangeKernels):
    """This rank's tokens' MoE feed-forward output [T, hidden].

    x [T, hidden] and topk_ids / topk_weights [T, topk] are this rank's tokens;
    gateup_local / down_local hold its expert range (expert_range).  The pairs
    are grouped by owner rank on the device, exchanged with all-to-all (the
    sizes first), run through the owner's experts as one-slot tokens (the
    routing weight is applied there), exchanged back and summed per token."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    t, topk = topk_ids.shape
    order, inv, counts, local_ids, x_send, w_send = kernels.dispatch(topk_ids, x, topk_weights, n_experts, world)
    send = counts[:world].to(torch.int64)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)          # how many rows come from each rank
    send_counts, recv_counts = send.cpu().tolist(), recv.cpu().tolist()
    n_send, n_recv = sum(send_counts), sum(recv_counts)

    def exchange(src, rows_out, split_out, split_in):
        dst = src.new_empty((rows_out,) + tuple(src.shape[1:]))
        dist.all_to_all_single(dst, src.contiguous(), split_out, split_in, group=group)
        return dst

    recv_x = exchange(x_send[:n_send], n_recv, recv_counts, send_counts)
    recv_ids = exchange(local_ids[:n_send], n_recv, recv_counts, send_counts)
    recv_w = None if w_send is None else exchange(w_send[:n_send], n_recv, recv_counts, send_counts)
    _, n_local = expert_range(n_experts, world, rank)
    if n_recv > 0:
        rows = kernels.ffn_rows(gateup_local, down_local, recv_x, recv_ids, recv_w, n, hidden, n_local, flags)
    else:
        rows = x.new_empty((0, hidden), dtype=getattr(torch, kernels.out_dtype))
    back = exchange(rows, n_send, send_counts, recv_counts)  # results, in this rank's send order
    return kernels.combine(back, inv, t, topk)
