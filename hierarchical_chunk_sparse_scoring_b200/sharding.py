"""Data-parallel sharding of the HiLS forward pass across GPUs (one process per GPU).

The forward pass is independent per (batch element, KV group): no step reads another sequence's
tokens or another KV group's heads.  A batch is therefore split across ranks by batch element with
no collective on the data path; the only cross-rank communication is host-side bookkeeping such as
the max-over-ranks step time.
"""
import torch


def shard_range(n_items, world, rank):
    """Contiguous [start, stop) of `n_items` owned by `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank: %r/%r" % (world, rank))
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_batch(tensors, world, rank):
    """The rank's slice along dim 0 (the batch) of every tensor, as contiguous tensors."""
    n = tensors[0].shape[0]
    a, b = shard_range(n, world, rank)
    return [t[a:b].contiguous() for t in tensors]


def max_over_ranks(value, group=None, device=None):
    """Max of a host float over all ranks (all_reduce MAX); the value itself with one process."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, ms_per_step_max, world):
    """Whole-job throughput of a weak-scaled run: every rank processed tokens_per_rank tokens per
    step, and a step ends when the slowest rank ends."""
    return tokens_per_rank * world / (ms_per_step_max * 1e-3)
