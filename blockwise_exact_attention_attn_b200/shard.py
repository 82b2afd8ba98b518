"""Data-parallel sharding of independent attention units across ranks.

Every (sequence, head) pair of a forward call is an independent problem (no
query ever attends another sequence or head), so N processes split a global
batch into contiguous slices of sequences and run their slices with no
exchange on the data path; outputs stay where they were computed.  The only
cross-rank operations are host-side: a barrier around timed regions and a
maximum of the per-rank device times.
"""

from __future__ import annotations


def batch_shard(global_batch: int, rank: int, world: int) -> tuple:
    """[start, stop) of the sequences rank `rank` of `world` owns: contiguous,
    sizes differing by at most one, earlier ranks taking the larger ones."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float) -> float:
    """Maximum of a host float over the default process group (the value
    itself without one)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
