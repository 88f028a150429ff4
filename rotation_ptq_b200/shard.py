"""Host logic of a multi-GPU run: token shards and max-over-ranks timing.

Every step of the path is row-independent: the online rotation acts on one
token's activation row, the INT4 scale is per token, the weight scale per
output channel, and the GEMM row m depends on activation row m alone
("SpinQuant, Reproduced", section Q5: per-token activation quantization).
So N GPUs run N replicas of the path, each on its own shard of the token
batch, with no collective on the data path.  The only collectives of a run
are the barrier around the timed region and the reductions below, which use
whatever backend the process group has (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def token_shard(total: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [start, stop) of a `total`-token batch owned by `rank` of `world`.

    Contiguous, disjoint, covering; shard sizes differ by at most one, the
    first `total % world` ranks taking the extra row.  A rank may own no rows
    when total < world.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d outside a world of %d" % (rank, world))
    if total < 0:
        raise ValueError("negative token count")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic activations; rank 0 keeps `base`."""
    return base + 1000 * rank


def _reduce(values: Sequence[float], op_name: str) -> List[float]:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    device = torch.device("cpu")
    if dist.get_backend() == "nccl":
        device = torch.device("cuda", torch.cuda.current_device())
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return t.cpu().tolist()


def max_over_ranks(values: Sequence[float]) -> List[float]:
    """Element-wise maximum of `values` over all ranks (identity without a group)."""
    return _reduce(values, "MAX")


def sum_over_ranks(values: Sequence[float]) -> List[float]:
    """Element-wise sum of `values` over all ranks (identity without a group)."""
    return _reduce(values, "SUM")


def job_rate(units_all_ranks: float, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    if max_seconds <= 0:
        raise ValueError("non-positive time")
    return units_all_ranks / max_seconds
