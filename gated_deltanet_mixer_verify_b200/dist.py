"""Host-side helpers for running the mixer on several GPUs of one node.

The path shards with no exchange step: sequences (and heads) are independent and the
recurrent state never crosses them. Each rank therefore owns its own batch of sequences
(weak scaling) and the only collective is the max over ranks of a measured time.
"""
import torch
import torch.distributed as dist

SEED_STRIDE = 7919


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: distinct sequences per rank, reproducible per rank."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    return base_seed + SEED_STRIDE * rank


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device()) \
            if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank processed `units_per_rank` in at most `max_seconds`."""
    if max_seconds <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / max_seconds
