"""Host-side logic of running the layer on several GPUs, one process per GPU.

Tokens are independent rows of the linear layer, so N GPUs run N independent
token batches (weak scaling) with no collective on the data path: each rank
rotates, quantizes and multiplies its own batch against its own copy of the
quantized weights. The only collectives are the timing barrier and the max of
the per-rank step times, which bench.py takes with these helpers (NCCL on GPUs;
the tests drive them with gloo on CPU).
"""
from __future__ import annotations

from . import inputs


def rank_token_seed(rank: int) -> int:
    """Seed of rank `rank`'s synthetic token batch (distinct per rank)."""
    return inputs.TOKEN_SEED + rank


def rank_activations(w: inputs.Workload, rank: int, M: int | None = None):
    """Rank `rank`'s BF16 token batch (uint16 bits), drawn independently."""
    return inputs.activations(w, M=M, token_seed=rank_token_seed(rank))


def max_over_ranks(dist, value: float, device=None) -> float:
    """The maximum of `value` over all ranks (every rank gets it); `dist` is
    torch.distributed or None for a single process."""
    if dist is None:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, step_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's step."""
    return tokens_per_rank * world / (step_ms * 1e-3)
