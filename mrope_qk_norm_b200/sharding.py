"""Token-range sharding of the normalise-then-rotate path across ranks.

Tokens are independent, so a batch splits into contiguous token ranges, one
per rank, with no exchange step.  A shard is exactly a chunked launch
(llama.cpp fork #286, "The change": a launch over part of the tokens indexes
the full-length position rows from its first token): rank r processes
tokens [t0, t1) of its inputs and passes ``token_offset = t0`` so angles are
read for the right tokens.
"""
from __future__ import annotations


def shard_range(n_tokens: int, rank: int, world: int) -> tuple[int, int]:
    """[t0, t1) of rank `rank` out of `world`: contiguous, sizes differ by <= 1."""
    if world < 1 or not 0 <= rank < world or n_tokens < 0:
        raise ValueError("need 0 <= rank < world and n_tokens >= 0")
    base, extra = divmod(n_tokens, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def max_over_ranks(value_ms: float, dist=None, device=None) -> float:
    """The slowest rank's device time: every rank contributes its own CUDA-event
    time and all of them get the maximum (one all-reduce; no-op on one rank)."""
    import torch
    if dist is None:
        return float(value_ms)
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own
    batch of tokens_per_rank each step, and a step lasts as long as the slowest
    rank's step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)
