"""Host-side plumbing for running the verify step on several GPUs.

Sequences are independent, so the batch is sharded over ranks with no
collective on the data path: rank r of N verifies sequences [r*B, (r+1)*B) of
one seeded stream (weak scaling).  Collectives are used only around the data
path: a barrier, the max of the per-rank device times, and (for callers that
want the whole batch's outputs on one rank) a gather of the small output
tensors.  Every function works with any torch.distributed backend (NCCL on
GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

from . import inputs as _inputs


def shard_range(per_rank: int, rank: int) -> Tuple[int, int]:
    """Sequence range [begin, end) of ``rank`` when every rank takes ``per_rank``."""
    if per_rank < 0 or rank < 0:
        raise ValueError("per_rank and rank must be non-negative")
    return rank * per_rank, (rank + 1) * per_rank


def generate_shard(workload: str, rank: int, world: int, per_rank: int = None,
                   sigma: float = None):
    """This rank's inputs: sequences [rank*B, (rank+1)*B) of a batch of
    world*B sequences of ``workload`` (B = the workload's batch by default;
    ``sigma`` overrides its draft noise).  Equal, array for array, to the same
    slice of the whole batch."""
    w = _inputs.WORKLOADS[workload]
    B = w.B if per_rank is None else per_rank
    b0, b1 = shard_range(B, rank)
    return _inputs.generate(workload, seq_begin=b0, seq_end=b1, B=B * world, sigma=sigma)


def max_over_ranks(value: float, device=None) -> float:
    """The max of ``value`` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_outputs(out_tokens, out_num_accepted, dst: int = 0):
    """Concatenate every rank's [B, K+1] tokens and [B] counts, in rank order,
    on rank ``dst`` (others get None).  Tensors may be CPU (gloo) or CUDA
    (NCCL); shapes must agree across ranks."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return out_tokens, out_num_accepted
    world = dist.get_world_size()
    toks = [torch.empty_like(out_tokens) for _ in range(world)]
    ns = [torch.empty_like(out_num_accepted) for _ in range(world)]
    dist.all_gather(toks, out_tokens.contiguous())
    dist.all_gather(ns, out_num_accepted.contiguous())
    if dist.get_rank() != dst:
        return None, None
    return torch.cat(toks, 0), torch.cat(ns, 0)


def concat_inputs(parts):
    """Concatenate shard inputs (rank order) into one VerifyInputs-like dict of
    arrays; used to check shards against a whole-batch generation."""
    keys = ("target", "draft", "tokens", "u_accept", "u_resample", "temperature")
    return {k: np.concatenate([getattr(p, k) for p in parts], axis=0) for k in keys}
