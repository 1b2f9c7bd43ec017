"""Data-parallel plumbing of the QLoRA layer.

The layer is data-parallel: every rank holds the same frozen quantised weight
and the same adapter factors A, B, and takes its own tokens.  The one exchange
on the path is the sum of the adapter gradients dA, dB over ranks (page
"LoRA vs QLoRA: Efficient Fine-Tuning Explained", section "How QLoRA Works":
only the adapters are trained, so only their gradients cross ranks).  Both are
sums over tokens, so the sum over ranks equals the gradient of the
concatenated batch.
"""

from __future__ import annotations

RANK_SEED_STRIDE = 100000


def token_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own token-side tensor (X, dY): distinct per rank."""
    return seed + RANK_SEED_STRIDE * rank


def replica_seed(seed: int, rank: int) -> int:
    """Seed of a replicated tensor (W, A, B): the same on every rank."""
    del rank
    return seed


def allreduce_adapter_grads(dA, dB, group=None) -> None:
    """Sum dA and dB over the ranks of `group`, in place, in their own dtype."""
    import torch.distributed as dist
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)
