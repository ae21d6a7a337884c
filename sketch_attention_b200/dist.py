"""Data-parallel host logic: users are independent problems (SequenceO1
Sec. 3.1 compresses each user's history on its own), so a batch splits by
user across ranks with no exchange on the data path.  The only collective is
the sum of the shared weights' gradients (P, W_Q, W_K, W_V), which is a sum
over users (the backward of eqs. (6)-(9) with weights shared by all users).
"""
from typing import Dict, Sequence, Tuple

import numpy as np

WEIGHT_GRADS = ("dP", "dW_Q", "dW_K", "dW_V")


def shard_users(B: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous user range [u0, u1) of `rank`; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError(f"bad shard request B={B} rank={rank} world={world}")
    base, extra = divmod(B, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def shard_offsets(offsets: Sequence[int], u0: int, u1: int) -> np.ndarray:
    """Offsets of users [u0, u1), rebased to the shard's first token."""
    off = np.asarray(offsets, np.int64)
    return off[u0:u1 + 1] - off[u0]


def allreduce_weight_grads(grads: Dict[str, "object"], group=None) -> None:
    """Sums the shared weights' gradients over ranks in place (torch tensors)."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    for name in WEIGHT_GRADS:
        dist.all_reduce(grads[name], group=group)
