"""Sharding of one MicroAdam vector over ranks (one process per GPU).

Blocks are independent except for the scalars delta_{t+1} / Delta_{t+1}, the
min and max of the residual over the whole vector ("MicroAdam
(Sparse-Gradient Adaptive Optimization with Quantized Error Feedback)",
paragraph 1). Each rank owns a contiguous run of blocks (a shard handle,
``MicroAdam(..., shard=(first_block, blocks))``); between ``select`` and
``apply`` of step t the ranks combine their partial (-delta, Delta) pairs with
one 8-byte all-reduce. Both words are fp32 values >= +0, whose bit patterns
order like the values, so MAX over the patterns read as int32 is MAX over
the values (also what the select kernel's atomics do inside one GPU).
"""
from __future__ import annotations


def shard_blocks(d: int, block_size: int, rank: int, world: int) -> tuple[int, int]:
    """(first_block, block_count) of ``rank``'s contiguous share of ceil(d/B_d) blocks."""
    nb = -(-d // block_size)
    if not (0 <= rank < world) or world > nb:
        raise ValueError(f"cannot split {nb} blocks over {world} ranks")
    b0 = nb * rank // world
    b1 = nb * (rank + 1) // world
    return b0, b1 - b0


def combine_minmax_(state, offset: int, group=None):
    """All-reduce (MAX) the 8-byte (-delta_{t+1}, Delta_{t+1}) pair at byte
    ``offset`` of ``state`` (a uint8 tensor) across the process group, in place."""
    import torch
    import torch.distributed as dist
    pair = state[offset: offset + 8].view(torch.int32)
    dist.all_reduce(pair, op=dist.ReduceOp.MAX, group=group)
    return pair


def pack_pair(delta: float, Delta: float):
    """The header encoding of (delta, Delta): int32 bits of (0 - delta, Delta + 0)."""
    import numpy as np
    neg = np.float32(0.0) - np.float32(delta)
    mx = np.float32(Delta) + np.float32(0.0)
    return np.array([neg, mx], dtype=np.float32).view(np.int32)


def unpack_pair(words) -> tuple[float, float]:
    import numpy as np
    f = np.asarray(words, dtype=np.int32).view(np.float32)
    return float(np.float32(0.0) - f[0]), float(f[1])
