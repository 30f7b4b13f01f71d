"""Batch sharding of the decode step over GPUs, one process per GPU.

The sequences of a decode batch are independent ("Build your own Llama 3 from
scratch" 六: each sequence has its own KV cache and its own next token), so a
step over B sequences splits over N ranks with no exchange on the data path:
rank r holds the whole model and the caches of its own contiguous run of
sequences, decodes them, and only the next-token ids travel, gathered on the
host.  This module holds the split and that gather; it does no arithmetic of
the decoder.
"""
from __future__ import annotations

import torch


def shard(batch: int, world: int, rank: int):
    """(first sequence, number of sequences) of ``rank``'s share of ``batch``.

    Contiguous runs whose sizes differ by at most one, the larger ones first:
    32 sequences over 8 ranks give 4 each; 10 over 4 give 3, 3, 2, 2.
    """
    if batch < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split: batch={batch} world={world} rank={rank}")
    base, extra = divmod(batch, world)
    count = base + (1 if rank < extra else 0)
    start = rank * base + min(rank, extra)
    return start, count


def gather_ids(local_ids: torch.Tensor, batch: int, world: int, rank: int, group=None, dst: int = 0):
    """Gather every rank's next-token ids (host int32 tensor of its share, in
    sequence order) onto rank ``dst`` through a CPU (gloo) process group.

    Returns the [batch] ids in sequence order on ``dst`` and None elsewhere.
    Every rank must call it (it is a collective of ``group``).
    """
    start, count = shard(batch, world, rank)
    if local_ids.shape != (count,) or local_ids.device.type != "cpu":
        raise ValueError(f"rank {rank} holds {count} sequences; got {tuple(local_ids.shape)} on "
                         f"{local_ids.device}")
    width = (batch + world - 1) // world
    send = torch.full((width,), -1, dtype=torch.int32)
    send[:count] = local_ids.to(torch.int32)
    if world == 1:
        return send[:count].clone()
    recv = [torch.empty((width,), dtype=torch.int32) for _ in range(world)] if rank == dst else None
    torch.distributed.gather(send, recv, dst=dst, group=group)
    if rank != dst:
        return None
    out = torch.empty((batch,), dtype=torch.int32)
    for r in range(world):
        s, c = shard(batch, world, r)
        out[s:s + c] = recv[r][:c]
    return out
