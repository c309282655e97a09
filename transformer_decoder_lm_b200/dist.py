"""Data-parallel forward over several GPUs (one process per GPU).

The forward pass shards over sequences: every rank holds all weights and runs
its own batch of B sequences through the C ABI; no activation crosses GPUs.
The only exchange is the loss: the mean over all ranks' scored positions
needs the sum of per-position losses and their count from every rank, one
all-reduce of two numbers ("Hand-writing GPT-2 from scratch: the Transformer
decoder core modules in PyTorch", section 6.2: the DDP set-up with the NCCL
backend; here only the forward's loss is combined).
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def shard_sequences(global_batch: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, stop) of the sequences rank `rank` runs when `global_batch`
    sequences are split as evenly as possible over `world` ranks (the first
    global_batch % world ranks take one more)."""
    if world < 1 or not (0 <= rank < world) or global_batch < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def global_mean_loss(local_mean: torch.Tensor, local_count: int, group=None) -> torch.Tensor:
    """Mean loss over every rank's scored positions from each rank's own mean
    and count: all-reduce (mean * count, count) and divide. `local_mean` is a
    1-element float tensor on the rank's device (the loss gpt2_loss wrote);
    returns a 1-element tensor. A rank with no scored position contributes
    (0, 0) even if its mean is NaN."""
    count = torch.tensor([float(local_count)], dtype=torch.float64, device=local_mean.device)
    num = torch.where(count > 0, local_mean.to(torch.float64) * count, torch.zeros_like(count))
    buf = torch.cat([num, count])
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return (buf[0:1] / buf[1:2]).to(torch.float32)


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest `value` over all ranks (step times are reported this way)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
