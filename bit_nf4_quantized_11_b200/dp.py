"""Data-parallel plumbing of the adapter training step.

Only the low-rank adapters A, B are trained while the NF4 base weight is
frozen ("QLoRA", aigrafen.se, opening paragraph), so data parallelism
replicates the quantized base and the adapters on every rank, gives each
rank its own token shard, and sums the adapter gradients dA, dB over ranks:
the layer gradients are sums over tokens, so the sum of the shards' dA, dB
is the gradient of the whole batch.  That sum is the only collective of the
step; the forward, dx and the per-shard gradients need no exchange.

The gradients of one layer live in one flat fp32 buffer (dA first, then
dB), so the sum is a single all-reduce.
"""

from __future__ import annotations

import torch


def shard_bounds(M: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [begin, end) of an M-token batch held by `rank` of `world`
    (contiguous shards, sizes differing by at most one)."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    return rank * M // world, (rank + 1) * M // world


def adapter_grad_buffers(r: int, n_in: int, n_out: int, device) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(flat, dA [r, in], dB [out, r]): fp32 views of one contiguous buffer."""
    flat = torch.empty(r * n_in + n_out * r, dtype=torch.float32, device=device)
    dA = flat[: r * n_in].view(r, n_in)
    dB = flat[r * n_in:].view(n_out, r)
    return flat, dA, dB


def allreduce_adapter_grads(flat: torch.Tensor, group=None) -> None:
    """Sum the flat adapter-gradient buffer over the ranks of `group`."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(flat, op=torch.distributed.ReduceOp.SUM, group=group)
