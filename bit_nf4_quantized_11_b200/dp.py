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

Quantizing the frozen base can be split the same way: each rank quantizes a
contiguous slice of the flattened weight (whole 4096-block chunks), and the
only exchange is an all-gather of the per-chunk sums of the scale-mean tree,
after which every rank holds the same mean and its own codes, q8 and step2,
bit-identical to quantizing the whole weight on one device.  A second
all-gather of those pieces gives every rank the full replica that the
data-parallel step uses.
"""

from __future__ import annotations

from dataclasses import dataclass

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


def layer_grad_buffers(r: int, shapes, device):
    """(flat, [(dA, dB), ...]) for several projections ((n_in, n_out), ...) of
    one layer: every projection's dA [r, in] and dB [out, r] are fp32 views of
    one contiguous buffer, so the layer's gradient sum is one all-reduce."""
    sizes = [r * n_in + n_out * r for n_in, n_out in shapes]
    flat = torch.empty(sum(sizes), dtype=torch.float32, device=device)
    views, off = [], 0
    for (n_in, n_out), n in zip(shapes, sizes):
        views.append((flat[off: off + r * n_in].view(r, n_in), flat[off + r * n_in: off + n].view(n_out, r)))
        off += n
    return flat, views


def allreduce_adapter_grads(flat: torch.Tensor, group=None) -> None:
    """Sum the flat adapter-gradient buffer over the ranks of `group`."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(flat, op=torch.distributed.ReduceOp.SUM, group=group)


def _world(group):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        return torch.distributed.get_world_size(group), torch.distributed.get_rank(group)
    return 1, 0


def _all_gather_equal(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """Concatenation in rank order of equal-sized 1-D tensors from every rank."""
    if world == 1:
        return t
    parts = [torch.empty_like(t) for _ in range(world)]
    torch.distributed.all_gather(parts, t, group=group)
    return torch.cat(parts)


@dataclass
class NF4Shard:
    """One rank's part of a sharded NF4 quantization: blocks [block_begin, block_end)
    of the flattened weight."""
    codes: torch.Tensor    # uint8 [(block_end - block_begin) * 32]
    q8: torch.Tensor       # int8  [block_end - block_begin]
    step2: torch.Tensor    # fp32  [ceil((block_end - block_begin) / 256)]
    mean: torch.Tensor     # fp32  [1], the same on every rank
    block_begin: int
    block_end: int
    roots_per_rank: int


def quantize_nf4_sharded(W_shard: torch.Tensor, n_blocks_total: int, group=None, lib=None) -> NF4Shard:
    """Quantize this rank's slice W_shard (fp32, the weights of blocks
    [block_begin, block_end) of the plan, flattened row-major) of a weight with
    n_blocks_total 64-weight blocks.  Collective: every rank of `group` calls it."""
    if lib is None:
        import bit_nf4_quantized_11_b200 as lib
    world, rank = _world(group)
    b0, b1, cpr = lib.quantize_shard_plan(n_blocks_total, world, rank)
    if W_shard.numel() != (b1 - b0) * 64:
        raise ValueError(f"rank {rank} holds blocks [{b0}, {b1}): {(b1 - b0) * 64} weights, got {W_shard.numel()}")
    codes, roots, ws = lib.quantize_nf4_shard_local(W_shard, cpr, world * cpr)
    roots_all = _all_gather_equal(roots, world, group)
    q8, step2, mean = lib.quantize_nf4_shard_finish(roots_all, n_blocks_total, b1 - b0, ws)
    return NF4Shard(codes, q8, step2, mean, b0, b1, cpr)


def gather_nf4_replica(shard: NF4Shard, n_blocks_total: int, group=None):
    """(codes uint8 [n_blocks_total*32], q8 int8 [n_blocks_total], step2 fp32
    [ceil(n_blocks_total/256)], mean) of the whole weight on every rank.
    Shards are padded to roots_per_rank chunks for the all-gather; the padding
    is cut off after it.  Collective."""
    world, _ = _world(group)
    full = shard.roots_per_rank * 4096

    def padded(t, n):
        out = torch.zeros(n, dtype=t.dtype, device=t.device)
        out[:t.numel()] = t
        return out

    codes = _all_gather_equal(padded(shard.codes, full * 32), world, group)[:n_blocks_total * 32]
    q8 = _all_gather_equal(padded(shard.q8, full), world, group)[:n_blocks_total]
    step2 = _all_gather_equal(padded(shard.step2, full // 256), world, group)[:(n_blocks_total + 255) // 256]
    return codes, q8, step2, shard.mean
