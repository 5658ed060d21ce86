"""Slots over ranks (one process per GPU).

Every step of the path is independent per slot (layer, batch row, KV head) except
ZigZagKV's bounded allocation (Eq. 4-6), which needs each layer's LMBA count over
all of the layer's heads. When a model's slots are spread over ranks, that is the
one exchange: an all-reduce (sum) of the per-layer count sums, n_layers int32 per
rank, before kvc_alloc_budgets. Benchmark replicas (each rank its own batch) need
no exchange at all.
"""
from __future__ import annotations

import torch


def slot_range(n_slots: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block of slots owned by `rank` (slots are row-major (layer, batch, kv head),
    so a block is whole layers when n_slots / world is a multiple of the slots per layer)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    lo = n_slots * rank // world
    hi = n_slots * (rank + 1) // world
    return lo, hi


def layer_count_sums(counts: torch.Tensor, slot_lo: int, slots_per_layer: int, n_layers: int) -> torch.Tensor:
    """Per-layer sums of this rank's LMBA counts (counts[i] belongs to slot slot_lo + i)."""
    sums = torch.zeros(n_layers, dtype=torch.int64, device=counts.device)
    layer = (torch.arange(counts.numel(), device=counts.device) + slot_lo) // slots_per_layer
    sums.index_add_(0, layer, counts.to(torch.int64))
    return sums


def allreduce_layer_counts(local_sums: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of every rank's per-layer count sums (the ZigZagKV allocation's only exchange)."""
    import torch.distributed as dist
    out = local_sums.clone()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out
