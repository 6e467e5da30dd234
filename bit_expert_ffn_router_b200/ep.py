"""Expert-parallel split of one MoE layer over N devices.

Prefill is the part of the step with enough work to shard: the experts are
independent, so device r holds the experts e with e % N == r (interleaved, so
that a Zipf-shaped load spreads evenly) and computes their share of y for
every token; the routing runs on every device. The shared expert and the
residual belong to device 0. The partial outputs (fp32) are gathered and
summed in rank order, so the result does not depend on timing. The pages'
engine splits a layer's experts between devices (GPU and CPU) and joins
their results before the next layer (vramglass.com, section
その2：GPUとCPUで同時に計算する), and runs a model over 2 to 3 NVIDIA GPUs
(vramglass.com, section Strataのインストール方法; news.blueqat.app/post/3262,
section 対応ハードウェア).

The library side is the slot table: an expert with slot MOE_SLOT_ABSENT (-1)
is not held on a device and its pairs are left out. This module holds the
host logic (who holds what, each rank's configuration, the fixed-order sum)
and a torch.distributed driver around Context.layer_forward."""
from __future__ import annotations

import numpy as np

SLOT_ABSENT = -1


def held(E: int, rank: int, world: int) -> np.ndarray:
    """Boolean mask of the experts rank `rank` of `world` holds: e % world == rank."""
    return (np.arange(E) % world) == rank


def rank_slot_table(slot_of, rank: int, world: int):
    """The slot table rank `rank` uses: its own experts keep their slots, the
    others are marked absent. slot_of: [..., E] (numpy or torch)."""
    E = slot_of.shape[-1]
    mask = held(E, rank, world)
    try:
        import torch
        if isinstance(slot_of, torch.Tensor):
            m = torch.from_numpy(mask).to(slot_of.device)
            return torch.where(m, slot_of, torch.full_like(slot_of, SLOT_ABSENT))
    except ImportError:  # pragma: no cover
        pass
    return np.where(mask, slot_of, SLOT_ABSENT).astype(np.int32)


def rank_cfg(cfg, rank: int):
    """Rank r's layer configuration: fp32 partial output; the shared expert
    and the residual on rank 0 only."""
    if rank == 0:
        return cfg.replace(out_fp32=1)
    return cfg.replace(out_fp32=1, n_shared=0, residual=0)


def combine_partials(parts):
    """y = parts[0] + parts[1] + ... in rank order, fp32 (numpy or torch)."""
    y = parts[0].clone() if hasattr(parts[0], "clone") else np.array(parts[0], dtype=np.float32, copy=True)
    for p in parts[1:]:
        y += p
    return y


def layer_forward_ep(ctx, cfg, x, T, w_router, bias, slot_of, n_slots, pool, stride, shared, ws, y,
                     group=None):
    """One layer split over the ranks of `group` (torch.distributed, one rank
    per device): this rank's partial through the library, an all-gather of
    the partials, their rank-order sum into y (cfg's output type)."""
    import torch
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    part = torch.empty(T, cfg.d, dtype=torch.float32, device=x.device)
    ctx.layer_forward(rank_cfg(cfg, rank), x, T, w_router, bias, rank_slot_table(slot_of, rank, world), n_slots,
                      pool, stride, shared if rank == 0 else None, ws, part)
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part, group=group)
    total = combine_partials(parts)
    y.copy_(total.to(y.dtype))
    return y
