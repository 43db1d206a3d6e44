"""Head-sharded prefill over several GPUs (one process per GPU).

GQA groups are independent in both branches: a group's index query selects
its own blocks, and its query heads attend only to its own K/V (ai-tool-zukan
"MiniMax MSA guide", section "GQAグループ単位の選択共有とは").  So a prefill
splits by group with no exchange inside attention: rank r takes a contiguous
range of groups with their query heads, K/V and index queries (the shared
index keys go to every rank), runs the unchanged single-GPU prefill on that
slice, and the head slices of the output are gathered once at the end
(NCCL all-gather over NVLink; gloo on the host in the tests).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch


def group_range(G: int, rank: int, world: int) -> Tuple[int, int]:
    """The contiguous groups [g0, g1) of `rank`: world must divide G."""
    if world < 1 or G % world:
        raise ValueError(f"{world} ranks cannot split {G} groups evenly")
    per = G // world
    return rank * per, (rank + 1) * per


def shard_inputs(q, k, v, q_idx, k_idx, H: int, G: int, rank: int, world: int):
    """This rank's contiguous copies of the prefill inputs (token-major layouts)."""
    g0, g1 = group_range(G, rank, world)
    HG = H // G
    return (q[:, g0 * HG:g1 * HG].contiguous(), k[:, g0:g1].contiguous(),
            v[:, g0:g1].contiguous(), q_idx[:, g0:g1].contiguous(), k_idx)


def gather_heads(local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather per-rank slices [N][n_r][...] (equal n_r, rank order) into [N][sum n_r][...]."""
    import torch.distributed as dist
    if world == 1:
        return local
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def head_sharded_prefill(cfg, q, k, v, q_idx, k_idx, prefill: Optional[Callable] = None,
                         group=None):
    """Prefill of the whole problem with this rank's share of the groups.

    ``cfg`` describes the whole problem; every rank passes the full inputs
    (or views of them) and gets the full ``(out, ids)`` back.  ``prefill``
    computes one slice: ``prefill(cfg_slice, q, k, v, q_idx, k_idx) ->
    (out [N][H_r][d], ids [N][G_r][k])``; the default is this library's
    msa_prefill.
    """
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    H, G = cfg.num_heads, cfg.num_groups
    g0, g1 = group_range(G, rank, world)
    from . import config as _config
    cfg_r = _config((g1 - g0) * (H // G), g1 - g0, cfg.head_dim, cfg.index_dim,
                    top_k=cfg.top_k, block=cfg.block_size, scale=cfg.softmax_scale)
    if prefill is None:
        from . import msa_prefill

        def prefill(c, *t):
            return msa_prefill(c, *t, ids_out=True)
    out_r, ids_r = prefill(cfg_r, *shard_inputs(q, k, v, q_idx, k_idx, H, G, rank, world))
    return gather_heads(out_r, world, group), gather_heads(ids_r, world, group)
