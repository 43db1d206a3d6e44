"""Sharding the path over several GPUs (one process per GPU).

Prefill by GQA group.  Groups are independent in both branches: a group's
index query selects its own blocks, and its query heads attend only to its own
K/V (ai-tool-zukan "MiniMax MSA guide", section "GQAグループ単位の選択共有とは").
So a prefill splits by group with no exchange inside attention: rank r takes a
contiguous range of groups with their query heads, K/V and index queries (the
shared index keys go to every rank), runs the unchanged single-GPU prefill on
that slice, and the head slices of the output are gathered once at the end
(NCCL all-gather over NVLink; gloo on the host in the tests).

Decode by sequence.  A decode step's sequences are independent: rank r takes a
contiguous run of them, balanced by cached length (the step's cost), with its
own packed slice of the caches, and the outputs are gathered in sequence order.
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


def sequence_range(cu_seqlens, rank: int, world: int) -> Tuple[int, int]:
    """The contiguous sequences [b0, b1) of `rank`: sequence b goes to the rank
    whose share of the total cached length holds the middle of b's cache."""
    cu = [int(x) for x in cu_seqlens]
    B, total = len(cu) - 1, cu[-1]
    if world < 1 or B < 1 or total < 1:
        raise ValueError("need world >= 1 and a non-empty batch")

    def owner(b):
        mid2 = cu[b] + cu[b + 1]  # twice the middle
        return min(world - 1, (mid2 * world) // (2 * total))
    owners = [owner(b) for b in range(B)]
    b0 = next((b for b in range(B) if owners[b] >= rank), B)
    b1 = next((b for b in range(B) if owners[b] > rank), B)
    return b0, b1


def shard_decode_inputs(q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens, rank: int,
                        world: int):
    """This rank's sequences: q / q_idx rows and its packed cache slice with the
    offsets rebased to 0 (cu_seqlens on the host)."""
    cu = [int(x) for x in cu_seqlens]
    b0, b1 = sequence_range(cu, rank, world)
    s0, s1 = cu[b0], cu[b1]
    cu_r = torch.tensor([c - s0 for c in cu[b0:b1 + 1]], dtype=torch.int64)
    return (q[b0:b1], q_idx[b0:b1], k_cache[s0:s1], v_cache[s0:s1], k_idx_cache[s0:s1], cu_r)


def gather_sequences(local: torch.Tensor, counts, group=None) -> torch.Tensor:
    """All-gather per-rank row blocks of different sizes (rank order) along dim 0."""
    import torch.distributed as dist
    world = len(counts)
    if world == 1:
        return local
    cap = max(max(counts), 1)
    pad = torch.zeros((cap,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)


def sequence_sharded_decode(cfg, q, q_idx, k_cache, v_cache, k_idx_cache, cu_seqlens,
                            decode: Optional[Callable] = None, group=None):
    """One decode step of the whole batch with this rank's share of the sequences.

    Every rank passes the whole batch (or views of it) with ``cu_seqlens`` on
    the host and gets the full ``(out [B][H][d], ids [B][G][k])`` back.
    ``decode(cfg, q, q_idx, k_cache, v_cache, k_idx_cache, cu) -> (out, ids)``
    runs one shard and returns out in bf16 and ids in int32 (what every rank
    contributes to the gather); the default is this library's msa_decode on
    q's device.
    """
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    cu = [int(x) for x in cu_seqlens]
    counts = [sequence_range(cu, r, world)[1] - sequence_range(cu, r, world)[0]
              for r in range(world)]
    if decode is None:
        from . import msa_decode

        def decode(c, qq, qi, kc, vc, kic, cu_r):
            lens = (cu_r[1:] - cu_r[:-1]).tolist()
            return msa_decode(c, qq, qi, kc, vc, kic, cu_r.to(qq.device), max(lens),
                              ids_out=True)
    args = shard_decode_inputs(q, q_idx, k_cache, v_cache, k_idx_cache, cu, rank, world)
    if counts[rank] > 0:
        out_r, ids_r = decode(cfg, *args)
    else:  # no sequences here: empty blocks for the gather
        out_r = torch.empty((0,) + tuple(q.shape[1:]), dtype=torch.bfloat16, device=q.device)
        ids_r = torch.empty((0, cfg.num_groups, cfg.top_k), dtype=torch.int32, device=q.device)
    return gather_sequences(out_r, counts, group), gather_sequences(ids_r, counts, group)
