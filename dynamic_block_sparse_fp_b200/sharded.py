"""Head-sharded execution of one layer across ranks (one process per GPU).

FlexPrefill (atlas.scime.ai summary, "Approach") decides the sparse pattern,
the budget and the selected blocks per attention head, from that head's
queries and its kv head's keys only; attention of a head reads only its own
lists.  So the whole path shards by kv head with no exchange: rank r of G
takes kv heads [r*Hkv/G, (r+1)*Hkv/G) and their g query heads each, and runs
the path on that slice through the C ABI.  The one collective is optional:
all-gathering the ranks' outputs into the full [Bt, Hq, N, d] tensor on every
rank (NCCL over NVLink on GPUs), for a caller that needs the whole layer's
output rather than feeding a tensor-parallel consumer.

Argument marshalling and torch.distributed plumbing only; every step of the
path runs in the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops


def head_shard(n_kv_heads: int, world: int, rank: int) -> tuple[int, int]:
    """(first kv head, kv head count) of rank `rank`; kv heads split evenly."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n_kv_heads % world:
        raise ValueError(f"{n_kv_heads} kv heads do not split evenly over {world} ranks")
    nk = n_kv_heads // world
    return rank * nk, nk


def shard_inputs(q, k, v, world: int, rank: int):
    """This rank's q [Bt, nk*g, N, d] and k, v [Bt, nk, N, d], contiguous."""
    hq, hkv = q.shape[1], k.shape[1]
    g = hq // hkv
    kv0, nk = head_shard(hkv, world, rank)
    return (q[:, kv0 * g:(kv0 + nk) * g].contiguous(), k[:, kv0:kv0 + nk].contiguous(),
            v[:, kv0:kv0 + nk].contiguous())


def gather_heads(out_local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather the ranks' [Bt, h, N, d] outputs into [Bt, world*h, N, d] (rank order)."""
    if world == 1:
        return out_local
    x = out_local.contiguous()
    if dist.get_backend(group) == "nccl":
        buf = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(buf, x, group=group)
        return heads_of_gathered(buf)
    else:
        parts = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(parts, x, group=group)
    return torch.cat(parts, dim=1)


def heads_of_gathered(buf: torch.Tensor) -> torch.Tensor:
    """[world, Bt, h, N, d] (rank-major, as all_gather_into_tensor leaves it) ->
    [Bt, world*h, N, d]; with Bt = 1 that is a view of the same memory (no copy)."""
    world, bt, h = buf.shape[:3]
    if bt == 1:
        return buf.view((1, world * h) + tuple(buf.shape[3:]))
    return torch.cat(buf.unbind(0), dim=1)


def sharded_prefill_attn(q, k, v, block_size: int, params, group=None, gather: bool = True):
    """The whole path for this rank's heads of one layer (fp_prefill_attn);
    the full output on every rank if `gather`, else this rank's heads."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    qs, ks, vs = shard_inputs(q, k, v, world, rank)
    out, _, _ = ops.prefill_attn(qs, ks, vs, block_size, params)
    return gather_heads(out, world, group) if gather else out
