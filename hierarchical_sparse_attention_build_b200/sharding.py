"""Sharding the build and attend across GPUs by KV head, with no collective on the data path.

The tree of a (sequence, KV head) and every tile of that KV group depend on nothing else:
the build reads only that head's tokens, and a tile's selection sums the scores of its own
group's query heads.  So a batch splits into contiguous blocks of KV heads, one block per
rank; each rank holds its block's token caches and tree, and runs the library on its block
as a smaller model (Hkv' = block size, Hq' = G * Hkv').  Query head h belongs to KV group
h // G (the repeat-kv convention), so a rank's query heads are the contiguous block
[G * h0, G * h1).  Outputs stay on the rank that computed them; `gather_outputs` joins
them for callers that want the whole batch on every rank (the only collective, and not
part of the hot path).
"""

from __future__ import annotations

import torch


def kv_head_range(num_kv_heads: int, rank: int, world: int) -> tuple[int, int]:
    """KV heads [h0, h1) of `rank`: contiguous blocks, the first num_kv_heads % world ranks
    one head larger.  A rank may get an empty block when world > num_kv_heads."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if num_kv_heads < 1:
        raise ValueError(f"num_kv_heads {num_kv_heads}")
    base, extra = divmod(num_kv_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_params(p, rank: int, world: int):
    """The library parameters of this rank's block (same branching, top-k, RoPE base and
    softmax scale; 1/sqrt(128) stays the scale when none was set)."""
    from . import Params

    h0, h1 = kv_head_range(p.num_kv_heads, rank, world)
    g = p.num_q_heads // p.num_kv_heads
    out = Params()
    for name, _ in Params._fields_:
        setattr(out, name, getattr(p, name))
    out.num_kv_heads = h1 - h0
    out.num_q_heads = g * (h1 - h0)
    return out


def shard_cache(x: torch.Tensor, h0: int, h1: int) -> torch.Tensor:
    """A token cache [B][Hkv][capacity][128] -> this block's own contiguous cache.  A paged
    pool [num_pages][Hkv][page_size][128] shards the same way (heads are its second axis), and
    every rank keeps the whole page table."""
    return x[:, h0:h1].contiguous()


def shard_tokens(x: torch.Tensor, h0: int, h1: int) -> torch.Tensor:
    """New K/V rows [B][C][Hkv][128] -> [B][C][h1 - h0][128]."""
    return x[:, :, h0:h1].contiguous()


def shard_queries(q: torch.Tensor, group: int, h0: int, h1: int) -> torch.Tensor:
    """Queries [B][Q][Hq][128] -> the block's query heads [B][Q][G * (h1 - h0)][128]."""
    return q[:, :, group * h0:group * h1].contiguous()


def gather_outputs(out_block: torch.Tensor, num_kv_heads: int, group: int, pg=None) -> torch.Tensor:
    """Every rank's output block [B][Q][G * (h1 - h0)][128] -> the whole [B][Q][Hq][128] on
    every rank (all-gather over the process group; blocks of unequal size are padded to
    the largest and cut back)."""
    import torch.distributed as dist

    world = dist.get_world_size(pg)
    sizes = [kv_head_range(num_kv_heads, r, world) for r in range(world)]
    most = max(h1 - h0 for h0, h1 in sizes) * group
    B, Q, _, D = out_block.shape
    pad = torch.zeros(B, Q, most, D, dtype=out_block.dtype, device=out_block.device)
    pad[:, :, :out_block.shape[2]] = out_block
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=pg)
    return torch.cat([parts[r][:, :, :group * (h1 - h0)] for r, (h0, h1) in enumerate(sizes)], dim=2)
