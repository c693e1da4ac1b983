"""Memory Parallel decode over several GPUs, one process per GPU.

"100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it), section "Das Gehirn mit zwei
Geschwindigkeiten": each GPU manages part of the routing keys, the queries are broadcast,
the relevance scores are aggregated, and only the selected top-k content is loaded.

Here a bank of nb blocks is split into contiguous block ranges, one per rank (the first
nb % world ranks take one block more).  A decode step on every rank:

  1. scan its own shard: the shard's best top-k keys per (query, group), with bank-wide
     block ids (msa_decode_select_shard);
  2. all-gather the keys (world x n_query x hkv x topk int64: 512 KB for 64 queries,
     8 groups, top-32 on 4 ranks) and merge them: the bank-wide selection, and the
     selected blocks this rank owns (msa_decode_merge_shards);
  3. attend its owned blocks (msa_decode_attn_tiled over the shard): a partial output
     normalised with its log-sum-exp;
  4. all-gather the partials and combine them by log-sum-exp (msa_decode_combine_shards).

Both exchanges are plain all-gathers of a few hundred KB over NCCL; K/V never move.
Every step of the arithmetic runs in the library's kernels; this module only holds the
shard's buffers and orders the calls and the two collectives.
"""
from __future__ import annotations

import torch

from . import (decode_attn_tiled, decode_combine_shards, decode_merge_shards,
               decode_select_shard, encode_bank, pool_keys)

__all__ = ["shard_ranges", "BankShard", "decode_step"]


def shard_ranges(nb: int, world: int) -> list[tuple[int, int]]:
    """(first block, block count) of each rank's contiguous shard of nb blocks."""
    base, extra = divmod(nb, world)
    out, lo = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((lo, n))
        lo += n
    return out


class BankShard:
    """One rank's shard of a bank: its tokens' K/V (natural layout [tokens, hkv, d]) are
    pooled and encoded once (the offline encoding of the bank) and kept as the encoded
    images the decode kernels stream."""

    def __init__(self, k_shard, v_shard, block: int, block_begin: int):
        self.seq, self.hkv, self.d = k_shard.shape
        self.block, self.block_begin = block, block_begin
        self.block_count = -(-self.seq // block)
        _, khi, klo = (t[0] for t in pool_keys(k_shard[None], block, split=True))
        self.k_tiles, self.v_tiles, self.kbar_tiles = encode_bank(k_shard, v_shard, khi, klo,
                                                                  block)


def _all_gather(x: torch.Tensor, group=None) -> torch.Tensor:
    import torch.distributed as dist
    world = dist.get_world_size(group)
    flat = torch.empty(world * x.numel(), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(flat, x.contiguous().view(-1), group=group)
    return flat.view((world,) + tuple(x.shape))


def decode_step(q, shard: BankShard, topk: int, scale=None, group=None, gather=None, ws=None):
    """One Memory Parallel decode step of q [n_query, hq, d] on this rank's shard.
    Returns (o [n_query, hq, d], lse [n_query, hq], idx [n_query, hkv, topk] bank-wide),
    identical on every rank.  `gather(x)` returns [world, *x.shape] in rank order
    (default: torch.distributed.all_gather_into_tensor over `group`)."""
    gather = gather or (lambda x: _all_gather(x, group))
    keys = decode_select_shard(q, shard.kbar_tiles, shard.seq, shard.hkv, shard.block, topk,
                               shard.block_begin, ws=ws)
    idx, idx_local = decode_merge_shards(gather(keys), q.shape[1], q.shape[2],
                                         shard.block_begin, shard.block_count, dtype=q.dtype)
    o_part, lse_part = decode_attn_tiled(q, shard.k_tiles, shard.v_tiles, idx_local, shard.seq,
                                         shard.hkv, shard.block, scale=scale, ws=ws)
    o, lse = decode_combine_shards(gather(o_part), gather(lse_part), shard.hkv)
    return o, lse, idx
