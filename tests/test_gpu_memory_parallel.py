"""Memory Parallel decode on one GPU: N shards of a bank run in one process, with the two
all-gathers done in memory (rank order), through the C ABI.  The merged selection must be
bitwise the unsharded tensor-core selection, and the combined output must match the fp64
oracle's unsharded decode."""
import pytest
import torch

import msa_inputs as mi
from parity_util import check_decode, pool_keys_chunked

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


CASES = [
    # (bank tokens, block, topk, n_query, shards)
    (300_000, 64, 32, 16, 3),
    (300_000, 64, 32, 16, 4),
    (250_000, 128, 16, 8, 2),
    (6_400, 64, 32, 4, 8),            # shards of 12-13 blocks: fewer than topk each
    (100_000, 64, 8, 70, 5),          # query tiles beyond 64, a ragged last shard block
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"S{c[0]}_b{c[1]}_k{c[2]}_q{c[3]}_n{c[4]}")
def test_sharded_decode_equals_unsharded(msa, case):
    from block_sparse_top_mean_b200.memory_parallel import BankShard, shard_ranges
    S, block, topk, nq, world = case
    w = mi.Workload("mp", "decode", 1, S, 32, 8, 128, block, topk, "bf16", n_query=nq)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=3)
    nb = w.nb
    # the unsharded tensor-core decode over the whole bank
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, block)
    _, _, idx_ref = msa.decode_fwd_tiled(q, bt, kt, vt, S, w.hkv, block, topk, w.scale)
    # every rank's shard, encoded on its own
    shards = []
    for begin, count in shard_ranges(nb, world):
        t0, t1 = begin * block, min(S, (begin + count) * block)
        shards.append(BankShard(kb[t0:t1].contiguous(), vb[t0:t1].contiguous(), block, begin))
    keys = torch.stack([msa.decode_select_shard(q, sh.kbar_tiles, sh.seq, sh.hkv, block, topk,
                                                sh.block_begin) for sh in shards])
    o_parts, l_parts, idx_all = [], [], []
    for sh in shards:
        idx, idx_local = msa.decode_merge_shards(keys, w.hq, w.d, sh.block_begin,
                                                 sh.block_count)
        idx_all.append(idx)
        o_p, l_p = msa.decode_attn_tiled(q, sh.k_tiles, sh.v_tiles, idx_local, sh.seq, sh.hkv,
                                         block, scale=w.scale)
        o_parts.append(o_p)
        l_parts.append(l_p)
        # the owned list is the bank-wide one restricted to the shard, renumbered
        own = (idx >= sh.block_begin) & (idx < sh.block_begin + sh.block_count)
        assert torch.equal(idx_local, torch.where(own, idx - sh.block_begin,
                                                  torch.full_like(idx, -1)))
    o, lse = msa.decode_combine_shards(torch.stack(o_parts), torch.stack(l_parts), w.hkv)
    torch.cuda.synchronize()
    for idx in idx_all:                       # the same selection on every rank ...
        assert torch.equal(idx, idx_ref)      # ... and exactly the unsharded one
    kbar_np = pool_keys_chunked(kb[None], block)[0]
    check_decode(q, kbar_np, kb, vb, block, topk, w.scale, idx_ref, o, lse)


def test_decode_step_single_rank_is_the_tiled_decode(msa):
    """world = 1 through decode_step (the gather is the identity): the plain decode."""
    from block_sparse_top_mean_b200.memory_parallel import BankShard, decode_step
    w = mi.Workload("mp1", "decode", 1, 50_000, 32, 8, 128, 64, 32, "bf16", n_query=8)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=4)
    sh = BankShard(kb, vb, w.block, 0)
    o, lse, idx = decode_step(q, sh, w.topk, w.scale, gather=lambda x: x[None])
    o_ref, lse_ref, idx_ref = msa.decode_fwd_tiled(q, sh.kbar_tiles, sh.k_tiles, sh.v_tiles,
                                                   w.seq, w.hkv, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref)
    # one shard: the combine only re-normalises the single partial (weight 1)
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_large_shards_take_the_certified_selection(msa):
    """Two shards of 8.5M tokens each: every shard's selection is the certified hi-plane
    path (keys written by the rescoring), and the merged selection is still exactly the
    unsharded one, whose bank (17M tokens) also takes that path."""
    from block_sparse_top_mean_b200.memory_parallel import BankShard, shard_ranges
    w = mi.Workload("mp_big", "decode", 1, 17_000_000, 4, 1, 128, 64, 32, "bf16", n_query=8)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=5)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    del khi, klo
    o_ref, lse_ref, idx_ref = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk,
                                                   w.scale)
    del kt, vt, bt
    shards = []
    for begin, count in shard_ranges(w.nb, 2):
        t0, t1 = begin * w.block, min(w.seq, (begin + count) * w.block)
        shards.append(BankShard(kb[t0:t1].contiguous(), vb[t0:t1].contiguous(), w.block, begin))
    keys = torch.stack([msa.decode_select_shard(q, sh.kbar_tiles, sh.seq, sh.hkv, w.block, w.topk,
                                                sh.block_begin) for sh in shards])
    o_parts, l_parts = [], []
    for sh in shards:
        idx, idx_local = msa.decode_merge_shards(keys, w.hq, w.d, sh.block_begin, sh.block_count)
        assert torch.equal(idx, idx_ref)
        o_p, l_p = msa.decode_attn_tiled(q, sh.k_tiles, sh.v_tiles, idx_local, sh.seq, sh.hkv,
                                         w.block, scale=w.scale)
        o_parts.append(o_p)
        l_parts.append(l_p)
    o, lse = msa.decode_combine_shards(torch.stack(o_parts), torch.stack(l_parts), w.hkv)
    torch.cuda.synchronize()
    # the combine re-weights per-shard partials: the one-bank result to the bf16 bars
    torch.testing.assert_close(o.float(), o_ref.float(), atol=2e-2, rtol=0)
    torch.testing.assert_close(lse, lse_ref, atol=2e-3, rtol=0)
