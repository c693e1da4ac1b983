"""Memory Parallel decode protocol on CPU ranks (gloo, world size 2 and 3).

Each rank owns a contiguous range of bank blocks (pooled keys, keys and values) and the
broadcast queries.  Per (query, group) it ranks its own blocks and all-gathers its best
k+1 (score, global block id); every rank merges the lists into the same global top-k;
each rank attends the selected blocks it owns and the (O, lse) partials are all-gathered
and merged by log-sum-exp.  The local arithmetic is the oracle's; what is under test is
the distributed protocol: the shard ranges, the id offsets, the collectives, and that the
result equals the unsharded decode on every rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

S, BLOCK, TOPK, HQ, HKV, D, NQ = 1500, 32, 8, 8, 2, 16, 4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _bank():
    rng = np.random.default_rng(5)
    K = rng.standard_normal((S, HKV, D)).astype(np.float32)
    V = rng.standard_normal((S, HKV, D)).astype(np.float32)
    Qd = rng.standard_normal((NQ, HQ, D)).astype(np.float32)
    return Qd, K, V


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    import oracle
    from block_sparse_top_mean_b200.memory_parallel import _all_gather, shard_ranges
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        Qd, K, V = _bank()
        kbar = oracle.pool_keys(K[None], BLOCK)[0]
        nb = kbar.shape[0]
        # the package's shard ranges (the ones the GPU decode uses) are the oracle's
        begin, count = shard_ranges(nb, world)[rank]
        lo, hi = oracle.shard_blocks(nb, world, rank)
        assert (begin, begin + count) == (lo, hi)
        # what this rank holds: its blocks' pooled keys and the keys/values of their tokens
        kb_mine = kbar[lo:hi]
        p_lo, p_hi = lo * BLOCK, min(S, hi * BLOCK)
        K_mine = np.zeros_like(K)
        V_mine = np.zeros_like(V)
        K_mine[p_lo:p_hi], V_mine[p_lo:p_hi] = K[p_lo:p_hi], V[p_lo:p_hi]
        G = HQ // HKV
        scale = 1 / np.sqrt(D)

        # 1. local candidates, padded to k+1 with (-inf, -1)
        sc = torch.full((NQ, HKV, TOPK + 1), float("-inf"), dtype=torch.float64)
        ids = torch.full((NQ, HKV, TOPK + 1), -1, dtype=torch.int64)
        for n in range(NQ):
            qs = oracle.group_query_sum(Qd[n], HKV)
            for g in range(HKV):
                for c, (s_, j) in enumerate(oracle.local_candidates(qs[g], kb_mine[:, g], lo,
                                                                    TOPK + 1)):
                    sc[n, g, c], ids[n, g, c] = s_, j
        # 2. all-gather and merge into the global selection (the same on every rank)
        # through the package's gather (the GPU decode's exchange): [world, ...], rank order
        all_sc = _all_gather(sc)
        all_ids = _all_gather(ids)
        idx = {}
        for n in range(NQ):
            for g in range(HKV):
                lists = [[(float(all_sc[r][n, g, c]), int(all_ids[r][n, g, c]))
                          for c in range(TOPK + 1) if int(all_ids[r][n, g, c]) >= 0]
                         for r in range(world)]
                idx[n, g] = oracle.merge_candidates(lists, TOPK)[0]
        # 3. partial attention over the owned selected blocks, all-gathered and merged
        O_r = torch.zeros((NQ, HQ, D), dtype=torch.float64)
        L_r = torch.full((NQ, HQ), float("-inf"), dtype=torch.float64)
        for (n, g), sel in idx.items():
            o, lse = oracle.attend_owned(Qd[n, g * G:(g + 1) * G], sel, lo, hi, K_mine, V_mine,
                                         S, BLOCK, g, scale)
            O_r[n, g * G:(g + 1) * G] = torch.from_numpy(o)
            L_r[n, g * G:(g + 1) * G] = torch.from_numpy(lse)
        all_O = _all_gather(O_r)
        all_L = _all_gather(L_r)
        O = np.zeros((NQ, HQ, D))
        L = np.zeros((NQ, HQ))
        for n in range(NQ):
            o, lse = oracle.merge_partials([a[n].numpy() for a in all_O],
                                           [a[n].numpy() for a in all_L])
            O[n], L[n] = o, lse

        # the unsharded decode, computed independently on every rank
        ref = oracle.decode_rows(Qd, kbar, K, V, S, BLOCK, TOPK, scale)
        err_o = err_l = 0.0
        same_idx = True
        for r in ref:
            same_idx &= (r.idx == idx[r.n, r.g])
            err_o = max(err_o, float(np.abs(O[r.n, r.g * G:(r.g + 1) * G] - r.O).max()))
            err_l = max(err_l, float(np.abs(L[r.n, r.g * G:(r.g + 1) * G] - r.lse).max()))
        out[rank] = (same_idx, err_o, err_l, (lo, hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_memory_parallel_protocol_equals_unsharded_decode(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    res = dict(out)
    assert sorted(res) == list(range(world))
    nb = -(-S // BLOCK)
    assert [res[r][3] for r in range(world)][0][0] == 0
    assert res[world - 1][3][1] == nb
    for r in range(world):
        same_idx, err_o, err_l, _ = res[r]
        assert same_idx
        assert err_o <= 1e-12 and err_l <= 1e-12
