"""Pins for the sharded-bank (Memory Parallel) decode oracle: whatever the number and size
of the shards, the selection and the output equal those of the unsharded decode oracle,
which is itself pinned against brute force and dense attention (test_oracle_pins.py)."""
import numpy as np
import pytest

import oracle


def _bank(seed, S, hq, hkv, d, block, nq):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((S, hkv, d)).astype(np.float32)
    V = rng.standard_normal((S, hkv, d)).astype(np.float32)
    Qd = rng.standard_normal((nq, hq, d)).astype(np.float32)
    kbar = oracle.pool_keys(K[None], block)[0]
    return Qd, K, V, kbar


@pytest.mark.parametrize("nb,n", [(10, 3), (7, 7), (5, 8), (156_250, 8), (1, 2), (64, 1)])
def test_shard_ranges_partition_the_blocks(nb, n):
    ranges = [oracle.shard_blocks(nb, n, r) for r in range(n)]
    assert ranges[0][0] == 0 and ranges[-1][1] == nb
    for (a, b), (c, _) in zip(ranges, ranges[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("seed,S,block,topk,n_shards", [
    (0, 1000, 16, 8, 2),        # 63 blocks, ragged last block
    (1, 1000, 16, 8, 5),
    (2, 640, 64, 4, 3),         # shards of 4, 3, 3 blocks: one shard holds fewer than k+1
    (3, 300, 64, 8, 2),         # 5 blocks < k: padded with -1
    (4, 2048, 32, 32, 7),
])
def test_sharded_decode_equals_unsharded(seed, S, block, topk, n_shards):
    Qd, K, V, kbar = _bank(seed, S, 8, 2, 32, block, 5)
    scale = 1 / np.sqrt(32)
    ref = oracle.decode_rows(Qd, kbar, K, V, S, block, topk, scale)
    got = oracle.decode_rows_sharded(Qd, kbar, K, V, S, block, topk, scale, n_shards)
    assert len(ref) == len(got)
    for a, b in zip(ref, got):
        assert (a.n, a.g) == (b.n, b.g)
        assert a.idx == b.idx
        # the margin of the cut: same scores, summed in slices of another length
        for x, y in [(a.last_taken, b.last_taken), (a.first_left, b.first_left)]:
            assert (x is None) == (y is None)
            if x is not None:
                assert abs(x - y) <= 1e-12 * max(1.0, abs(x))
        np.testing.assert_allclose(b.O, a.O, rtol=0, atol=1e-12)
        np.testing.assert_allclose(b.lse, a.lse, rtol=0, atol=1e-12)


def test_sharded_selection_with_exact_ties_across_shards():
    """Equal scores in different shards: the lower global block id wins, as unsharded.
    Integer pooled keys and queries make every score exact, whatever the summation order."""
    S, block, topk = 512, 16, 4
    Qd, K, V, _ = _bank(7, S, 4, 1, 16, block, 2)
    rng = np.random.default_rng(8)
    Qd = rng.integers(1, 4, Qd.shape).astype(np.float64)            # positive group sums
    kbar = rng.integers(-3, 4, (S // block, 1, 16)).astype(np.float64)
    tied = [3, 9, 20, 29, 31]                   # five equal top scores around a cut of four
    kbar[tied] = 40.0
    scale = 0.25
    for n_shards in (2, 3, 4):
        ref = oracle.decode_rows(Qd, kbar, K, V, S, block, topk, scale)
        got = oracle.decode_rows_sharded(Qd, kbar, K, V, S, block, topk, scale, n_shards)
        assert [r.idx for r in got] == [r.idx for r in ref] == [tied[:4]] * len(ref)


def test_cut_margin_when_one_shard_holds_the_whole_top():
    """All of the global top-(k+1) lie in one shard: the first left-out score (the margin
    the parity gate reads) must still be the unsharded one."""
    S, block, topk = 1024, 16, 8                    # 64 blocks, two shards of 32
    Qd, K, V, _ = _bank(9, S, 4, 1, 16, block, 3)
    rng = np.random.default_rng(10)
    Qd = rng.integers(1, 4, Qd.shape).astype(np.float64)
    kbar = rng.integers(-3, 4, (S // block, 1, 16)).astype(np.float64)
    kbar[:topk + 1] = 10.0 + np.arange(topk + 1)[:, None, None]   # blocks 0..k, shard 0
    ref = oracle.decode_rows(Qd, kbar, K, V, S, block, topk, 0.25)
    got = oracle.decode_rows_sharded(Qd, kbar, K, V, S, block, topk, 0.25, 2)
    for a, b in zip(ref, got):
        assert a.idx == b.idx == list(range(1, topk + 1))
        assert a.first_left == b.first_left and a.last_taken == b.last_taken


def test_merge_partials_is_attention_over_the_union():
    """Attention over a key set split into disjoint parts (one empty) and merged by the
    log-sum-exp rule equals attention over the whole set."""
    rng = np.random.default_rng(11)
    q = rng.standard_normal((4, 16))
    k = rng.standard_normal((50, 16))
    v = rng.standard_normal((50, 16))
    O, lse = oracle.attend_row(q, k, v, 0.3)
    cuts = [0, 7, 7, 31, 50]
    parts = []
    for a, b in zip(cuts, cuts[1:]):
        if a == b:
            parts.append((np.zeros((4, 16)), np.full(4, -np.inf)))
        else:
            parts.append(oracle.attend_row(q, k[a:b], v[a:b], 0.3))
    O2, lse2 = oracle.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


def test_local_candidates_rank_and_global_ids():
    qs = np.array([1.0, 0.0])
    kb = np.array([[0.5, 9.0], [2.0, 0.0], [0.5, -1.0], [3.0, 3.0]])
    got = oracle.local_candidates(qs, kb, 100, 3)
    assert got == [(3.0, 103), (2.0, 101), (0.5, 100)]
