"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names the mistake it is there to catch.  Sources of truth: a hand-derived
worked example (tests/golden), closed forms, library routines (torch's avg_pool1d and
scaled_dot_product_attention in fp64), brute force over subsets, and invariants.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import msa_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _sdpa(Q, K, V, scale, mask):
    """torch fp64 SDPA with GQA: Q [S, hq, d], K/V [S, hkv, d], mask [S, S] bool (True keeps)."""
    q = torch.from_numpy(Q.astype(np.float64)).permute(1, 0, 2)
    G = Q.shape[1] // K.shape[1]
    k = torch.from_numpy(K.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    v = torch.from_numpy(V.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
    m = torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    logits = scale * (q @ k.transpose(1, 2))
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.numpy()          # [S, hq, d], [hq, S]


def _rows_to_arrays(rows, S, hq, hkv, d):
    G = hq // hkv
    O = np.zeros((S, hq, d))
    L = np.zeros((hq, S))
    for r in rows:
        O[r.t, r.g * G:(r.g + 1) * G] = r.O
        L[r.g * G:(r.g + 1) * G, r.t] = r.lse
    return O, L


# ---------------------------------------------------------------- worked example

def _ev(expr):
    return eval(expr, {"__builtins__": {}}, {"e": math.e, "log": math.log})


def test_worked_example_prefill():
    """Hand-derived 6-token example: pooling, the tie to the lower index, causal mask."""
    ex = json.load(open(os.path.join(GOLDEN, "worked_example_s6_b2.json")))
    sh = ex["shape"]
    K = np.array(ex["K"], np.float32)[None, :, None, :]
    V = np.array(ex["V"], np.float32)[None, :, None, :]
    Q = np.array(ex["Q"], np.float32)[None]
    kbar = oracle.pool_keys(K, sh["block"])
    np.testing.assert_array_equal(kbar[0, :, 0, :], np.array(ex["kbar"]))
    rows = oracle.prefill_rows(Q, K, V, sh["block"], sh["topk"], sh["scale"])
    assert len(rows) == 6
    for r in rows:
        want = ex["prefill"][f"t{r.t}"]
        assert r.idx == want["idx"], (r.t, r.idx)
        np.testing.assert_allclose(r.O, [[_ev(x) for x in h] for h in want["O"]], atol=1e-14)
        np.testing.assert_allclose(r.lse, [_ev(x) for x in want["lse"]], atol=1e-14)


def test_worked_example_decode():
    ex = json.load(open(os.path.join(GOLDEN, "worked_example_s6_b2.json")))
    sh = ex["shape"]
    K = np.array(ex["K"], np.float32)[:, None, :]
    V = np.array(ex["V"], np.float32)[:, None, :]
    kbar = oracle.pool_keys(K[None], sh["block"])[0]
    Qd = np.array(ex["decode"]["Q"], np.float32)[None]
    (r,) = oracle.decode_rows(Qd, kbar, K, V, 6, sh["block"], sh["topk"], sh["scale"])
    assert r.idx == ex["decode"]["idx"]
    np.testing.assert_allclose(r.O, [[_ev(x) for x in h] for h in ex["decode"]["O"]], atol=1e-14)
    np.testing.assert_allclose(r.lse, [_ev(x) for x in ex["decode"]["lse"]], atol=1e-14)


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("S,block", [(256, 64), (250, 64), (7, 3), (64, 64)])
def test_pool_keys_ramp_closed_form(S, block):
    """Keys linear in t: the block mean is the value at the block's mid-position.
    Catches a wrong divisor for the ragged last block and a wrong reduction axis."""
    hkv, d = 3, 5
    a = np.arange(hkv * d, dtype=np.float32).reshape(hkv, d)
    c = (np.arange(hkv * d, dtype=np.float32).reshape(hkv, d) % 4) - 1.5
    t = np.arange(S, dtype=np.float32)[:, None, None]
    K = (a + c * t)[None]
    kbar = oracle.pool_keys(K, block)
    for j in range(kbar.shape[1]):
        lo, hi = j * block, min(S, (j + 1) * block)
        np.testing.assert_allclose(kbar[0, j], a + c * (lo + hi - 1) / 2.0, rtol=0, atol=1e-9)


@pytest.mark.parametrize("S,block", [(512, 64), (1000, 128), (96, 1)])
def test_pool_keys_vs_avg_pool1d(S, block):
    """Library routine: torch avg_pool1d (ceil mode divides a ragged window by its size)."""
    K = _rand((2, S, 2, 16), 1)
    kbar = oracle.pool_keys(K, block)
    x = torch.from_numpy(K.astype(np.float64)).permute(0, 2, 3, 1).reshape(-1, 1, S)
    ref = F.avg_pool1d(x, block, block, ceil_mode=True).reshape(2, 2, 16, -1).permute(0, 3, 1, 2)
    np.testing.assert_allclose(kbar, ref.numpy(), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- selection

def _brute_best_subset(scores, n_take):
    """Brute force over subsets: the set with the largest total score (no ties here)."""
    best, arg = -math.inf, None
    for sub in itertools.combinations(range(len(scores)), n_take):
        s = sum(scores[j] for j in sub)
        if s > best:
            best, arg = s, sub
    return sorted(arg)


@pytest.mark.parametrize("seed", range(4))
def test_selection_equals_brute_force_subset(seed):
    """Taking the k-1 best past blocks = the subset of past blocks with the largest sum.
    Catches a flipped sort direction and an off-by-one in the number taken."""
    S, block, hq, hkv, d, topk = 96, 8, 4, 2, 16, 4
    Q, K, V = _rand((1, S, hq, d), seed), _rand((1, S, hkv, d), seed + 10), _rand((1, S, hkv, d), 3)
    rows = oracle.prefill_rows(Q, K, V, block, topk, 0.25)
    kbar = oracle.pool_keys(K, block)
    for r in rows:
        i = r.t // block
        qs = Q[0, r.t].astype(np.float64).reshape(hkv, hq // hkv, d).sum(1)[r.g]
        sc = [float(qs @ kbar[0, j, r.g]) for j in range(i)]
        want = sorted(_brute_best_subset(sc, min(topk - 1, i)) + [i])
        assert [j for j in r.idx if j >= 0] == want


def test_selection_ties_go_to_lower_index():
    """All-zero queries make every score 0: the k-1 lowest past blocks are taken."""
    S, block, topk = 64, 4, 5
    Q = np.zeros((1, S, 2, 8), np.float32)
    K, V = _rand((1, S, 1, 8), 1), _rand((1, S, 1, 8), 2)
    for r in oracle.prefill_rows(Q, K, V, block, topk, 1.0):
        i = r.t // block
        assert r.idx[:min(topk - 1, i)] == list(range(min(topk - 1, i)))
        assert i in r.idx


def test_selection_invariants_random():
    """Own block present, nothing in the future, distinct ascending, |set| = min(k, i+1),
    padding with -1 at the end."""
    S, block, topk = 300, 16, 6                       # ragged last block (300 = 18*16 + 12)
    Q, K, V = _rand((2, S, 4, 8), 5), _rand((2, S, 1, 8), 6), _rand((2, S, 1, 8), 7)
    for r in oracle.prefill_rows(Q, K, V, block, topk, 0.3):
        i = r.t // block
        sel = [j for j in r.idx if j >= 0]
        assert i in sel and max(sel) == i
        assert sel == sorted(set(sel))
        assert len(sel) == min(topk, i + 1)
        assert r.idx[len(sel):] == [-1] * (topk - len(sel))


def test_selection_group_mapping_planted():
    """Query head h belongs to group h // G.  Plant direction u in block 5 for both KV
    heads, add +u to the queries of group 1 and -u to those of group 0: group 1 always
    takes block 5, group 0 never.  A head->group mapping of h % hkv cancels u in both
    group sums and fails."""
    S, block, hq, hkv, d, topk = 256, 16, 4, 2, 32, 3
    rng = np.random.default_rng(0)
    Q = 0.1 * rng.standard_normal((1, S, hq, d)).astype(np.float32)
    K = 0.1 * rng.standard_normal((1, S, hkv, d)).astype(np.float32)
    V = rng.standard_normal((1, S, hkv, d)).astype(np.float32)
    u = np.zeros(d, np.float32)
    u[3] = 1.0
    K[0, 5 * block:6 * block, :] += 4 * u                 # block 5, both KV heads
    Q[0, :, 2:4] += 4 * u                                 # heads 2,3 = group 1 (G = 2)
    Q[0, :, 0:2] -= 4 * u                                 # heads 0,1 = group 0
    for r in oracle.prefill_rows(Q, K, V, block, topk, 0.2):
        if r.t // block > 5:
            assert (5 in r.idx) == (r.g == 1), (r.t, r.g, r.idx)


def test_selection_positive_rescale_invariant():
    S, block, topk = 128, 8, 4
    Q, K, V = _rand((1, S, 2, 8), 11), _rand((1, S, 1, 8), 12), _rand((1, S, 1, 8), 13)
    a = [r.idx for r in oracle.prefill_rows(Q, K, V, block, topk, 0.3)]
    b = [r.idx for r in oracle.prefill_rows(Q * np.float32(2.0), K, V, block, topk, 0.3)]
    assert a == b


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("S,block,hq,hkv", [(128, 16, 4, 2), (100, 16, 2, 1), (64, 64, 2, 2)])
def test_all_blocks_equals_dense_causal_sdpa(S, block, hq, hkv):
    """top-k >= nb: sparse attention is dense causal GQA attention (library routine).
    Catches a missing scale, p < t instead of p <= t, a transposed product, a wrong lse,
    and a wrong key range for a ragged last block."""
    d, scale = 16, 0.37
    Q, K, V = _rand((1, S, hq, d), 21), _rand((1, S, hkv, d), 22), _rand((1, S, hkv, d), 23)
    nb = -(-S // block)
    rows = oracle.prefill_rows(Q, K, V, block, nb + 2, scale)
    O, L = _rows_to_arrays(rows, S, hq, hkv, d)
    Oref, Lref = _sdpa(Q[0], K[0], V[0], scale, np.tril(np.ones((S, S), bool)))
    np.testing.assert_allclose(O, Oref, atol=1e-12)
    np.testing.assert_allclose(L, Lref, atol=1e-12)


def test_block_size_one_full_topk_is_dense_causal():
    S, hq, hkv, d = 40, 2, 1, 8
    Q, K, V = _rand((1, S, hq, d), 31), _rand((1, S, hkv, d), 32), _rand((1, S, hkv, d), 33)
    rows = oracle.prefill_rows(Q, K, V, 1, S, 0.5)
    O, _ = _rows_to_arrays(rows, S, hq, hkv, d)
    Oref, _ = _sdpa(Q[0], K[0], V[0], 0.5, np.tril(np.ones((S, S), bool)))
    np.testing.assert_allclose(O, Oref, atol=1e-12)


def test_topk_one_is_block_local_causal():
    """k = 1 keeps only the own block: block-diagonal causal attention."""
    S, block, hq, hkv, d = 96, 32, 2, 1, 16
    Q, K, V = _rand((1, S, hq, d), 41), _rand((1, S, hkv, d), 42), _rand((1, S, hkv, d), 43)
    rows = oracle.prefill_rows(Q, K, V, block, 1, 0.25)
    O, _ = _rows_to_arrays(rows, S, hq, hkv, d)
    t = np.arange(S)
    mask = (t[:, None] // block == t[None, :] // block) & (t[None, :] <= t[:, None])
    Oref, _ = _sdpa(Q[0], K[0], V[0], 0.25, mask)
    np.testing.assert_allclose(O, Oref, atol=1e-12)


def test_constant_values_pass_through():
    S, block = 80, 8
    Q, K = _rand((1, S, 4, 8), 51), _rand((1, S, 2, 8), 52)
    V = np.broadcast_to(np.arange(8, dtype=np.float32), (1, S, 2, 8)).copy()
    for r in oracle.prefill_rows(Q, K, V, block, 3, 1.0):
        np.testing.assert_allclose(r.O, np.broadcast_to(np.arange(8.0), r.O.shape), atol=1e-12)


def test_weights_sum_to_one_via_lse():
    """sum_p exp(scale q.k_p - lse) = 1 over the keys the row attends."""
    S, block, topk, scale = 120, 8, 3, 0.4
    Q, K, V = _rand((1, S, 2, 8), 61), _rand((1, S, 1, 8), 62), _rand((1, S, 1, 8), 63)
    for r in oracle.prefill_rows(Q, K, V, block, topk, scale):
        p = oracle.prefill_keys_of(r.idx, r.t, S, block)
        for hh in range(2):
            lg = scale * (K[0, p, 0].astype(np.float64) @ Q[0, r.t, hh].astype(np.float64))
            assert abs(np.exp(lg - r.lse[hh]).sum() - 1.0) < 1e-12


# ---------------------------------------------------------------- decode

def test_decode_all_blocks_equals_dense_sdpa():
    S, block, hq, hkv, d, scale = 200, 16, 4, 2, 8, 0.3     # ragged last bank block
    K, V = _rand((S, hkv, d), 71), _rand((S, hkv, d), 72)
    Qd = _rand((3, hq, d), 73)
    kbar = oracle.pool_keys(K[None], block)[0]
    rows = oracle.decode_rows(Qd, kbar, K, V, S, block, kbar.shape[0], scale)
    G = hq // hkv
    for r in rows:
        o, lse = _sdpa(Qd[r.n][None, r.g * G:(r.g + 1) * G], K[:, r.g:r.g + 1],
                       V[:, r.g:r.g + 1], scale, np.ones((1, S), bool))
        np.testing.assert_allclose(r.O, o[0], atol=1e-12)
        np.testing.assert_allclose(r.lse, lse[:, 0], atol=1e-12)


def test_decode_selection_equals_brute_force_subset():
    S, block, hq, hkv, d, topk = 96, 8, 2, 1, 8, 3
    K, V = _rand((S, hkv, d), 81), _rand((S, hkv, d), 82)
    Qd = _rand((5, hq, d), 83)
    kbar = oracle.pool_keys(K[None], block)[0]
    for r in oracle.decode_rows(Qd, kbar, K, V, S, block, topk, 0.5):
        qs = Qd[r.n].astype(np.float64).sum(0)
        sc = [float(qs @ kbar[j, 0]) for j in range(kbar.shape[0])]
        assert r.idx == _brute_best_subset(sc, topk)


# ---------------------------------------------------------------- the planted workload

def test_planted_blocks_always_selected_after_they_appear():
    """The planted workload adds 3u to keys of 1% of blocks and to every query: those
    blocks score far above the rest and are taken by every later token.  Small version
    of the 128K workload's recipe (same generator, fewer tokens)."""
    w = mi.WORKLOADS["prefill_128k_b128_k16_planted"].with_(seq=2048, block=64, hq=8, hkv=2,
                                                            d=64, dtype="f32",
                                                            planted_frac=0.1, topk=6)
    q, k, v = mi.prefill_inputs(w)
    pl = mi.planted_blocks(w.nb, w.planted_frac, 0)
    assert len(pl) == 3
    Q, K, V = q.numpy(), k.numpy(), v.numpy()
    rows = [(0, t) for t in range(0, w.seq, 37)]
    for r in oracle.prefill_rows(Q, K, V, w.block, w.topk, w.scale, rows=rows):
        for j in pl:
            if j < r.t // w.block:
                assert j in r.idx, (r.t, r.g, j, r.idx)


# ---------------------------------------------------------------- the parity gate
# last_taken / first_left and their relative gap decide which rows must match the
# oracle's selection exactly; these pins hold them to values derived outside the oracle.

def _gate_value(x):
    return None if x is None else float(_ev(x))


def test_worked_example_gate_prefill():
    """Hand-derived cut scores of every row: t4 (gap 0.5), the exact tie at t5 (gap 0),
    and the rows where nothing is left out (infinite gap)."""
    ex = json.load(open(os.path.join(GOLDEN, "worked_example_s6_b2.json")))
    sh = ex["shape"]
    K = np.array(ex["K"], np.float32)[None, :, None, :]
    V = np.array(ex["V"], np.float32)[None, :, None, :]
    Q = np.array(ex["Q"], np.float32)[None]
    for r in oracle.prefill_rows(Q, K, V, sh["block"], sh["topk"], sh["scale"]):
        want = ex["prefill"][f"t{r.t}"]["gate"]
        assert r.last_taken == _gate_value(want["last_taken"]), r.t
        assert r.first_left == _gate_value(want["first_left"]), r.t
        gap = math.inf if want["gap"] is None else float(_ev(want["gap"]))
        assert r.gap == gap, (r.t, r.gap)


def test_worked_example_gate_decode():
    ex = json.load(open(os.path.join(GOLDEN, "worked_example_s6_b2.json")))
    sh = ex["shape"]
    K = np.array(ex["K"], np.float32)[:, None, :]
    kbar = oracle.pool_keys(K[None], sh["block"])[0]
    Qd = np.array(ex["decode"]["Q"], np.float32)[None]
    (r,) = oracle.decode_rows(Qd, kbar, K, K, 6, sh["block"], sh["topk"], sh["scale"])
    want = ex["decode"]["gate"]
    assert (r.last_taken, r.first_left) == (float(want["last_taken"]), float(want["first_left"]))
    assert r.gap == float(want["gap"])


@pytest.mark.parametrize("a,b,gap", [(2.0, 1.0, 0.5), (2.0, 2.0, 0.0), (-1.0, -2.0, 0.5),
                                     (-2.0, -2.0, 0.0), (1.0, -1.0, 2.0), (0.0, 0.0, 0.0),
                                     (3.0, 0.0, 1.0), (0.0, -4.0, 1.0), (1e-3, -1e-3, 2.0)])
def test_rel_gap_closed_forms(a, b, gap):
    """(a - b) / max(|a|, |b|) by hand, including negative scores, where the larger
    magnitude is the left-out score's (-1 vs -2 gives 1/2, not 1)."""
    assert oracle.rel_gap(a, b) == gap


def test_rel_gap_nothing_left_out_is_infinite():
    assert oracle.rel_gap(None, 1.0) == math.inf
    assert oracle.rel_gap(1.0, None) == math.inf
    assert oracle.rel_gap(None, None) == math.inf


def _kth_by_counting(vals, k):
    """The k-th largest value (k >= 1) found by counting, not sorting: the v with
    #{x > v} < k <= #{x >= v}."""
    for v in vals:
        if sum(x > v for x in vals) < k <= sum(x >= v for x in vals):
            return v
    raise AssertionError("no k-th value")


@pytest.mark.parametrize("seed", range(6))
def test_prefill_cut_scores_by_counting(seed):
    """Random rows, scores rounded to a coarse grid so ties occur: last_taken is the
    (k-1)-th best past score and first_left the k-th, found by counting.  Covers
    negative scores, rows with fewer eligible blocks than k-1 (nothing left out) and
    top-k 1 (nothing ranked: infinite gap)."""
    rng = np.random.default_rng(seed)
    for _ in range(200):
        n_past = int(rng.integers(0, 12))
        topk = int(rng.integers(1, 8))
        sc = np.round(rng.standard_normal(n_past) * 2, 0 if seed % 2 else 1)
        idx, last, first = oracle.select_prefill_row(sc, n_past, topk)
        vals = [float(x) for x in sc]
        n_take = min(topk - 1, n_past)
        assert idx[:n_take + 1] == sorted(idx[:n_take + 1]) and n_past in idx
        if n_take == 0 or n_past <= n_take:
            assert last is None or n_past <= n_take
            assert oracle.rel_gap(last, first) == math.inf
        if n_take >= 1 and n_past > n_take:
            assert last == _kth_by_counting(vals, n_take)
            assert first == _kth_by_counting(vals, n_take + 1)
        else:
            assert last is None
        # every taken past block scores >= last_taken >= first_left >= every left-out one
        taken = [j for j in idx if 0 <= j < n_past]
        assert len(taken) == n_take
        if last is not None:
            left = [j for j in range(n_past) if j not in taken]
            assert min(vals[j] for j in taken) == last
            assert max(vals[j] for j in left) == first


@pytest.mark.parametrize("seed", range(4))
def test_decode_cut_scores_by_counting(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(200):
        nb = int(rng.integers(1, 14))
        topk = int(rng.integers(1, 9))
        sc = np.round(rng.standard_normal(nb) * 3, 0 if seed % 2 else 1)
        idx, last, first = oracle.select_decode_row(sc, topk)
        vals = [float(x) for x in sc]
        if nb > topk:
            assert last == _kth_by_counting(vals, topk)
            assert first == _kth_by_counting(vals, topk + 1)
            taken = [j for j in idx if j >= 0]
            assert min(vals[j] for j in taken) == last
            assert max(vals[j] for j in range(nb) if j not in taken) == first
        else:
            assert last is None and first is None
            assert oracle.rel_gap(last, first) == math.inf


def test_decode_gap_closed_form():
    """Scores (qsum . kbar_j) = j for a bank whose block j has pooled key j * e0 and a
    query sum e0: top-3 of 10 blocks takes {7, 8, 9}, last_taken 7, first_left 6, gap
    1/7; with the query negated the lowest blocks win and the gap is (-2 + 3) / 3."""
    nb, block, d = 10, 4, 8
    K = np.zeros((nb * block, 1, d), np.float32)
    for j in range(nb):
        K[j * block:(j + 1) * block, 0, 0] = j
    kbar = oracle.pool_keys(K[None], block)[0]
    q = np.zeros((1, 2, d), np.float32)
    q[0, 0, 0] = 1.0
    (r,) = oracle.decode_rows(q, kbar, K, K, nb * block, block, 3, 1.0)
    assert (r.idx, r.last_taken, r.first_left) == ([7, 8, 9], 7.0, 6.0)
    assert r.gap == 1.0 / 7.0
    q[0, 0, 0] = -1.0
    (r,) = oracle.decode_rows(q, kbar, K, K, nb * block, block, 3, 1.0)
    assert (r.idx, r.last_taken, r.first_left) == ([0, 1, 2], -2.0, -3.0)
    assert r.gap == 1.0 / 3.0


def test_strict_rows_are_stable_under_small_perturbations():
    """What the gate means: when the gap exceeds 1e-3, moving every score by less than
    a quarter of the margin cannot change the selection; a row built with a smaller
    margin flips when its two cut scores move apart the other way."""
    rng = np.random.default_rng(7)
    n_strict = 0
    for _ in range(300):
        sc = rng.standard_normal(20)
        idx, last, first = oracle.select_prefill_row(sc, 20, 6)
        gap = oracle.rel_gap(last, first)
        if gap <= 1e-3:
            continue
        n_strict += 1
        margin = (last - first) / 4
        noise = rng.uniform(-margin, margin, size=20) * 0.999
        assert oracle.select_prefill_row(sc + noise, 20, 6)[0] == idx
    assert n_strict > 250
    sc = np.array([5.0, 1.0, 1.0 + 5e-4, 0.0])        # blocks 1, 2 within the 1e-3 band
    idx, last, first = oracle.select_prefill_row(sc, 4, 3)
    assert idx == [0, 2, 4] and oracle.rel_gap(last, first) <= 1e-3
    sc2 = sc.copy()
    sc2[1] += 1e-3
    assert oracle.select_prefill_row(sc2, 4, 3)[0] == [0, 1, 4]
