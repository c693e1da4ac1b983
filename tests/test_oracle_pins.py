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
