"""Plain fp64 CPU oracle of block-sparse top-k attention.  TEST INFRASTRUCTURE ONLY.

Only tests, the smoke check and the benchmark's CPU-baseline leg use this module; the
CUDA library never does.  Every function takes numpy arrays that hold the exact input
values (fp32 arrays for fp32 or bf16 inputs; bf16 values are exact in fp32) and does
all arithmetic in float64.

What it computes, and where that comes from:

* Block partition and pooled routing key per block.  "100 Millionen Token: Gedaechtnis
  oder Trugbild?" (aitalk.it), section "Das Gehirn mit zwei Geschwindigkeiten": each
  document gets small, strongly compressed routing keys that live on the GPU and decide
  relevance.  "MoBA" catalogue card (ross.abutalabs.com/products/moba.json), field
  what_it_is: top-k gating selects KV *blocks*.  The pages never state the pooling
  operator.  Reading taken here: the arithmetic mean of the block's keys, per KV head,
  over the tokens the block holds (a ragged last block averages its own tokens).
* Index-branch score.  "MiniMax released MSA: sparse attention speeds up 1M-token
  context processing by 28x", section "How MSA Works": the index branch selects, for
  each query and each GQA group, the top-k blocks.  Reading: the score of block j for
  token t and group g is the sum over the group's query heads of q_h . kbar_j, i.e.
  (sum_h q_h) . kbar_j, unscaled (a positive scale cannot change a ranking).
* Top-k.  Same section, and the MoBA card ("MoE-style top-k gating").  The pages are
  silent on ties, on the query's own block and on causality.  Readings: blocks are
  ranked by (score descending, block index ascending); in causal prefill the query's
  own block i = t // block is always taken and the other k-1 slots go to the best
  strictly-past blocks j < i (a future block is never eligible); when fewer than k-1
  past blocks exist all of them are taken and the index list is padded with -1.  In
  decode against a memory bank every block is eligible and the top k are taken.
* Main branch.  "MiniMax released MSA ...", sections "How MSA Works" and "Why Long
  Context is Hard to Scale": full, exact attention, but only over the selected blocks.
  Reading: one softmax per query head over the union of the selected blocks' keys,
  logits scale * q_h . k_p; inside the own block only keys p <= t are kept.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = [
    "pool_keys", "group_query_sum", "prefill_block_scores", "select_prefill_row",
    "select_decode_row", "attend_row", "prefill_rows", "decode_rows", "PrefillRow",
    "DecodeRow", "rel_gap", "prefill_keys_of", "decode_keys_of",
]


def pool_keys(K: np.ndarray, block: int) -> np.ndarray:
    """Mean of each block's keys.  K [b, S, hkv, d] -> kbar [b, nb, hkv, d] (fp64)."""
    b, S, hkv, d = K.shape
    nb = -(-S // block)
    kbar = np.empty((b, nb, hkv, d), dtype=np.float64)
    for j in range(nb):
        lo, hi = j * block, min(S, (j + 1) * block)
        kbar[:, j] = K[:, lo:hi].astype(np.float64).sum(axis=1) / (hi - lo)
    return kbar


def group_query_sum(q_tok: np.ndarray, hkv: int) -> np.ndarray:
    """Sum of the query heads of each GQA group.  q_tok [hq, d] -> [hkv, d] (fp64).

    Query head h belongs to group h // (hq // hkv)."""
    hq, d = q_tok.shape
    G = hq // hkv
    return q_tok.astype(np.float64).reshape(hkv, G, d).sum(axis=1)


def prefill_block_scores(q_tok: np.ndarray, kbar_b: np.ndarray, n_eligible: int) -> np.ndarray:
    """Scores of the first `n_eligible` blocks for one token: [hkv, n_eligible] (fp64).

    q_tok [hq, d] is the token's queries, kbar_b [nb, hkv, d] the pooled keys."""
    hkv = kbar_b.shape[1]
    qs = group_query_sum(q_tok, hkv)                               # [hkv, d]
    return np.einsum("gd,jgd->gj", qs, kbar_b[:n_eligible])


def rel_gap(a: float | None, b: float | None) -> float:
    """(a - b) / max(|a|, |b|): the relative margin between the last taken and the
    first left-out score (inf when nothing was left out)."""
    if a is None or b is None:
        return float("inf")
    den = max(abs(a), abs(b))
    return 0.0 if den == 0.0 else (a - b) / den


def _rank(scores: np.ndarray) -> np.ndarray:
    """Block ids ordered by (score descending, block index ascending)."""
    j = np.arange(scores.shape[0])
    return np.lexsort((j, -scores))


def select_prefill_row(scores_past: np.ndarray, own: int, topk: int):
    """Causal selection for one (token, group).

    scores_past: the scores of blocks 0..own-1.  Returns (idx, last_taken, first_left):
    idx has `topk` entries, ascending, padded with -1; the two scores bound the cut."""
    order = _rank(scores_past)
    n_take = min(topk - 1, order.shape[0])
    chosen = sorted([int(j) for j in order[:n_take]] + [own])
    idx = chosen + [-1] * (topk - len(chosen))
    last = float(scores_past[order[n_take - 1]]) if n_take >= 1 and order.shape[0] > n_take else None
    first_left = float(scores_past[order[n_take]]) if order.shape[0] > n_take else None
    return idx, last, first_left


def select_decode_row(scores: np.ndarray, topk: int):
    """Top-k of all blocks for one (query, group); same return convention."""
    order = _rank(scores)
    n_take = min(topk, order.shape[0])
    chosen = sorted(int(j) for j in order[:n_take])
    idx = chosen + [-1] * (topk - len(chosen))
    last = float(scores[order[n_take - 1]]) if order.shape[0] > n_take else None
    first_left = float(scores[order[n_take]]) if order.shape[0] > n_take else None
    return idx, last, first_left


def attend_row(q_heads: np.ndarray, k_keys: np.ndarray, v_keys: np.ndarray, scale: float):
    """Exact softmax attention of G query heads over n keys (fp64).

    q_heads [G, d], k_keys/v_keys [n, d] -> (O [G, d], lse [G]) with
    lse = log sum_p exp(scale * q . k_p)."""
    q = q_heads.astype(np.float64)
    k = k_keys.astype(np.float64)
    v = v_keys.astype(np.float64)
    logits = scale * (q @ k.T)                                     # [G, n]
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    den = w.sum(axis=1, keepdims=True)
    return (w @ v) / den, m[:, 0] + np.log(den[:, 0])


def prefill_keys_of(idx, t: int, S: int, block: int) -> np.ndarray:
    """Key positions of the selected blocks, keeping only p <= t (causal)."""
    pos = [np.arange(j * block, min(S, (j + 1) * block)) for j in idx if j >= 0]
    p = np.concatenate(pos) if pos else np.zeros(0, dtype=np.int64)
    return p[p <= t]


def decode_keys_of(idx, S: int, block: int) -> np.ndarray:
    pos = [np.arange(j * block, min(S, (j + 1) * block)) for j in idx if j >= 0]
    return np.concatenate(pos) if pos else np.zeros(0, dtype=np.int64)


@dataclass
class PrefillRow:
    b: int
    t: int
    g: int
    idx: list
    last_taken: float | None
    first_left: float | None
    O: np.ndarray          # [G, d] fp64, heads g*G .. g*G+G-1
    lse: np.ndarray        # [G] fp64

    @property
    def gap(self) -> float:
        return rel_gap(self.last_taken, self.first_left)


@dataclass
class DecodeRow:
    n: int
    g: int
    idx: list
    last_taken: float | None
    first_left: float | None
    O: np.ndarray
    lse: np.ndarray

    @property
    def gap(self) -> float:
        return rel_gap(self.last_taken, self.first_left)


def prefill_rows(Q, K, V, block: int, topk: int, scale: float, rows=None, kbar=None,
                 idx_override=None):
    """Causal prefill for the requested (b, t) rows, every GQA group.

    Q [b, S, hq, d], K/V [b, S, hkv, d] (exact input values).  rows: iterable of (b, t);
    all rows when None.  kbar: this module's pool_keys(K, block), recomputed if None.
    idx_override: optional {(b, t, g): idx} to attend a given selection instead (used to
    check a kernel's output on rows whose selection is a near-tie).
    Returns a list of PrefillRow."""
    bsz, S, hq, d = Q.shape
    hkv = K.shape[2]
    G = hq // hkv
    if kbar is None:
        kbar = pool_keys(K, block)
    if rows is None:
        rows = [(b, t) for b in range(bsz) for t in range(S)]
    out = []
    for b, t in rows:
        i = t // block
        sc = prefill_block_scores(Q[b, t], kbar[b], i)               # [hkv, i]
        for g in range(hkv):
            idx, last, first = select_prefill_row(sc[g], i, topk)
            use = idx if idx_override is None else idx_override.get((b, t, g), idx)
            p = prefill_keys_of(use, t, S, block)
            O, lse = attend_row(Q[b, t, g * G:(g + 1) * G], K[b, p, g], V[b, p, g], scale)
            out.append(PrefillRow(b, t, g, idx, last, first, O, lse))
    return out


def decode_rows(Qd, kbar, K, V, S: int, block: int, topk: int, scale: float, queries=None,
                idx_override=None):
    """Decode of independent queries against a memory bank (no causal mask).

    Qd [n_query, hq, d]; kbar [nb, hkv, d] from pool_keys over the bank; K, V are the
    bank [S, hkv, d] or any object whose K[p, g] returns a numpy [len(p), d] array.
    Returns a list of DecodeRow, one per (query, group)."""
    nq, hq, d = Qd.shape
    hkv = kbar.shape[1]
    G = hq // hkv
    if queries is None:
        queries = range(nq)
    out = []
    for n in queries:
        qs = group_query_sum(Qd[n], hkv)                             # [hkv, d]
        for g in range(hkv):
            sc = kbar[:, g, :] @ qs[g]                               # [nb]
            idx, last, first = select_decode_row(sc, topk)
            use = idx if idx_override is None else idx_override.get((n, g), idx)
            p = decode_keys_of(use, S, block)
            O, lse = attend_row(Qd[n, g * G:(g + 1) * G], K[p, g], V[p, g], scale)
            out.append(DecodeRow(n, g, idx, last, first, O, lse))
    return out
