"""Decode against a memory bank sharded over several devices, in fp64.  TEST INFRASTRUCTURE
ONLY (same rules as msa_oracle.py: tests, the smoke check and the bench's CPU legs).

Where it comes from: "100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it),
section "Das Gehirn mit zwei Geschwindigkeiten": the routing phase is spread over several
GPUs, each holding a part of the routing keys; the queries are broadcast, the relevance
scores are aggregated, and only the selected top-k documents are loaded.  The page names
the scheme Memory Parallel and gives no more detail.  Readings taken here:

* a shard is a contiguous range of bank blocks (with their keys and values); the ranges
  partition [0, nb) and block ids stay global;
* "aggregated" means: each shard ranks its own blocks for every (query, group) and sends
  its best k+1 as (score, global block id); the union of those lists is ranked by the
  same rule as the unsharded selection (score descending, block id ascending) and its
  first k are the selection.  This equals the unsharded top-k, because every block of
  the global top-(k+1) is among the top-(k+1) of its own shard (the extra candidate makes
  the first left-out score, the margin of the cut, exact as well);
* attention stays exact: each shard attends the selected blocks it owns and returns a
  partial (O_r, lse_r) (lse_r = -inf and O_r = 0 when it owns none); the partials are
  combined with weights exp(lse_r - lse), lse = log sum_r exp(lse_r), which is the
  softmax over the union of the keys.
"""
from __future__ import annotations

import numpy as np

from .msa_oracle import DecodeRow, attend_row, group_query_sum

__all__ = ["shard_blocks", "local_candidates", "merge_candidates", "attend_owned",
           "merge_partials", "decode_rows_sharded"]


def shard_blocks(nb: int, n_shards: int, r: int) -> tuple[int, int]:
    """Block range [lo, hi) of shard r: contiguous, sizes differ by at most one."""
    base, extra = divmod(nb, n_shards)
    lo = r * base + min(r, extra)
    return lo, lo + base + (1 if r < extra else 0)


def local_candidates(qs_g: np.ndarray, kbar_shard_g: np.ndarray, lo: int, n_best: int):
    """A shard's best `n_best` blocks for one (query, group).

    qs_g [d]: the group's summed query; kbar_shard_g [n, d]: the shard's pooled keys of
    that group, blocks lo .. lo + n - 1.  Returns a list of (score, global block id) in
    rank order (score descending, id ascending); shorter when the shard has fewer blocks."""
    scores = kbar_shard_g.astype(np.float64) @ qs_g.astype(np.float64)
    ids = lo + np.arange(scores.shape[0])
    order = np.lexsort((ids, -scores))[:n_best]
    return [(float(scores[i]), int(ids[i])) for i in order]


def merge_candidates(lists, topk: int):
    """Selection from the shards' candidate lists: (idx ascending and padded with -1,
    last taken score, first left-out score), the unsharded selection's convention."""
    cand = [c for lst in lists for c in lst]
    cand.sort(key=lambda c: (-c[0], c[1]))
    n_take = min(topk, len(cand))
    idx = sorted(c[1] for c in cand[:n_take]) + [-1] * (topk - n_take)
    last = cand[n_take - 1][0] if len(cand) > n_take else None
    first_left = cand[n_take][0] if len(cand) > n_take else None
    return idx, last, first_left


def attend_owned(q_heads, idx, lo: int, hi: int, K, V, S: int, block: int, g: int,
                 scale: float):
    """Partial attention of one (query, group) over the selected blocks in [lo, hi).

    Returns (O [G, d], lse [G]); lse = -inf and O = 0 when no selected block is owned.
    K, V: the bank [S, hkv, d] (global positions) or any object indexed as K[p, g]."""
    own = [j for j in idx if lo <= j < hi]
    G, d = q_heads.shape
    if not own:
        return np.zeros((G, d)), np.full(G, -np.inf)
    p = np.concatenate([np.arange(j * block, min(S, (j + 1) * block)) for j in own])
    return attend_row(q_heads, K[p, g], V[p, g], scale)


def merge_partials(Os, lses):
    """Combine partial attentions over disjoint key sets: (O, lse) of their union."""
    lses = np.asarray(lses, dtype=np.float64)             # [R, G]
    m = lses.max(axis=0)
    w = np.where(np.isfinite(lses), np.exp(lses - m), 0.0)
    den = w.sum(axis=0)
    O = sum(w[r][:, None] * Os[r] for r in range(len(Os))) / den[:, None]
    return O, m + np.log(den)


def decode_rows_sharded(Qd, kbar, K, V, S: int, block: int, topk: int, scale: float,
                        n_shards: int, queries=None):
    """Decode with the bank split into `n_shards` block ranges (see the module notes).

    Same arguments and result (a list of DecodeRow) as msa_oracle.decode_rows."""
    nq, hq, d = Qd.shape
    nb, hkv, _ = kbar.shape
    G = hq // hkv
    ranges = [shard_blocks(nb, n_shards, r) for r in range(n_shards)]
    if queries is None:
        queries = range(nq)
    out = []
    for n in queries:
        qs = group_query_sum(Qd[n], hkv)
        for g in range(hkv):
            lists = [local_candidates(qs[g], kbar[lo:hi, g, :], lo, topk + 1)
                     for lo, hi in ranges]
            idx, last, first = merge_candidates(lists, topk)
            parts = [attend_owned(Qd[n, g * G:(g + 1) * G], idx, lo, hi, K, V, S, block, g,
                                  scale) for lo, hi in ranges]
            O, lse = merge_partials([p[0] for p in parts], [p[1] for p in parts])
            out.append(DecodeRow(n, g, idx, last, first, O, lse))
    return out
