"""Backward pass of the causal block-sparse attention, in fp64.  TEST INFRASTRUCTURE ONLY
(same rules as msa_oracle.py).

Where it comes from: "100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it),
section "Eleganter Proof-of-Concept oder fertiges System?": the router and the sparse
attention are trained end to end (with an extra routing loss the page does not define);
"MiniMax released MSA ...", section "How MSA Works": the main branch is exact attention
over the selected blocks.  Readings taken here:

* the selection is held fixed.  Top-k is piecewise constant in its inputs, so it passes
  no gradient; the pooled keys receive none through it (a routing loss would be a separate
  term, and the pages do not define one);
* the rest is the gradient of exact softmax attention over the selected keys.  For one
  query head with logits s_p = scale * q . k_p over its key set U, weights P_p =
  softmax(s)_p and output O = sum_p P_p v_p, an upstream gradient dO gives
      dv_p += P_p dO,      dP_p = dO . v_p,      dS_p = P_p (dP_p - dO . O),
      dq = scale * sum_p dS_p k_p,      dk_p += scale * dS_p q.
  Keys shared by several queries (or heads of a group) accumulate their contributions.
"""
from __future__ import annotations

import numpy as np

from .msa_oracle import pool_keys, prefill_block_scores, prefill_keys_of, select_prefill_row

__all__ = ["attend_row_backward", "prefill_backward"]


def attend_row_backward(q_heads, k_keys, v_keys, dO, scale: float):
    """Gradients of G heads' attention over n keys (fp64).

    q_heads [G, d], k_keys/v_keys [n, d], dO [G, d] -> (dq [G, d], dk [n, d], dv [n, d])."""
    q = np.asarray(q_heads, dtype=np.float64)
    k = np.asarray(k_keys, dtype=np.float64)
    v = np.asarray(v_keys, dtype=np.float64)
    g = np.asarray(dO, dtype=np.float64)
    s = scale * (q @ k.T)                                   # [G, n]
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    O = P @ v                                               # [G, d]
    dv = P.T @ g                                            # [n, d]
    dP = g @ v.T                                            # [G, n]
    dS = P * (dP - (g * O).sum(axis=1, keepdims=True))
    dq = scale * (dS @ k)
    dk = scale * (dS.T @ q)
    return dq, dk, dv


def prefill_backward(Q, K, V, dO, block: int, topk: int, scale: float, kbar=None,
                     idx_override=None):
    """dQ, dK, dV (fp64, shapes of Q, K, V) of the causal sparse prefill for upstream dO
    [b, S, hq, d], with every row's selection computed as in msa_oracle.prefill_rows (or
    given by idx_override {(b, t, g): idx}) and held fixed."""
    bsz, S, hq, d = Q.shape
    hkv = K.shape[2]
    G = hq // hkv
    if kbar is None:
        kbar = pool_keys(K, block)
    dQ = np.zeros(Q.shape, dtype=np.float64)
    dK = np.zeros(K.shape, dtype=np.float64)
    dV = np.zeros(V.shape, dtype=np.float64)
    for b in range(bsz):
        for t in range(S):
            i = t // block
            sc = prefill_block_scores(Q[b, t], kbar[b], i)
            for g in range(hkv):
                idx = select_prefill_row(sc[g], i, topk)[0]
                if idx_override is not None:
                    idx = idx_override.get((b, t, g), idx)
                p = prefill_keys_of(idx, t, S, block)
                hs = slice(g * G, (g + 1) * G)
                dq, dk, dv = attend_row_backward(Q[b, t, hs], K[b, p, g], V[b, p, g],
                                                 dO[b, t, hs], scale)
                dQ[b, t, hs] = dq
                np.add.at(dK[b, :, g], p, dk)
                np.add.at(dV[b, :, g], p, dv)
    return dQ, dK, dV
