"""Document-wise rotary positions and packed variable-length documents (fp64 oracle).
TEST INFRASTRUCTURE ONLY: tests, the smoke check and the bench's CPU legs use it; the
CUDA library never does.

Source: "100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it), section "Das
Gehirn mit zwei Geschwindigkeiten": EverMind's MSA uses a document-wise variant of the
rotary position embedding (RoPE); the position counter restarts at zero at the start of
every document, so each text starts at position 0 however many documents precede it in
memory.  The same section describes each document being processed on its own (its
routing keys and content are produced per document).

The page names RoPE but prints no formula.  Readings taken here:
  * RoPE is the usual rotary embedding of the query and key heads: dimensions i and
    i + d/2 (i < d/2) form a pair that is rotated by the angle pos * theta_i, with
    theta_i = base^(-2i/d); the base is a parameter (the backbone the page names uses a
    large base; 10000 is the classic one).  The pairing (first half with second half)
    is the common "rotate half" layout.
  * pos = t - start of the document that holds token t.
  * The rotated q and k feed every step of the method unchanged (pooling, scoring,
    selection and attention all see rotated keys); values are not rotated.
  * Packed documents ("varlen"): documents are concatenated along the token axis and
    each is its own causal sequence: blocks restart at the document start, selection and
    attention never cross a document boundary.
"""
from __future__ import annotations

import numpy as np

from .msa_oracle import prefill_rows

__all__ = ["rope_angles", "rope_docwise", "doc_positions", "prefill_varlen_rows"]


def doc_positions(cu_seqlens) -> np.ndarray:
    """Position of every packed token inside its own document (0 at each start)."""
    cu = [int(x) for x in cu_seqlens]
    pos = np.zeros(cu[-1], dtype=np.int64)
    for a, b in zip(cu[:-1], cu[1:]):
        pos[a:b] = np.arange(b - a)
    return pos


def rope_angles(pos: np.ndarray, d: int, base: float) -> np.ndarray:
    """[n, d/2] rotation angles pos * base^(-2i/d) in fp64."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    return pos.astype(np.float64)[:, None] * theta[None, :]


def rope_docwise(x: np.ndarray, cu_seqlens, base: float) -> np.ndarray:
    """Rotates x [T, h, d] (packed tokens) by each token's in-document position.

    For pair (i, i + d/2) with angle a: (x_i, x_{i+d/2}) ->
    (x_i cos a - x_{i+d/2} sin a, x_{i+d/2} cos a + x_i sin a).  fp64 result."""
    T, h, d = x.shape
    half = d // 2
    ang = rope_angles(doc_positions(cu_seqlens), d, base)        # [T, d/2]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x = x.astype(np.float64)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def prefill_varlen_rows(Q, K, V, cu_seqlens, block: int, topk: int, scale: float, rows=None):
    """The causal prefill of each packed document on its own.

    Q [T, hq, d], K/V [T, hkv, d] (exact input values, already rotated if the caller
    applies RoPE); cu_seqlens the document starts and the end (T).  rows: packed token
    indices to compute (all when None).  Returns a list of (t, PrefillRow) where the
    row's own t and idx are relative to its document (block ids count from the
    document's first block)."""
    cu = [int(x) for x in cu_seqlens]
    want = None if rows is None else set(int(t) for t in rows)
    out = []
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        local = None if want is None else [(0, t - a) for t in range(a, b) if t in want]
        if local is not None and not local:
            continue
        res = prefill_rows(Q[None, a:b], K[None, a:b], V[None, a:b], block, topk, scale,
                           rows=local)
        out.extend((a + r.t, r) for r in res)
    return out
