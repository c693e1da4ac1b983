"""Pins of the document-wise RoPE and packed-document (varlen) oracle (oracle/msa_docs.py)
against facts from outside it: complex multiplication (numpy), closed forms, the
relative-position property that defines a rotary embedding, and the batched prefill
oracle for documents of equal length."""
import math

import numpy as np
import pytest

import oracle
from oracle import msa_docs


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def test_rope_equals_complex_rotation():
    """Pair (i, i + d/2) as the complex number x_i + 1j x_{i+d/2}, multiplied by
    exp(1j * pos * base^(-2i/d)) (numpy complex arithmetic)."""
    T, h, d, base = 37, 3, 16, 500.0
    x = _rand((T, h, d), 1)
    cu = [0, 10, 10, 37]                        # an empty document in the middle
    got = msa_docs.rope_docwise(x, cu, base)
    pos = np.concatenate([np.arange(10), np.arange(27)])
    z = x[..., :d // 2].astype(np.float64) + 1j * x[..., d // 2:].astype(np.float64)
    w = np.exp(1j * pos[:, None, None] * base ** (-np.arange(d // 2) * 2.0 / d)[None, None, :])
    ref = z * w
    np.testing.assert_allclose(got, np.concatenate([ref.real, ref.imag], -1), atol=1e-12)


def test_rope_closed_form_d4():
    """d = 4, base 10000: theta = (1, 1/100); position 3 rotates pair 0 by 3 rad and
    pair 1 by 0.03 rad."""
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]] * 4, np.float32)      # positions 0..3
    got = msa_docs.rope_docwise(x, [0, 4], 10000.0)[3, 0]
    a0, a1 = 3.0, 0.03
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
    np.testing.assert_allclose(got, want, atol=1e-14)
    np.testing.assert_array_equal(msa_docs.rope_docwise(x, [0, 4], 10000.0)[0, 0], x[0, 0])


def test_positions_restart_at_every_document():
    """Identical documents placed anywhere rotate identically; the first token of each
    document is unchanged (position 0)."""
    doc = _rand((9, 2, 8), 2)
    x = np.concatenate([_rand((5, 2, 8), 3), doc, doc, _rand((4, 2, 8), 4)])
    cu = [0, 5, 14, 23, 27]
    r = msa_docs.rope_docwise(x, cu, 10000.0)
    np.testing.assert_array_equal(r[5:14], r[14:23])
    np.testing.assert_allclose(r[5:14], msa_docs.rope_docwise(doc, [0, 9], 10000.0), atol=0)
    for a in cu[:-1]:
        np.testing.assert_array_equal(r[a], x[a].astype(np.float64))
    assert list(msa_docs.doc_positions(cu)) == list(range(5)) + list(range(9)) * 2 + list(range(4))


def test_rope_relative_position_and_norm():
    """What makes an embedding rotary: rope(q, m) . rope(k, n) depends on m - n only, and
    each pair keeps its length."""
    d = 32
    q, k = _rand((1, 1, d), 5), _rand((1, 1, d), 6)
    L = 60
    Qs = np.repeat(q, L, axis=0)
    Ks = np.repeat(k, L, axis=0)
    rq = msa_docs.rope_docwise(Qs, [0, L], 1000.0)[:, 0]
    rk = msa_docs.rope_docwise(Ks, [0, L], 1000.0)[:, 0]
    for m, n, s in [(10, 3, 17), (40, 40, 5), (2, 30, 11)]:
        assert abs(rq[m] @ rk[n] - rq[m + s] @ rk[n + s]) < 1e-12
    half = d // 2
    nrm = np.hypot(rq[:, :half], rq[:, half:])
    np.testing.assert_allclose(nrm, np.broadcast_to(np.hypot(q[0, 0, :half], q[0, 0, half:]),
                                                    nrm.shape), atol=1e-12)


def test_varlen_single_document_is_the_plain_prefill():
    S, hq, hkv, d, block, topk = 200, 4, 2, 8, 16, 3
    Q, K, V = _rand((S, hq, d), 7), _rand((S, hkv, d), 8), _rand((S, hkv, d), 9)
    got = msa_docs.prefill_varlen_rows(Q, K, V, [0, S], block, topk, 0.4)
    ref = oracle.prefill_rows(Q[None], K[None], V[None], block, topk, 0.4)
    assert len(got) == len(ref)
    for (t, a), b in zip(got, ref):
        assert t == b.t and a.idx == b.idx
        np.testing.assert_array_equal(a.O, b.O)


def test_varlen_equal_lengths_equal_the_batch():
    """Documents of equal length are the batch dimension of the plain prefill."""
    n, L, hq, hkv, d, block, topk = 3, 70, 2, 1, 8, 16, 2
    Q, K, V = _rand((n * L, hq, d), 10), _rand((n * L, hkv, d), 11), _rand((n * L, hkv, d), 12)
    got = dict(msa_docs.prefill_varlen_rows(Q, K, V, [0, L, 2 * L, 3 * L], block, topk, 0.3))
    ref = oracle.prefill_rows(Q.reshape(n, L, hq, d), K.reshape(n, L, hkv, d),
                              V.reshape(n, L, hkv, d), block, topk, 0.3)
    for r in ref:
        g = [x for (t, x) in msa_docs.prefill_varlen_rows(
            Q, K, V, [0, L, 2 * L, 3 * L], block, topk, 0.3, rows=[r.b * L + r.t]) if x.g == r.g]
        assert g[0].idx == r.idx
        np.testing.assert_array_equal(g[0].O, r.O)
    assert len(got) == n * L


def test_varlen_documents_do_not_see_each_other():
    """Changing a later document's keys and values changes nothing in an earlier one, and
    a document's blocks start at its first token (its first token sees only itself)."""
    hq, hkv, d, block, topk = 2, 1, 8, 8, 4
    cu = [0, 45, 45, 101, 130]
    T = cu[-1]
    Q, K, V = _rand((T, hq, d), 13), _rand((T, hkv, d), 14), _rand((T, hkv, d), 15)
    a = dict(msa_docs.prefill_varlen_rows(Q, K, V, cu, block, topk, 0.5))
    K2, V2 = K.copy(), V.copy()
    K2[101:] += 3.0
    V2[101:] -= 2.0
    b = dict(msa_docs.prefill_varlen_rows(Q, K2, V2, cu, block, topk, 0.5))
    for t in range(101):
        np.testing.assert_array_equal(a[t].O, b[t].O)
    r = a[45]                                     # first token of the second document
    assert r.idx == [0, -1, -1, -1]
    np.testing.assert_allclose(r.O, np.repeat(V[45:46, 0].astype(np.float64), hq, 0), atol=1e-15)
