"""Pins for the backward oracle (oracle/msa_backward.py): central differences of the
pinned forward oracle, dense causal attention differentiated by torch autograd (when every
past block is selected, and block-local when k = 1), and the closed form for constant
values."""
import numpy as np
import pytest
import torch

import oracle
from oracle.msa_backward import attend_row_backward, prefill_backward


def _inputs(seed, S, hq, hkv, d):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((1, S, hq, d))
    K = rng.standard_normal((1, S, hkv, d))
    V = rng.standard_normal((1, S, hkv, d))
    dO = rng.standard_normal((1, S, hq, d))
    return Q, K, V, dO


def _loss(Q, K, V, dO, block, topk, scale, kbar, fixed):
    rows = oracle.prefill_rows(Q, K, V, block, topk, scale, kbar=kbar, idx_override=fixed)
    G = Q.shape[2] // K.shape[2]
    return sum(float((dO[r.b, r.t, r.g * G:(r.g + 1) * G] * r.O).sum()) for r in rows)


@pytest.mark.parametrize("seed,S,block,topk", [(0, 40, 8, 3), (1, 37, 8, 2), (2, 24, 4, 8)])
def test_gradients_match_central_differences(seed, S, block, topk):
    hq, hkv, d = 4, 2, 6
    Q, K, V, dO = _inputs(seed, S, hq, hkv, d)
    scale = 0.4
    kbar = oracle.pool_keys(K, block)
    rows = oracle.prefill_rows(Q, K, V, block, topk, scale, kbar=kbar)
    fixed = {(r.b, r.t, r.g): r.idx for r in rows}          # hold the selection
    dQ, dK, dV = prefill_backward(Q, K, V, dO, block, topk, scale, kbar=kbar)
    rng = np.random.default_rng(100 + seed)
    h = 1e-6
    for X, dX in [(Q, dQ), (K, dK), (V, dV)]:
        for _ in range(12):
            c = tuple(int(rng.integers(0, n)) for n in X.shape)
            old = X[c]
            X[c] = old + h
            lp = _loss(Q, K, V, dO, block, topk, scale, kbar, fixed)
            X[c] = old - h
            lm = _loss(Q, K, V, dO, block, topk, scale, kbar, fixed)
            X[c] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - dX[c]) <= 1e-6 * max(1.0, abs(fd)), (c, fd, dX[c])


def _dense_grads(Q, K, V, dO, scale, mask):
    """torch autograd (fp64, CPU) of attention with a boolean mask [S, S] (True = kept)."""
    hq, hkv = Q.shape[2], K.shape[2]
    G = hq // hkv
    q = torch.tensor(Q[0].transpose(1, 0, 2), requires_grad=True)     # [hq, S, d]
    k = torch.tensor(K[0].transpose(1, 0, 2), requires_grad=True)     # [hkv, S, d]
    v = torch.tensor(V[0].transpose(1, 0, 2), requires_grad=True)
    kk = k.repeat_interleave(G, dim=0)
    vv = v.repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(
        q, kk, vv, attn_mask=torch.tensor(mask), scale=scale)
    (o * torch.tensor(dO[0].transpose(1, 0, 2))).sum().backward()
    back = lambda t: t.grad.numpy().transpose(1, 0, 2)[None]   # noqa: E731
    return back(q), back(k), back(v)


@pytest.mark.parametrize("S,block,hq,hkv", [(48, 8, 4, 2), (30, 8, 2, 1), (16, 16, 2, 2)])
def test_all_blocks_selected_equals_dense_causal_autograd(S, block, hq, hkv):
    d = 8
    Q, K, V, dO = _inputs(3, S, hq, hkv, d)
    nb = -(-S // block)
    mask = np.tril(np.ones((S, S), dtype=bool))
    got = prefill_backward(Q, K, V, dO, block, nb, 0.3)
    ref = _dense_grads(Q, K, V, dO, 0.3, mask)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_topk_one_equals_block_local_causal_autograd():
    S, block, hq, hkv, d = 40, 8, 4, 2, 8
    Q, K, V, dO = _inputs(4, S, hq, hkv, d)
    t = np.arange(S)
    mask = (t[:, None] >= t[None, :]) & (t[:, None] // block == t[None, :] // block)
    got = prefill_backward(Q, K, V, dO, block, 1, 0.5)
    ref = _dense_grads(Q, K, V, dO, 0.5, mask)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_constant_values_closed_form():
    """With every value vector equal to c the output is c whatever the weights, so dQ and
    dK vanish, and the weights of each (row, head) sum to one, so the dV rows of a group
    sum to the sum of that group's dO."""
    S, block, hq, hkv, d = 33, 8, 4, 2, 5
    Q, K, _, dO = _inputs(5, S, hq, hkv, d)
    c = np.random.default_rng(6).standard_normal(d)
    V = np.broadcast_to(c, (1, S, hkv, d)).copy()
    dQ, dK, dV = prefill_backward(Q, K, V, dO, block, 2, 0.7)
    assert np.abs(dQ).max() < 1e-12 and np.abs(dK).max() < 1e-12
    G = hq // hkv
    for g in range(hkv):
        np.testing.assert_allclose(dV[0, :, g].sum(axis=0),
                                   dO[0, :, g * G:(g + 1) * G].sum(axis=(0, 1)), atol=1e-12)


def test_row_backward_single_key():
    """One key: the weight is 1, so dq = dk = 0 and dv = sum of the heads' dO."""
    rng = np.random.default_rng(9)
    q, k, v, g = rng.standard_normal((3, 4)), rng.standard_normal((1, 4)), \
        rng.standard_normal((1, 4)), rng.standard_normal((3, 4))
    dq, dk, dv = attend_row_backward(q, k, v, g, 0.9)
    assert np.abs(dq).max() < 1e-15 and np.abs(dk).max() < 1e-15
    np.testing.assert_allclose(dv[0], g.sum(axis=0), atol=1e-15)
