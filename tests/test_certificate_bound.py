"""The certificate of the encoded-bank decode selection, checked on the host in float64.

The selection scores every block with the hi plane only, a_j = Khi_j . (Qhi + Qlo), keeps
each row's 64 best as candidates, rescores them exactly (the three-term split score
s_j = Khi_j . Qhi + Khi_j . Qlo + Klo_j . Qhi) and accepts the row when the k-th best exact
score among the candidates lies strictly above amin + eps, amin being the 64th candidate's
a and eps = (max ||Klo_j|| + 2^-9 max ||Khi_j||) ||Q|| * 1.01 (the encoded image stores the
two maxima).  These tests hold that reasoning to the arithmetic:
  * |s_j - a_j| <= eps for every block, also when both sides are summed in float32 in
    the order the tensor cores use (16-term products, then accumulation);
  * whenever a row is accepted, the candidates' top k is the bank's exact top k, on
    random banks and on banks built with near-ties at the cut;
  * near-ties wider than eps make rows fail (so the exact rescan decides).
No CUDA: the GPU's bitwise agreement with the natural-layout scan is tested separately.
"""
import numpy as np
import pytest
import torch

K_CAND = 64


def _split(x):
    """x (float32) -> (hi, lo) bf16 values as float64: hi = bf16(x), lo = bf16(x - hi)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    hi = t.to(torch.bfloat16).float()
    lo = (t - hi).to(torch.bfloat16).float()
    return hi.double().numpy(), lo.double().numpy()


def _bank(rng, nb, d=128, spread=1 / 8):
    kbar = (rng.standard_normal((nb, d)) * spread).astype(np.float32)
    return _split(kbar)


def _query(rng, d=128, heads=4):
    q = torch.from_numpy(rng.standard_normal((heads, d)).astype(np.float32)).to(torch.bfloat16)
    qs = q.float().sum(dim=0).numpy()                    # fp32 group sum of the bf16 heads
    qhi, qlo = _split(qs)
    return qs.astype(np.float64), qhi, qlo


def _eps(khi, klo, qs):
    L = np.linalg.norm(klo, axis=1).max()
    H = np.linalg.norm(khi, axis=1).max()
    return (L + 2.0 ** -9 * H) * np.linalg.norm(qs) * 1.01


def _fp32_dot(a, b):
    """Blocked float32 accumulation: 16-term products summed per k-step, steps in order."""
    acc = np.zeros(a.shape[0], dtype=np.float32)
    for k0 in range(0, a.shape[1], 16):
        part = (a[:, k0:k0 + 16] * b[k0:k0 + 16]).sum(axis=1).astype(np.float32)
        acc = (acc + part).astype(np.float32)
    return acc.astype(np.float64)


def _certify(khi, klo, qs, qhi, qlo, k):
    """(accepted, candidates' top k, exact top k) for one row, keys (score desc, id asc)."""
    a = khi @ (qhi + qlo)
    s = khi @ qhi + khi @ qlo + klo @ qhi
    nb = a.shape[0]
    order_a = sorted(range(nb), key=lambda j: (-a[j], j))
    cand = order_a[:K_CAND]
    amin = a[cand[-1]] if nb > K_CAND else -np.inf
    top_c = sorted(cand, key=lambda j: (-s[j], j))[:k]
    top_all = sorted(range(nb), key=lambda j: (-s[j], j))[:k]
    sk = s[top_c[-1]]
    accepted = amin == -np.inf or sk > amin + _eps(khi, klo, qs)
    return accepted, top_c, top_all


def test_eps_bounds_the_dropped_term():
    rng = np.random.default_rng(11)
    for spread in (1 / 8, 1.0, 37.0):
        khi, klo = _bank(rng, 4096, spread=spread)
        for _ in range(8):
            qs, qhi, qlo = _query(rng)
            a = khi @ (qhi + qlo)
            s = khi @ qhi + khi @ qlo + klo @ qhi
            assert np.abs(s - a).max() <= _eps(khi, klo, qs)


def test_eps_bounds_float32_accumulation():
    rng = np.random.default_rng(12)
    khi, klo = _bank(rng, 2048)
    for _ in range(4):
        qs, qhi, qlo = _query(rng)
        a32 = _fp32_dot(khi, qhi) + _fp32_dot(khi, qlo)   # the hi-plane scan's two columns
        s32 = _fp32_dot(np.concatenate([khi, khi, klo], axis=1),
                        np.concatenate([qhi, qlo, qhi]))
        assert np.abs(s32 - a32).max() <= _eps(khi, klo, qs)


@pytest.mark.parametrize("seed", range(6))
def test_accepted_rows_are_exact(seed):
    rng = np.random.default_rng(100 + seed)
    khi, klo = _bank(rng, 3000)
    n_acc = 0
    for _ in range(6):
        qs, qhi, qlo = _query(rng)
        ok, top_c, top_all = _certify(khi, klo, qs, qhi, qlo, 32)
        if ok:
            n_acc += 1
            assert top_c == top_all
    assert n_acc > 0                                      # random banks certify


def test_near_ties_at_the_cut_fail_or_stay_exact():
    # 100 blocks share one hi row along the query and differ only in lo: the hi-plane
    # scores tie across the cut, the lo terms (below eps) decide the exact order
    rng = np.random.default_rng(7)
    khi, klo = _bank(rng, 2000)
    qs, qhi, qlo = _query(rng)
    u = qs / np.linalg.norm(qs)
    hi_row = torch.from_numpy((3.0 * np.linalg.norm(khi, axis=1).mean() * u)
                              .astype(np.float32)).to(torch.bfloat16).double().numpy()
    khi[500:600] = hi_row
    klo[500:600] = (rng.standard_normal((100, khi.shape[1])) * 1e-3).astype(np.float64)
    ok, top_c, top_all = _certify(khi, klo, qs, qhi, qlo, 32)
    assert not ok                                         # the bound cannot separate them
    assert all(500 <= j < 600 for j in top_all)


def test_small_banks_are_all_candidates():
    rng = np.random.default_rng(3)
    khi, klo = _bank(rng, 40)                             # fewer blocks than candidates
    qs, qhi, qlo = _query(rng)
    ok, top_c, top_all = _certify(khi, klo, qs, qhi, qlo, 32)
    assert ok and top_c == top_all
