"""The softmax's own base-2 exponential (csrc/fastmath.cuh): a range reduction to
[-1/2, 1/2] and a cubic fitted for minimal relative error.

Host tests read the coefficients from the source and hold them to the minimax optimum,
computed here independently as a linear program, and to the stated 7.5e-5 bound, with
the device's fp32 FMA arithmetic emulated in float64.  The GPU test runs the device
code itself (msa_exp2_poly_eval) on a grid and compares it with exp2.
"""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "block_sparse_top_mean_b200", "csrc", "fastmath.cuh")
BOUND = 7.5e-5


def _coeffs():
    src = open(HDR).read()
    c = {k: float(v) for k, v in re.findall(r"constexpr float kExp2(C\d) = ([0-9.e+-]+)f;", src)}
    return [np.float32(c["C0"]), np.float32(c["C1"]), np.float32(c["C2"]), np.float32(c["C3"])]


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in float64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _cubic32(f):
    c0, c1, c2, c3 = _coeffs()
    q = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = _fma32(q, f, np.full_like(f, c1))
    return _fma32(q, f, np.full_like(f, c0))


def _poly_exp2_32(x):
    """Emulates poly_exp2x2 step by step in fp32 (range reduction, cubic, exponent add)."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), x)
    q = _cubic32(f)
    bits = q.view(np.int32) + (t.view(np.int32) << 23).astype(np.int32)
    return bits.astype(np.int32).view(np.float32)


def test_cubic_is_the_minimax_relative_fit():
    """A linear program finds the cubic with the smallest largest relative error on
    [-1/2, 1/2]; the shipped coefficients are within 0.2% of that optimum and inside
    the stated bound.  Catches a mistyped or truncated coefficient."""
    from scipy.optimize import linprog
    g = np.linspace(-0.5, 0.5, 4097)
    A = np.stack([g ** i / np.exp2(g) for i in range(4)], 1)
    one = np.ones((len(g), 1))
    r = linprog([0, 0, 0, 0, 1], A_ub=np.vstack([np.hstack([A, -one]), np.hstack([-A, -one])]),
                b_ub=np.concatenate([np.ones(len(g)), -np.ones(len(g))]),
                bounds=[(None, None)] * 5)
    assert r.status == 0
    opt = r.fun
    f = np.linspace(-0.5, 0.5, 200001)
    c0, c1, c2, c3 = (float(c) for c in _coeffs())
    err = np.abs((((c3 * f + c2) * f + c1) * f + c0) / np.exp2(f) - 1).max()
    assert 7.0e-5 < opt < 7.5e-5
    assert err <= opt * 1.002, (err, opt)
    assert err <= BOUND


def test_fp32_evaluation_meets_the_bound():
    """The whole 2^x in fp32 arithmetic, over the range the softmax uses (x <= 0 after
    the max is subtracted) and beyond, including the integer boundaries of the range
    reduction."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125.5, 8, 400000), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9) - 0.5, np.arange(-125, 9).astype(float),
                        np.linspace(-1, 1, 20001)]).astype(np.float32)
    y = _poly_exp2_32(x)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() <= BOUND, rel.max()
    # below -125.5 the result leaves the normal range: it stays in [0, 2^-125], an
    # absolute error below 2^-125 (nothing next to the softmax's largest term, 1)
    lo = np.concatenate([np.linspace(-140, -125.5, 100001), [-1e30, -200.0]]).astype(np.float32)
    yl = _poly_exp2_32(lo).astype(np.float64)
    assert np.all(yl >= 0) and np.all(yl <= 2.0 ** -125)
    assert np.abs(yl - np.exp2(lo.astype(np.float64))).max() < 2.0 ** -125


@pytest.mark.gpu
def test_device_exp2_against_exp2():
    """The device code (the same header the attention kernel includes) against exp2 on
    a grid: relative error <= 7.5e-5 for -125.5 <= x <= 8, at most 2^-125 below, and
    equal to the host emulation to within one fp32 ulp."""
    import block_sparse_top_mean_b200 as msa
    from block_sparse_top_mean_b200 import build
    build.build()
    rng = np.random.default_rng(1)
    xs = np.concatenate([np.linspace(-125.5, 8, 1_000_001), rng.uniform(-125.5, 8, 1_000_000),
                         np.arange(-125, 9) + 0.5, np.linspace(-140, -125.5, 1001)]
                        ).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y = msa.exp2_poly_eval(x)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    normal = x >= -125.5
    rel = (y.double()[normal] / ref[normal] - 1).abs().max().item()
    assert rel <= BOUND, rel
    assert (y.double()[~normal] - ref[~normal]).abs().max().item() < 2.0 ** -125
    emu = torch.from_numpy(_poly_exp2_32(xs)).cuda()
    ulp = (y.view(torch.int32).long() - emu.view(torch.int32).long()).abs().max().item()
    assert ulp <= 1, ulp
    # odd length: the last element has no partner lane
    y3 = msa.exp2_poly_eval(x[:3])
    assert torch.equal(y3, y[:3])
