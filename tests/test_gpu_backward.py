"""Backward of the causal sparse attention on the GPU vs the fp64 oracle
(oracle/msa_backward.py), through the C ABI.  The selection is an input of the backward:
both sides use the GPU forward's idx, held fixed, as the definition does."""
import numpy as np
import pytest
import torch

import msa_inputs as mi
import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


def _tol(ref):
    """Gradient tolerance: the forward's 2e-2 absolute bar for bf16 inputs, plus one bf16
    rounding (2^-9 relative) of the tensor's largest magnitude.  The gradients are sums
    over up to thousands of (row, key) terms whose P and dS factors are rounded to bf16
    before the tensor-core products, so their error grows with their magnitude; on these
    cases the observed errors are <= 1.8e-2 for magnitudes up to 12."""
    return 2e-2 + 2.0 ** -9 * float(np.abs(ref).max())


CASES = [
    mi.Workload("bwd_b128_g4", "prefill", 1, 3000, 8, 2, 128, 128, 6, "bf16"),
    mi.Workload("bwd_b256_g4", "prefill", 1, 2600, 16, 4, 128, 256, 4, "bf16"),
    mi.Workload("bwd_g1", "prefill", 1, 1500, 4, 4, 128, 128, 4, "bf16"),
    mi.Workload("bwd_g8_b2", "prefill", 2, 1100, 16, 2, 128, 128, 5, "bf16"),
    mi.Workload("bwd_planted", "prefill", 1, 4096, 8, 2, 128, 128, 8, "bf16",
                planted_frac=0.02, planted_shift=3.0),
]


def _run(msa, w, seed=0, ws=None):
    q, k, v = mi.prefill_inputs(w, device="cuda", seed=seed)
    o, lse, idx = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    dout = mi.normal(q.shape, seed + 7, mi.STREAM_DECODE_Q, "cuda", torch.bfloat16)
    dq, dk, dv = msa.sparse_attn_bwd(q, k, v, o, lse, dout, idx, w.block, w.scale, ws=ws)
    torch.cuda.synchronize()
    return q, k, v, dout, idx, (dq, dk, dv)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_vs_oracle(msa, w):
    q, k, v, dout, idx, grads = _run(msa, w)
    Q, K, V, dO = (x.float().cpu().numpy() for x in (q, k, v, dout))
    gi = idx.cpu().numpy()
    fixed = {(b, t, g): [int(x) for x in gi[b, g, t]]
             for b in range(w.batch) for t in range(w.seq) for g in range(w.hkv)}
    ref = oracle.prefill_backward(Q, K, V, dO, w.block, w.topk, w.scale, idx_override=fixed)
    for name, got, want in zip(("dq", "dk", "dv"), grads, ref):
        err = float(np.abs(got.double().cpu().numpy() - want).max())
        print(f"{w.name} {name}: max |err| {err:.3e}, max |ref| {float(np.abs(want).max()):.3e}")
        assert err <= _tol(want), (name, err, float(np.abs(want).max()))


def test_backward_is_deterministic_and_slab_independent(msa):
    w = CASES[0].with_(seq=6000)
    _, _, _, _, _, a = _run(msa, w)
    _, _, _, _, _, b = _run(msa, w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # the smallest workspace walks the sequence in 2048-token slabs: dq is unchanged, and
    # dk, dv only differ by the fp32 order of the per-slab sums
    p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block, topk=w.topk,
                   scale=w.scale, dtype=torch.bfloat16)
    ws = msa.workspace(p, msa.OP_SPARSE_ATTN_BWD_MIN)
    _, _, _, _, _, c = _run(msa, w, ws=ws)
    assert torch.equal(a[0], c[0])
    for x, y in zip(a[1:], c[1:]):
        assert (x - y).abs().max().item() <= 1e-4 * max(1.0, x.abs().max().item())
