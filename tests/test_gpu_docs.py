"""Document-wise RoPE and packed-document prefill on the GPU vs the fp64 oracle
(oracle/msa_docs.py), through the C ABI."""
import numpy as np
import pytest
import torch

import msa_inputs as mi
import oracle
from parity_util import check_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


def _packed(T, hq, hkv, d, dtype, seed):
    q = mi.normal((T, hq, d), seed, mi.STREAM_Q, "cuda", dtype)
    k = mi.normal((T, hkv, d), seed, mi.STREAM_K, "cuda", dtype)
    v = mi.normal((T, hkv, d), seed, mi.STREAM_V, "cuda", dtype)
    return q, k, v


def _check_rope(x_in, x_out, cu, base):
    """|gpu - oracle| <= one rounding to the output dtype plus fp32 arithmetic."""
    ref = oracle.rope_docwise(x_in.float().cpu().numpy(), cu, base)
    got = x_out.double().cpu().numpy()
    d = ref.shape[-1]
    x = x_in.double().cpu().numpy()
    pair = np.abs(x) + np.abs(np.roll(x, d // 2, axis=-1))
    u = 2.0 ** -8 if x_out.dtype == torch.bfloat16 else 2.0 ** -24
    bound = u * np.abs(ref) + 1e-6 * pair + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), float((err / bound).max())
    return float(err.max())


@pytest.mark.parametrize("dtype,d,hq,hkv,cu,base", [
    (torch.bfloat16, 128, 8, 2, [0, 700, 700, 3000, 5123], 10000.0),
    (torch.float32, 64, 4, 4, [0, 1, 2, 1000, 1029], 500.0),
    (torch.bfloat16, 128, 32, 8, [0, 4096], 1_000_000.0),
    (torch.float32, 128, 2, 1, [0, 17, 300_017], 10000.0),       # positions up to 300K
])
def test_rope_docwise_vs_oracle(msa, dtype, d, hq, hkv, cu, base):
    T = cu[-1]
    q, k, _ = _packed(T, hq, hkv, d, dtype, 3)
    q0, k0 = q.clone(), k.clone()
    cu_d = torch.tensor(cu, dtype=torch.int32, device="cuda")
    msa.rope_docwise(q, k, cu_d, base)
    torch.cuda.synchronize()
    _check_rope(q0, q, cu, base)
    _check_rope(k0, k, cu, base)
    # the first token of every non-empty document keeps its values (position 0)
    starts = [a for a, b in zip(cu[:-1], cu[1:]) if b > a]
    assert torch.equal(q[starts], q0[starts]) and torch.equal(k[starts], k0[starts])


VARLEN = [
    ("bf16_tc", torch.bfloat16, 128, 8, 2, 128, 6, [0, 1000, 1000, 3500, 3600, 6000]),
    ("bf16_b256", torch.bfloat16, 128, 16, 4, 256, 4, [0, 2048, 2300, 4100]),
    ("f32_simt", torch.float32, 64, 4, 2, 64, 4, [0, 130, 131, 900, 1500]),
]


@pytest.mark.parametrize("case", VARLEN, ids=[c[0] for c in VARLEN])
def test_rope_then_varlen_prefill_vs_oracle(msa, case):
    _, dtype, d, hq, hkv, block, topk, cu = case
    T = cu[-1]
    scale = d ** -0.5
    q, k, v = _packed(T, hq, hkv, d, dtype, 5)
    msa.rope_docwise(q, k, torch.tensor(cu, dtype=torch.int32, device="cuda"), 10000.0)
    o, lse, idx = msa.prefill_varlen_fwd(q, k, v, cu, block, topk, scale)
    torch.cuda.synchronize()
    # each document against the oracle's prefill of that document alone, read from the
    # very (rotated) tensors the kernels consumed
    for a, b in zip(cu[:-1], cu[1:]):
        L = b - a
        if L == 0:
            continue
        idx_d = idx[a * hkv * topk:b * hkv * topk].view(1, hkv, L, topk)
        lse_d = lse[a * hq:b * hq].view(1, hq, L)
        check_prefill(q[a:b][None], k[a:b][None], v[a:b][None], block, topk, scale, idx_d,
                      o[a:b][None], lse_d)
    # the packed oracle on a few rows: global token numbering and document-local blocks
    Qh, Kh, Vh = (x.float().cpu().numpy() for x in (q, k, v))
    rows = [0, cu[1] - 1, cu[2], T - 1]
    ref = oracle.prefill_varlen_rows(Qh, Kh, Vh, cu, block, topk, scale, rows=rows)
    G = hq // hkv
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    for t, r in ref:
        doc = max(i for i in range(len(cu) - 1) if cu[i] <= t and cu[i + 1] > cu[i])
        a, L = cu[doc], cu[doc + 1] - cu[doc]
        if r.gap > 1e-3:
            sel = idx[a * hkv * topk:].view(-1)[(r.g * L + (t - a)) * topk:][:topk]
            assert sel.tolist() == r.idx, (t, r.g)
            err = (o[t, r.g * G:(r.g + 1) * G].double().cpu().numpy() - r.O).max()
            assert abs(err) <= tol


def test_varlen_rejects_bad_boundaries(msa):
    from block_sparse_top_mean_b200 import _lib
    q, k, v = _packed(100, 2, 1, 64, torch.float32, 1)
    for cu in ([0, 50], [1, 100], [0, 60, 40, 100]):
        with pytest.raises(_lib.MsaError):
            msa.prefill_varlen_fwd(q, k, v, cu, 64, 2, ws=torch.zeros(1 << 20, dtype=torch.uint8,
                                                                        device="cuda"))
