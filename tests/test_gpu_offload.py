"""Decode with the bank's K/V in pinned host memory (msa_decode_fwd_offload) vs the same
decode with everything in HBM, and vs the fp64 oracle, through the C ABI."""
import ctypes

import pytest
import torch

import msa_inputs as mi
from parity_util import check_decode, pool_keys_chunked

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


@pytest.mark.parametrize("S,block,topk,nq", [(200_000, 64, 32, 16), (256_000, 128, 16, 70),
                                             (6_400, 64, 32, 3)])
def test_offload_equals_hbm_decode(msa, S, block, topk, nq):
    w = mi.Workload("off", "decode", 1, S, 32, 8, 128, block, topk, "bf16", n_query=nq)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=9)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, block)
    o_ref, lse_ref, idx_ref = msa.decode_fwd_tiled(q, bt, kt, vt, S, w.hkv, block, topk, w.scale)
    kt_h, vt_h = kt.cpu().pin_memory(), vt.cpu().pin_memory()
    for call in range(2):                    # the staging scratch is reused: call twice
        o, lse, idx = msa.decode_fwd_offload(q, bt, kt_h, vt_h, S, w.hkv, block, topk, w.scale)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref), call
        assert torch.equal(o, o_ref), call
        assert torch.equal(lse, lse_ref), call
    kbar_np = pool_keys_chunked(kb[None], block)[0]
    check_decode(q, kbar_np, kb, vb, block, topk, w.scale, idx, o, lse, queries=range(min(nq, 8)))


def test_offload_rejects_pageable_memory_and_ragged_banks(msa):
    from block_sparse_top_mean_b200 import _lib
    w = mi.Workload("off", "decode", 1, 6_400, 32, 8, 128, 64, 32, "bf16", n_query=2)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=1)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], 64, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, 64)
    kt_pageable, vt_pageable = kt.cpu(), vt.cpu()
    with pytest.raises(ValueError):
        msa.decode_fwd_offload(q, bt, kt_pageable, vt_pageable, w.seq, w.hkv, 64, 32)
    lib = _lib.load()
    p = msa.params(batch=1, seq=w.seq, hq=32, hkv=8, d=128, block=64, topk=32, scale=w.scale,
                   dtype=torch.bfloat16)
    ws = msa.workspace(p, _lib.OP_DECODE_OFFLOAD, 2)
    out = [torch.empty(2, 8, 32, dtype=torch.int32, device="cuda"), torch.empty_like(q)]
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = lib.msa_decode_fwd_offload(ctypes.byref(p), 2, P(q), P(bt), P(kt_pageable),
                                    P(vt_pageable), P(out[0]), P(out[1]), None, P(ws),
                                    ws.numel(), None)
    assert st == _lib.MSA_ERR_INVALID_ARG
    p.seq = w.seq - 10                                 # not a whole number of blocks
    st = lib.msa_decode_fwd_offload(ctypes.byref(p), 2, P(q), P(bt), P(kt), P(vt), P(out[0]),
                                    P(out[1]), None, P(ws), ws.numel(), None)
    assert st == _lib.MSA_ERR_UNSUPPORTED


def test_offload_of_a_10m_token_bank(msa):
    # a bank long enough for the certified hi-plane selection, its K/V in host memory
    w = mi.Workload("off_10m", "decode", 1, 10_000_000, 4, 1, 128, 64, 32, "bf16", n_query=8)
    q, kb, vb = mi.decode_inputs(w, device="cuda", seed=4)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    o_ref, lse_ref, idx_ref = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk,
                                                   w.scale)
    kt_h, vt_h = kt.cpu().pin_memory(), vt.cpu().pin_memory()
    del kt, vt
    o, lse, idx = msa.decode_fwd_offload(q, bt, kt_h, vt_h, w.seq, w.hkv, w.block, w.topk,
                                         w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref)
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
