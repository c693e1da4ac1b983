"""The allocation-free decode entry point (msa_decode_fwd_static).

Some callers cannot allocate device memory at decode time: a runtime that reserves all
device memory up front and forbids allocation on its hot path, or a plug-in whose host
framework owns every allocation and hands it only the step's tensors.  They use a fixed
device scratch inside the library instead of a workspace.  This checks, through the C
ABI, that two calls in a row give exactly the selection and outputs of msa_decode_fwd
with a caller workspace (the same kernels on the same inputs are bitwise
deterministic).  It sits in its own file that pytest collects last, and it holds
whether it runs alone in a fresh process or after the other tests.
"""
import ctypes

import pytest
import torch

import msa_inputs as mi

pytestmark = pytest.mark.gpu


def test_static_scratch_decode_matches_workspace_decode():
    import block_sparse_top_mean_b200 as msa
    from block_sparse_top_mean_b200 import _lib, build
    build.build()
    lib = _lib.load()
    w = mi.Workload("decode_static_check", "decode", 1, 60_000, 32, 8, 128, 64, 32, "bf16",
                    n_query=16)
    _, kb, vb = mi.decode_inputs(w, device="cuda")
    kbar, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block, topk=w.topk,
                   scale=w.scale, dtype=torch.bfloat16)
    assert lib.msa_workspace_bytes(ctypes.byref(p), _lib.OP_DECODE, w.n_query) <= 32 << 20
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    # two calls in a row with different queries: the fp32 scan, then the tensor-core scan
    for call, (seed, split) in enumerate(((11, False), (12, True))):
        q = mi.normal((w.n_query, w.hq, w.d), seed, mi.STREAM_DECODE_Q, "cuda", torch.bfloat16)
        hi, lo = (khi, klo) if split else (None, None)
        o_ref, lse_ref, idx_ref = msa.decode_fwd(q, kbar, kb, vb, w.block, w.topk, w.scale,
                                                 kbar_hi=hi, kbar_lo=lo)
        o = torch.empty_like(q)
        lse = torch.empty(w.n_query, w.hq, dtype=torch.float32, device="cuda")
        idx = torch.empty(w.n_query, w.hkv, w.topk, dtype=torch.int32, device="cuda")
        Pn = lambda t: None if t is None else P(t)  # noqa: E731
        torch.cuda.synchronize()
        held = torch.cuda.memory_allocated()
        st = lib.msa_decode_fwd_static(ctypes.byref(p), w.n_query, P(q), P(kbar), Pn(hi), Pn(lo),
                                       P(kb), P(vb), P(idx), P(o), P(lse), stream)
        assert st == _lib.MSA_OK, (call, st)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == held, call   # nothing from torch's allocator
        assert torch.equal(idx, idx_ref), call
        assert torch.equal(o, o_ref), call
        assert torch.equal(lse, lse_ref), call
        bits = ctypes.c_int32(-1)
        assert lib.msa_decode_static_read_error(ctypes.byref(bits), stream) == _lib.MSA_OK
        assert bits.value == 0, call


def test_static_scratch_rejects_sizes_beyond_the_limit():
    from block_sparse_top_mean_b200 import _lib
    import block_sparse_top_mean_b200 as msa
    lib = _lib.load()
    p = msa.params(batch=1, seq=10_000_000, hq=32, hkv=8, d=128, block=64, topk=32, scale=0.088,
                   dtype=torch.bfloat16)
    n_query = 4096                                   # needs far more than 32 MiB
    assert lib.msa_workspace_bytes(ctypes.byref(p), _lib.OP_DECODE, n_query) > 32 << 20
    fake = ctypes.c_void_p(4096)
    st = lib.msa_decode_fwd_static(ctypes.byref(p), n_query, fake, fake, None, None, fake, fake,
                                   fake, fake, None, None)
    assert st == _lib.MSA_ERR_WORKSPACE
