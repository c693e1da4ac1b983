"""B200 (sm_100a) block-sparse top-k attention: pool -> score -> top-k -> sparse attention.

Thin PyTorch-facing binding of the C ABI in include/msa.h.  These functions only
marshal arguments (shapes, pointers, the current CUDA stream) and allocate outputs
and workspaces with torch; every step of the computation runs in the library's CUDA
kernels.  There is no CPU path: tensors must be CUDA tensors and the library must be
built (`python -m block_sparse_top_mean_b200.build`).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (  # noqa: F401
    MsaError, MsaParams, OP_DECODE, OP_PREFILL, OP_SPARSE_ATTN, OP_TOPK_SELECT,
    OP_SPARSE_ATTN_MIN, OP_PREFILL_MIN, OP_DECODE_OFFLOAD, OP_SPARSE_ATTN_BWD,
    OP_SPARSE_ATTN_BWD_MIN,
    DEVERR_IDX_RANGE, DEVERR_TIMEOUT, MSA_F32, MSA_BF16,
)

__all__ = [
    "params", "workspace", "pool_keys", "block_scores", "topk_select", "sparse_attn_fwd",
    "prefill_fwd", "decode_fwd", "decode_fwd_static", "encode_bank", "decode_fwd_tiled",
    "decode_select_tiled", "decode_attn_tiled", "attn_slab_tokens",
    "read_device_error",
    "clear_device_error", "version", "exp2_poly_eval", "rope_docwise", "prefill_varlen_fwd",
    "decode_select_shard", "decode_merge_shards", "decode_combine_shards", "decode_fwd_offload",
    "sparse_attn_bwd",
    "MsaError", "MsaParams",
]

_DT = {torch.float32: MSA_F32, torch.bfloat16: MSA_BF16}


def version() -> str:
    return _lib.load().msa_version().decode()


def params(*, batch, seq, hq, hkv, d, block, topk, scale, dtype) -> MsaParams:
    dt = _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return MsaParams(int(batch), int(seq), int(hq), int(hkv), int(d), int(block), int(topk),
                     float(scale), dt)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("block_sparse_top_mean_b200 takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def workspace(p: MsaParams, op: int, n_query: int = 0, device="cuda") -> torch.Tensor:
    """A workspace for `op` (uint8 CUDA tensor, 256-byte aligned by the caching
    allocator), with the device error word cleared."""
    n = _lib.load().msa_workspace_bytes(ctypes.byref(p), op, n_query)
    if n == 0:
        raise MsaError("msa_workspace_bytes", _lib.MSA_ERR_INVALID_ARG, "invalid shapes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def attn_slab_tokens(p: MsaParams, op: int, ws_bytes: int) -> int:
    """Tokens per slab the prefill attention walks with ws_bytes of workspace for `op`
    (OP_SPARSE_ATTN or OP_PREFILL); p.seq means one pass, 0 means too small."""
    n = _lib.load().msa_attn_slab_tokens(ctypes.byref(p), op, ws_bytes)
    if n < 0:
        raise MsaError("msa_attn_slab_tokens", _lib.MSA_ERR_INVALID_ARG, "invalid shapes or op")
    return n


def _prefill_params(q, k, block, topk, scale):
    b, S, hq, d = q.shape
    hkv = k.shape[2]
    return params(batch=b, seq=S, hq=hq, hkv=hkv, d=d, block=block, topk=topk,
                  scale=scale if scale is not None else d ** -0.5, dtype=q.dtype)


def pool_keys(k: torch.Tensor, block: int, split: bool = False):
    """k [b, S, hkv, d] -> kbar fp32 [b, nb, hkv, d] (and bf16 hi/lo planes if split)."""
    b, S, hkv, d = k.shape
    p = params(batch=b, seq=S, hq=hkv, hkv=hkv, d=d, block=block, topk=1, scale=1.0,
               dtype=k.dtype)
    nb = -(-S // block)
    kbar = torch.empty(b, nb, hkv, d, dtype=torch.float32, device=k.device)
    hi = lo = None
    if split:
        hi = torch.empty(b, nb, hkv, d, dtype=torch.bfloat16, device=k.device)
        lo = torch.empty_like(hi)
    _lib.check("msa_pool_keys", _lib.load().msa_pool_keys(
        ctypes.byref(p), _ptr(k), _ptr(kbar), _ptr(hi), _ptr(lo), _stream(k.device)))
    return (kbar, hi, lo) if split else kbar


def block_scores(q: torch.Tensor, kbar: torch.Tensor, block: int, hkv: int) -> torch.Tensor:
    """Materialised causal block scores [b, hkv, S, nb] (small shapes only)."""
    b, S, hq, d = q.shape
    p = params(batch=b, seq=S, hq=hq, hkv=hkv, d=d, block=block, topk=1, scale=1.0,
               dtype=q.dtype)
    nb = -(-S // block)
    out = torch.empty(b, hkv, S, nb, dtype=torch.float32, device=q.device)
    _lib.check("msa_block_scores", _lib.load().msa_block_scores(
        ctypes.byref(p), _ptr(q), _ptr(kbar), _ptr(out), _stream(q.device)))
    return out


def topk_select(q, kbar, block: int, topk: int, hkv: int, kbar_hi=None, kbar_lo=None, ws=None):
    """Causal selection idx [b, hkv, S, topk] (int32, ascending, -1 padded)."""
    b, S, hq, d = q.shape
    p = params(batch=b, seq=S, hq=hq, hkv=hkv, d=d, block=block, topk=topk, scale=1.0,
               dtype=q.dtype)
    idx = torch.empty(b, hkv, S, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_TOPK_SELECT, device=q.device)
    _lib.check("msa_topk_select", _lib.load().msa_topk_select(
        ctypes.byref(p), _ptr(q), _ptr(kbar), _ptr(kbar_hi), _ptr(kbar_lo), _ptr(idx),
        _ptr(ws), ws.numel(), _stream(q.device)))
    return idx


def sparse_attn_fwd(q, k, v, idx, block: int, scale=None, want_lse=True, ws=None):
    """Causal attention over the blocks in idx.  Returns (o, lse or None)."""
    topk = idx.shape[-1]
    p = _prefill_params(q, k, block, topk, scale)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float32,
                      device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(p, OP_SPARSE_ATTN, device=q.device)
    _lib.check("msa_sparse_attn_fwd", _lib.load().msa_sparse_attn_fwd(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(q.device)))
    return o, lse


def prefill_fwd(q, k, v, block: int, topk: int, scale=None, want_lse=True, ws=None, out=None):
    """Whole causal prefill.  Returns (o, lse or None, idx).  `out` may pass preallocated
    (o, lse, idx) tensors."""
    p = _prefill_params(q, k, block, topk, scale)
    b, S, hq, d = q.shape
    hkv = k.shape[2]
    if out is not None:
        o, lse, idx = out
    else:
        o = torch.empty_like(q)
        lse = torch.empty(b, hq, S, dtype=torch.float32, device=q.device) if want_lse else None
        idx = torch.empty(b, hkv, S, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_PREFILL, device=q.device)
    _lib.check("msa_prefill_fwd", _lib.load().msa_prefill_fwd(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(q.device)))
    return o, lse, idx


def decode_fwd(q, kbar, k_bank, v_bank, block: int, topk: int, scale=None, kbar_hi=None,
               kbar_lo=None, want_lse=True, ws=None, out=None):
    """Decode of q [n_query, hq, d] against a bank (k/v [S, hkv, d], pooled keys
    [nb, hkv, d]: fp32 kbar and/or the bf16 hi/lo planes; with both planes and bf16 q,
    d = 128, the tensor-core scan runs and kbar may be None).
    Returns (o, lse or None, idx [n_query, hkv, topk])."""
    nq, hq, d = q.shape
    S, hkv, _ = k_bank.shape
    p = params(batch=1, seq=S, hq=hq, hkv=hkv, d=d, block=block, topk=topk,
               scale=scale if scale is not None else d ** -0.5, dtype=q.dtype)
    if out is not None:
        o, lse, idx = out
    else:
        o = torch.empty_like(q)
        lse = torch.empty(nq, hq, dtype=torch.float32, device=q.device) if want_lse else None
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_DECODE, nq, device=q.device)
    _lib.check("msa_decode_fwd", _lib.load().msa_decode_fwd(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar), _ptr(kbar_hi), _ptr(kbar_lo), _ptr(k_bank),
        _ptr(v_bank), _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse, idx


def decode_fwd_static(q, kbar, k_bank, v_bank, block: int, topk: int, scale=None,
                      kbar_hi=None, kbar_lo=None, want_lse=True, out=None):
    """decode_fwd without a workspace: the library's fixed device scratch is used (for
    callers that cannot allocate device memory; see msa_decode_fwd_static in msa.h)."""
    nq, hq, d = q.shape
    S, hkv, _ = k_bank.shape
    p = params(batch=1, seq=S, hq=hq, hkv=hkv, d=d, block=block, topk=topk,
               scale=scale if scale is not None else d ** -0.5, dtype=q.dtype)
    if out is not None:
        o, lse, idx = out
    else:
        o = torch.empty_like(q)
        lse = torch.empty(nq, hq, dtype=torch.float32, device=q.device) if want_lse else None
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=q.device)
    _lib.check("msa_decode_fwd_static", _lib.load().msa_decode_fwd_static(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar), _ptr(kbar_hi), _ptr(kbar_lo), _ptr(k_bank),
        _ptr(v_bank), _ptr(idx), _ptr(o), _ptr(lse), _stream(q.device)))
    return o, lse, idx


def _bank_params(q, seq, hkv, block, topk, scale):
    nq, hq, d = q.shape
    return params(batch=1, seq=seq, hq=hq, hkv=hkv, d=d, block=block, topk=topk,
                  scale=scale if scale is not None else d ** -0.5, dtype=q.dtype)


def encode_bank(k_bank, v_bank, kbar_hi, kbar_lo, block: int):
    """Encoded images of a bank (see msa_encode_bank): returns (k_tiles, v_tiles,
    kbar_tiles) as uint8 CUDA tensors."""
    S, hkv, d = k_bank.shape
    p = params(batch=1, seq=S, hq=hkv, hkv=hkv, d=d, block=block, topk=1, scale=1.0,
               dtype=k_bank.dtype)
    lib = _lib.load()
    nkv, nkb = lib.msa_bank_tiles_bytes(ctypes.byref(p), 0), lib.msa_bank_tiles_bytes(ctypes.byref(p), 1)
    if nkv == 0 or nkb == 0:
        raise MsaError("msa_bank_tiles_bytes", _lib.MSA_ERR_INVALID_ARG, "invalid shapes")
    dev = k_bank.device
    kt = torch.empty(nkv, dtype=torch.uint8, device=dev)
    vt = torch.empty(nkv, dtype=torch.uint8, device=dev)
    bt = torch.empty(nkb, dtype=torch.uint8, device=dev)
    _lib.check("msa_encode_bank", lib.msa_encode_bank(
        ctypes.byref(p), _ptr(k_bank), _ptr(v_bank), _ptr(kbar_hi), _ptr(kbar_lo), _ptr(kt),
        _ptr(vt), _ptr(bt), _stream(dev)))
    return kt, vt, bt


def decode_fwd_tiled(q, kbar_tiles, k_tiles, v_tiles, seq: int, hkv: int, block: int, topk: int,
                     scale=None, want_lse=True, ws=None, out=None):
    """decode_fwd over an encoded bank of `seq` tokens (images from encode_bank)."""
    nq, hq, d = q.shape
    p = _bank_params(q, seq, hkv, block, topk, scale)
    if out is not None:
        o, lse, idx = out
    else:
        o = torch.empty_like(q)
        lse = torch.empty(nq, hq, dtype=torch.float32, device=q.device) if want_lse else None
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_DECODE, nq, device=q.device)
    _lib.check("msa_decode_fwd_tiled", _lib.load().msa_decode_fwd_tiled(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar_tiles), _ptr(k_tiles), _ptr(v_tiles), _ptr(idx),
        _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse, idx


def decode_select_tiled(q, kbar_tiles, seq: int, hkv: int, block: int, topk: int, ws=None,
                        idx=None):
    """The selection step of decode_fwd_tiled: idx [n_query, hkv, topk]."""
    nq = q.shape[0]
    p = _bank_params(q, seq, hkv, block, topk, None)
    if idx is None:
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_DECODE, nq, device=q.device)
    _lib.check("msa_decode_select_tiled", _lib.load().msa_decode_select_tiled(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar_tiles), _ptr(idx), _ptr(ws), ws.numel(),
        _stream(q.device)))
    return idx


def decode_attn_tiled(q, k_tiles, v_tiles, idx, seq: int, hkv: int, block: int, scale=None,
                      want_lse=True, ws=None):
    """The attention step of decode_fwd_tiled for a given idx [n_query, hkv, topk]."""
    nq, hq, d = q.shape
    topk = idx.shape[-1]
    p = _bank_params(q, seq, hkv, block, topk, scale)
    o = torch.empty_like(q)
    lse = torch.empty(nq, hq, dtype=torch.float32, device=q.device) if want_lse else None
    if ws is None:
        ws = workspace(p, OP_DECODE, nq, device=q.device)
    _lib.check("msa_decode_attn_tiled", _lib.load().msa_decode_attn_tiled(
        ctypes.byref(p), nq, _ptr(q), _ptr(k_tiles), _ptr(v_tiles), _ptr(idx), _ptr(o), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse


def read_device_error(ws: torch.Tensor) -> int:
    """Synchronises the current stream and returns the workspace's device error bits."""
    bits = ctypes.c_int32(0)
    st = _lib.load().msa_read_device_error(_ptr(ws), ctypes.byref(bits), _stream(ws.device))
    if st not in (_lib.MSA_OK, _lib.MSA_ERR_DEVICE):
        _lib.check("msa_read_device_error", st)
    return bits.value


def clear_device_error(ws: torch.Tensor) -> None:
    _lib.check("msa_clear_device_error", _lib.load().msa_clear_device_error(
        _ptr(ws), _stream(ws.device)))


def exp2_poly_eval(x: torch.Tensor) -> torch.Tensor:
    """The attention softmax's own FMA-pipe 2^x on a CUDA fp32 tensor (diagnostic)."""
    if x.dtype != torch.float32:
        raise ValueError("exp2_poly_eval takes fp32")
    y = torch.empty_like(x)
    _lib.check("msa_exp2_poly_eval", _lib.load().msa_exp2_poly_eval(
        _ptr(x), _ptr(y), x.numel(), _stream(x.device)))
    return y


def rope_docwise(q: torch.Tensor, k: torch.Tensor, cu_seqlens: torch.Tensor, base: float):
    """Rotates packed q [T, hq, d] and k [T, hkv, d] in place by each token's position in
    its own document (cu_seqlens: int32 CUDA tensor of the n_docs + 1 boundaries)."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    p = params(batch=1, seq=T, hq=hq, hkv=hkv, d=d, block=1, topk=1, scale=1.0, dtype=q.dtype)
    _lib.check("msa_rope_docwise", _lib.load().msa_rope_docwise(
        ctypes.byref(p), _ptr(cu_seqlens), cu_seqlens.numel() - 1, _ptr(q), _ptr(k),
        float(base), _stream(q.device)))
    return q, k


def varlen_workspace(q, k, cu_seqlens, block: int, topk: int, minimum: bool = False):
    """A workspace for prefill_varlen_fwd (sized for the longest document)."""
    T, hq, d = q.shape
    longest = max(int(b) - int(a) for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:]))
    p = params(batch=1, seq=max(1, longest), hq=hq, hkv=k.shape[1], d=d, block=block, topk=topk,
               scale=1.0, dtype=q.dtype)
    return workspace(p, OP_PREFILL_MIN if minimum else OP_PREFILL, device=q.device)


def prefill_varlen_fwd(q, k, v, cu_seqlens, block: int, topk: int, scale=None, want_lse=True,
                       ws=None):
    """Causal prefill of packed documents (q [T, hq, d], k/v [T, hkv, d]; cu_seqlens a host
    sequence of the n_docs + 1 boundaries).  Returns (o [T, hq, d], lse, idx) with idx and
    lse in the per-document layout of msa_prefill_varlen_fwd (flat tensors)."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    cu = [int(x) for x in cu_seqlens]
    p = params(batch=1, seq=T, hq=hq, hkv=hkv, d=d, block=block, topk=topk,
               scale=scale if scale is not None else d ** -0.5, dtype=q.dtype)
    o = torch.empty_like(q)
    lse = torch.empty(T * hq, dtype=torch.float32, device=q.device) if want_lse else None
    idx = torch.empty(T * hkv * topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = varlen_workspace(q, k, cu, block, topk)
    cu_host = (ctypes.c_int64 * len(cu))(*cu)
    _lib.check("msa_prefill_varlen_fwd", _lib.load().msa_prefill_varlen_fwd(
        ctypes.byref(p), cu_host, len(cu) - 1, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o),
        _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse, idx


def decode_select_shard(q, kbar_tiles, seq: int, hkv: int, block: int, topk: int,
                        block_offset: int, ws=None, keys=None):
    """Memory Parallel step 1: the best topk keys per (query, group) of one bank shard of
    `seq` tokens whose first block has bank-wide id block_offset.  Returns keys
    [n_query, hkv, topk] as int64 bit patterns (score bits above ~block id; 0 = empty)."""
    nq = q.shape[0]
    p = _bank_params(q, seq, hkv, block, topk, None)
    if keys is None:
        keys = torch.empty(nq, hkv, topk, dtype=torch.int64, device=q.device)
    if ws is None:
        ws = workspace(p, OP_DECODE, nq, device=q.device)
    _lib.check("msa_decode_select_shard", _lib.load().msa_decode_select_shard(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar_tiles), int(block_offset), _ptr(keys),
        _ptr(ws), ws.numel(), _stream(q.device)))
    return keys


def decode_merge_shards(keys_all, hq: int, d: int, block_begin: int, block_count: int,
                        dtype=torch.bfloat16, idx=None, idx_local=None):
    """Memory Parallel step 2: keys_all [world, n_query, hkv, topk] (all ranks' lists in
    rank order) -> (idx [n_query, hkv, topk] bank-wide, idx_local: the ids local to the
    shard [block_begin, block_begin + block_count) of the blocks it owns, -1 elsewhere)."""
    world, nq, hkv, topk = keys_all.shape
    p = params(batch=1, seq=1, hq=hq, hkv=hkv, d=d, block=1, topk=topk, scale=1.0, dtype=dtype)
    dev = keys_all.device
    if idx is None:
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=dev)
    if idx_local is None:
        idx_local = torch.empty_like(idx)
    _lib.check("msa_decode_merge_shards", _lib.load().msa_decode_merge_shards(
        ctypes.byref(p), nq, _ptr(keys_all), world, int(block_begin), int(block_count),
        _ptr(idx), _ptr(idx_local), _stream(dev)))
    return idx, idx_local


def decode_combine_shards(o_parts, lse_parts, hkv: int, o=None, lse=None):
    """Memory Parallel step 4: partials o [world, n_query, hq, d] and lse [world, n_query,
    hq] -> the softmax over the whole selection (o [n_query, hq, d], lse [n_query, hq])."""
    world, nq, hq, d = o_parts.shape
    p = params(batch=1, seq=1, hq=hq, hkv=hkv, d=d, block=1, topk=1, scale=1.0,
               dtype=o_parts.dtype)
    if o is None:
        o = torch.empty(nq, hq, d, dtype=o_parts.dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty(nq, hq, dtype=torch.float32, device=o_parts.device)
    _lib.check("msa_decode_combine_shards", _lib.load().msa_decode_combine_shards(
        ctypes.byref(p), nq, _ptr(o_parts), _ptr(lse_parts), world, _ptr(o), _ptr(lse),
        _stream(o_parts.device)))
    return o, lse


def decode_fwd_offload(q, kbar_tiles, k_tiles_host, v_tiles_host, seq: int, hkv: int, block: int,
                       topk: int, scale=None, want_lse=True, ws=None, out=None):
    """decode_fwd_tiled with the encoded K/V images in PINNED host memory (k_tiles_host,
    v_tiles_host: pinned CPU uint8 tensors from encode_bank); the pooled-key planes
    (kbar_tiles) in HBM.  Selected blocks are fetched over PCIe into a staging bank in the
    workspace."""
    nq, hq, d = q.shape
    p = _bank_params(q, seq, hkv, block, topk, scale)
    for t in (k_tiles_host, v_tiles_host):
        if t.is_cuda or not t.is_pinned():
            raise ValueError("k_tiles_host / v_tiles_host must be pinned host tensors")
    if out is not None:
        o, lse, idx = out
    else:
        o = torch.empty_like(q)
        lse = torch.empty(nq, hq, dtype=torch.float32, device=q.device) if want_lse else None
        idx = torch.empty(nq, hkv, topk, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_DECODE_OFFLOAD, nq, device=q.device)
    _lib.check("msa_decode_fwd_offload", _lib.load().msa_decode_fwd_offload(
        ctypes.byref(p), nq, _ptr(q), _ptr(kbar_tiles),
        ctypes.c_void_p(k_tiles_host.data_ptr()), ctypes.c_void_p(v_tiles_host.data_ptr()),
        _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse, idx


def sparse_attn_bwd(q, k, v, o, lse, dout, idx, block: int, scale=None, ws=None, out=None):
    """Gradients of the causal sparse attention for a fixed selection idx: (dq, dk, dv),
    fp32, shapes of q, k, v.  o and lse are the forward's outputs, dout the upstream
    gradient of o."""
    topk = idx.shape[-1]
    p = _prefill_params(q, k, block, topk, scale)
    if out is not None:
        dq, dk, dv = out
    else:
        dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
        dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(p, OP_SPARSE_ATTN_BWD, device=q.device)
    _lib.check("msa_sparse_attn_bwd", _lib.load().msa_sparse_attn_bwd(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(idx),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(), _stream(q.device)))
    return dq, dk, dv
