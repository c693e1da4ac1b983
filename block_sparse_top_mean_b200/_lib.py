"""ctypes binding of libmsa_b200.so (the C ABI declared in include/msa.h).

Loading fails loudly when the library is missing: there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmsa_b200.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_WORKSPACE, MSA_ERR_CUDA, \
    MSA_ERR_DEVICE, MSA_ERR_TIMEOUT = range(7)
MSA_F32, MSA_BF16 = 0, 1
OP_TOPK_SELECT, OP_SPARSE_ATTN, OP_PREFILL, OP_DECODE, OP_SPARSE_ATTN_MIN, OP_PREFILL_MIN, \
    OP_DECODE_OFFLOAD, OP_SPARSE_ATTN_BWD, OP_SPARSE_ATTN_BWD_MIN = range(9)
DEVERR_IDX_RANGE, DEVERR_TIMEOUT = 0x1, 0x2

# Every symbol include/msa.h declares, with (restype, argtypes).
SIGNATURES = {
    "msa_version": (c_char_p, []),
    "msa_status_string": (c_char_p, [c_int32]),
    "msa_workspace_bytes": (c_size_t, [c_void_p, c_int32, c_int64]),
    "msa_attn_slab_tokens": (c_int64, [c_void_p, c_int32, c_size_t]),
    "msa_pool_keys": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "msa_block_scores": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "msa_topk_select": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_size_t, c_void_p]),
    "msa_sparse_attn_fwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "msa_prefill_fwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_size_t, c_void_p]),
    "msa_decode_fwd": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]),
    "msa_decode_fwd_static": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p]),
    "msa_decode_static_read_error": (c_int32, [c_void_p, c_void_p]),
    "msa_bank_tiles_bytes": (c_size_t, [c_void_p, c_int32]),
    "msa_encode_bank": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p]),
    "msa_decode_select_tiled": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_size_t, c_void_p]),
    "msa_decode_attn_tiled": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
    "msa_decode_fwd_tiled": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_size_t, c_void_p]),
    "msa_read_device_error": (c_int32, [c_void_p, POINTER(c_int32), c_void_p]),
    "msa_clear_device_error": (c_int32, [c_void_p, c_void_p]),
    "msa_workspace_size": (c_size_t, [c_void_p, c_int32, c_int64]),
    "msa_get_device_status": (c_int32, [c_void_p, c_void_p]),
    "msa_exp2_poly_eval": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p]),
    "msa_decode_select_shard": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_int64,
                                          c_void_p, c_void_p, c_size_t, c_void_p]),
    "msa_decode_merge_shards": (c_int32, [c_void_p, c_int64, c_void_p, c_int64, c_int64,
                                          c_int64, c_void_p, c_void_p, c_void_p]),
    "msa_decode_combine_shards": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_int64,
                                            c_void_p, c_void_p, c_void_p]),
    "msa_sparse_attn_bwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "msa_decode_fwd_offload": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_size_t, c_void_p]),
    "msa_rope_docwise": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_double,
                                   c_void_p]),
    "msa_prefill_varlen_fwd": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_size_t, c_void_p]),
}


class MsaParams(ctypes.Structure):
    """Mirror of msa_params (include/msa.h)."""
    _fields_ = [("batch", c_int64), ("seq", c_int64), ("hq", c_int64), ("hkv", c_int64),
                ("d", c_int64), ("block", c_int64), ("topk", c_int64), ("scale", c_float),
                ("dtype", c_int32)]


class MsaError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: {text} (status {status})")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the library once.  Raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m block_sparse_top_mean_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != MSA_OK:
        text = load().msa_status_string(status).decode()
        raise MsaError(fn, status, text)
