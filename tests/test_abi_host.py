"""The C ABI on the host: the library loads, exports every symbol include/msa.h declares,
and rejects bad arguments before touching the device (these calls need no GPU)."""
import ctypes
import os
import re

import pytest

from block_sparse_top_mean_b200 import _lib
from block_sparse_top_mean_b200._lib import MsaParams

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_top_mean_b200 import build
    build.build()
    return _lib.load()


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for n in ["msa_pool_keys", "msa_block_scores", "msa_topk_select", "msa_sparse_attn_fwd",
              "msa_decode_fwd", "msa_prefill_fwd", "msa_workspace_bytes"]:
        assert n in names


def test_header_is_plain_c(tmp_path):
    """include/msa.h is a C header (no C++ or CUDA types): it compiles as C99 alone."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "msa.h"\nint main(void) { msa_params p; (void)p; return 0; }\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o",
                        str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_constants_match_the_header():
    """Status codes, dtypes, workspace ops and device-error bits: the binding's values are
    the header's."""
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    enum = {k: int(v) for k, v in re.findall(r"\b(MSA_[A-Z0-9_]+)\s*=\s*(\d+)", src)}
    defs = {k: int(v, 0) for k, v in re.findall(r"#define\s+(MSA_DEVERR_\w+)\s+(0x[0-9a-fA-F]+)",
                                                 src)}
    for name in ("MSA_OK", "MSA_ERR_INVALID_ARG", "MSA_ERR_UNSUPPORTED", "MSA_ERR_WORKSPACE",
                 "MSA_ERR_CUDA", "MSA_ERR_DEVICE", "MSA_ERR_TIMEOUT", "MSA_F32", "MSA_BF16"):
        assert getattr(_lib, name) == enum[name], name
    for name in ("TOPK_SELECT", "SPARSE_ATTN", "PREFILL", "DECODE", "SPARSE_ATTN_MIN",
                 "PREFILL_MIN", "DECODE_OFFLOAD", "SPARSE_ATTN_BWD", "SPARSE_ATTN_BWD_MIN"):
        assert getattr(_lib, "OP_" + name) == enum["MSA_OP_" + name], name
    assert _lib.DEVERR_IDX_RANGE == defs["MSA_DEVERR_IDX_RANGE"]
    assert _lib.DEVERR_TIMEOUT == defs["MSA_DEVERR_TIMEOUT"]


def test_library_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"
    for n in names:
        assert hasattr(lib, n), n
    assert lib.msa_version().decode().startswith("msa-b200")


def _p(**kw):
    base = dict(batch=1, seq=1024, hq=32, hkv=8, d=128, block=128, topk=16, scale=0.088,
                dtype=_lib.MSA_BF16)
    base.update(kw)
    return MsaParams(*[base[k] for k in ["batch", "seq", "hq", "hkv", "d", "block", "topk",
                                         "scale", "dtype"]])


FAKE = ctypes.c_void_p(4096)       # non-null, aligned; never dereferenced (checks fail first)


@pytest.mark.parametrize("kw,code", [
    (dict(hq=30), _lib.MSA_ERR_INVALID_ARG),          # hq % hkv != 0
    (dict(block=0), _lib.MSA_ERR_INVALID_ARG),
    (dict(topk=0), _lib.MSA_ERR_INVALID_ARG),
    (dict(seq=-1), _lib.MSA_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.MSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.MSA_ERR_INVALID_ARG),
    (dict(d=96), _lib.MSA_ERR_UNSUPPORTED),
    (dict(topk=33), _lib.MSA_ERR_UNSUPPORTED),
    (dict(hq=24, hkv=8), _lib.MSA_ERR_UNSUPPORTED),     # G = 3
])
def test_bad_params_rejected_before_launch(lib, kw, code):
    p = _p(**kw)
    st = lib.msa_sparse_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                 1 << 20, None)
    assert st == code
    assert lib.msa_workspace_bytes(ctypes.byref(p), _lib.OP_PREFILL, 0) == 0
    assert lib.msa_pool_keys(ctypes.byref(p), FAKE, FAKE, None, None, None) == code


def test_null_and_misaligned_pointers_rejected(lib):
    p = _p()
    assert lib.msa_pool_keys(None, FAKE, FAKE, None, None, None) == _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_pool_keys(ctypes.byref(p), None, FAKE, None, None, None) == \
        _lib.MSA_ERR_INVALID_ARG
    odd = ctypes.c_void_p(4096 + 8)
    assert lib.msa_pool_keys(ctypes.byref(p), odd, FAKE, None, None, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_sparse_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE, None, FAKE,
                                   1 << 20, None) == _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_read_device_error(None, None, None) == _lib.MSA_ERR_INVALID_ARG


def test_workspace_checks(lib):
    p = _p()
    need = lib.msa_workspace_bytes(ctypes.byref(p), _lib.OP_PREFILL, 0)
    assert need >= 256 + 8 * 8 * 128 * 4          # header + pooled keys [1, 8, 8, 128] fp32
    st = lib.msa_prefill_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                             need - 1, None)
    assert st == _lib.MSA_ERR_WORKSPACE
    st = lib.msa_prefill_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None,
                             ctypes.c_void_p(4096 + 16), need, None)
    assert st == _lib.MSA_ERR_WORKSPACE              # not 256-byte aligned
    st = lib.msa_prefill_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, need, None)
    assert st == _lib.MSA_ERR_WORKSPACE
    nd = lib.msa_workspace_bytes(ctypes.byref(_p(seq=10_000_000, block=64, topk=32)),
                                 _lib.OP_DECODE, 64)
    assert nd > 256
    assert lib.msa_workspace_bytes(ctypes.byref(p), 99, 0) == 0


def test_attention_workspace_bounded_by_token_slabs(lib):
    """The key-centric attention keeps one partial per (token, group, selected segment);
    at 1M tokens that is ~140 GB, so the library walks the sequence in token slabs:
    the recommended size stays near 32 GiB and the minimum is one 2048-token slab."""
    def ws(op, **kw):
        return lib.msa_workspace_bytes(ctypes.byref(_p(**kw)), op, 0)
    big = dict(seq=1_048_576, hq=32, hkv=8, block=256, topk=16)
    rec, mn = ws(_lib.OP_SPARSE_ATTN, **big), ws(_lib.OP_SPARSE_ATTN_MIN, **big)
    assert 16 << 30 < rec <= (33 << 30)
    assert 0 < mn < (1 << 30) and mn < rec
    # prefill adds the same fixed part (pooled keys, split planes, flags) to both
    frec, fmn = ws(_lib.OP_PREFILL, **big), ws(_lib.OP_PREFILL_MIN, **big)
    assert frec - rec == fmn - mn > 0
    # short sequences: one slab, minimum == recommended
    assert ws(_lib.OP_SPARSE_ATTN, seq=1500) == ws(_lib.OP_SPARSE_ATTN_MIN, seq=1500)
    # the slab plan: evened-out slabs of 2048-token multiples, one pass when it all fits
    p = _p(**big)
    slab = lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_SPARSE_ATTN, rec)
    assert slab % 2048 == 0 and 1 < -(-big["seq"] // slab) <= 8
    assert lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_PREFILL, frec) == slab
    assert lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_SPARSE_ATTN, mn) == 2048
    assert lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_SPARSE_ATTN, mn - 1) == 0
    assert lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_SPARSE_ATTN, 1 << 40) == big["seq"]
    assert lib.msa_attn_slab_tokens(ctypes.byref(p), _lib.OP_DECODE, 1 << 40) == -1
    # the minimum is the floor the calls accept
    st = lib.msa_sparse_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                 mn - 1, None)
    assert st == _lib.MSA_ERR_WORKSPACE
    st = lib.msa_prefill_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                             fmn - 1, None)
    assert st == _lib.MSA_ERR_WORKSPACE


def test_encoded_bank_sizes_closed_form(lib):
    p = _p(seq=10_000_000, block=64, topk=32)
    nb = -(-10_000_000 // 64)
    assert lib.msa_bank_tiles_bytes(ctypes.byref(p), 0) == 8 * (-(-10_000_000 // 64)) * 16384
    # hi plane, lo plane, then 256 bytes of per-head bounds (max ||lo_j||, max ||hi_j||)
    assert lib.msa_bank_tiles_bytes(ctypes.byref(p), 1) == 2 * 8 * (-(-nb // 128)) * 32768 + 256
    assert lib.msa_bank_tiles_bytes(ctypes.byref(p), 2) == 0
    assert lib.msa_bank_tiles_bytes(ctypes.byref(_p(seq=1000, hq=30)), 0) == 0
    # the bounds hold at most 32 KV heads
    assert lib.msa_bank_tiles_bytes(ctypes.byref(_p(seq=1000, hq=64, hkv=64)), 1) == 0
    assert lib.msa_bank_tiles_bytes(ctypes.byref(_p(seq=1000, hq=32, hkv=32)), 1) > 0


def test_encoded_bank_entries_check_arguments_before_launch(lib):
    p = _p(seq=1_000_000, block=64, topk=32)
    pp = ctypes.byref(p)
    odd = ctypes.c_void_p(4096 + 8)
    # encoding: only the tensor-core decode shapes; each image needs its source
    assert lib.msa_encode_bank(ctypes.byref(_p(seq=1000, block=64, dtype=_lib.MSA_F32)), FAKE,
                               FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
        _lib.MSA_ERR_UNSUPPORTED
    assert lib.msa_encode_bank(pp, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_encode_bank(pp, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_encode_bank(pp, odd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_encode_bank(ctypes.byref(_p(seq=0, block=64)), None, None, None, None,
                               FAKE, FAKE, FAKE, None) == _lib.MSA_OK
    need = lib.msa_workspace_bytes(pp, _lib.OP_DECODE, 64)
    assert need > 256
    sel, att, fwd = lib.msa_decode_select_tiled, lib.msa_decode_attn_tiled, \
        lib.msa_decode_fwd_tiled
    # no queries: nothing to do, nothing launched
    assert sel(pp, 0, None, None, None, None, 0, None) == _lib.MSA_OK
    assert att(pp, 0, None, None, None, None, None, None, None, 0, None) == _lib.MSA_OK
    assert fwd(pp, 0, None, None, None, None, None, None, None, None, 0, None) == _lib.MSA_OK
    assert sel(pp, -1, FAKE, FAKE, FAKE, FAKE, need, None) == _lib.MSA_ERR_INVALID_ARG
    assert sel(pp, 64, None, FAKE, FAKE, FAKE, need, None) == _lib.MSA_ERR_INVALID_ARG
    assert sel(pp, 64, FAKE, None, FAKE, FAKE, need, None) == _lib.MSA_ERR_INVALID_ARG
    assert sel(pp, 64, FAKE, odd, FAKE, FAKE, need, None) == _lib.MSA_ERR_INVALID_ARG
    assert sel(pp, 64, FAKE, FAKE, FAKE, FAKE, need - 1, None) == _lib.MSA_ERR_WORKSPACE
    assert att(pp, 64, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, need, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert att(pp, 64, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need - 1, None) == \
        _lib.MSA_ERR_WORKSPACE
    # fp32 banks and d = 64 have no encoded form
    for bad in (_p(seq=1000, block=64, dtype=_lib.MSA_F32), _p(seq=1000, block=64, d=64)):
        assert sel(ctypes.byref(bad), 4, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == \
            _lib.MSA_ERR_UNSUPPORTED


def test_static_decode_rejects_before_touching_the_device(lib):
    p = _p(seq=10_000_000, block=64, topk=32)
    st = lib.msa_decode_fwd_static
    assert st(None, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == \
        _lib.MSA_ERR_INVALID_ARG
    assert st(ctypes.byref(p), -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
              None) == _lib.MSA_ERR_INVALID_ARG
    assert st(ctypes.byref(p), 0, None, None, None, None, None, None, None, None, None,
              None) == _lib.MSA_OK
    # more queries than the fixed 32 MiB scratch can hold
    assert st(ctypes.byref(p), 100_000, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
              None) == _lib.MSA_ERR_WORKSPACE
    # null and misaligned pointers, and unsupported shapes, give msa_decode_fwd's own
    # statuses without any CUDA call (on this host any CUDA call would return an error)
    odd = ctypes.c_void_p(4096 + 8)
    args = [FAKE] * 8                                 # q, kbar, hi, lo, k, v, idx, o
    for i, bad in [(0, None), (4, None), (5, None), (6, None), (7, None), (0, odd), (4, odd),
                   (7, odd), (2, odd)]:
        a = list(args)
        a[i] = bad
        assert st(ctypes.byref(p), 4, *a, None, None) == _lib.MSA_ERR_INVALID_ARG, (i, bad)
    # no planes and no fp32 pooled keys
    assert st(ctypes.byref(p), 4, FAKE, None, None, None, FAKE, FAKE, FAKE, FAKE, None,
              None) == _lib.MSA_ERR_INVALID_ARG
    for kw in (dict(d=96), dict(hq=24)):              # G = 3 and d = 96 are unsupported
        bad = _p(seq=10_000, block=64, topk=32, **kw)
        assert st(ctypes.byref(bad), 4, *args, None, None) == _lib.MSA_ERR_UNSUPPORTED
    # the array's error bits: a null destination is rejected before any CUDA call
    assert lib.msa_decode_static_read_error(None, None) == _lib.MSA_ERR_INVALID_ARG


def test_empty_inputs_are_noops(lib):
    for kw in (dict(seq=0), dict(batch=0)):
        p = _p(**kw)
        assert lib.msa_prefill_fwd(ctypes.byref(p), None, None, None, None, None, None, None, 0,
                                   None) == _lib.MSA_OK
        assert lib.msa_pool_keys(ctypes.byref(p), None, None, None, None, None) == _lib.MSA_OK
    p = _p()
    assert lib.msa_decode_fwd(ctypes.byref(p), 0, None, None, None, None, None, None, None,
                              None, None, None, 0, None) == _lib.MSA_OK


def test_status_strings(lib):
    for c in range(7):
        assert lib.msa_status_string(c).decode()


def test_interface_sketch_names(lib):
    """msa_workspace_size is msa_workspace_bytes; msa_get_device_status rejects a null
    workspace before any CUDA call."""
    for op in range(6):
        p = _p()
        assert lib.msa_workspace_size(ctypes.byref(p), op, 64) == \
            lib.msa_workspace_bytes(ctypes.byref(p), op, 64)
    assert lib.msa_get_device_status(None, None) == _lib.MSA_ERR_INVALID_ARG
    assert lib.msa_status_string(_lib.MSA_ERR_TIMEOUT).decode() == "a bounded device wait ran out"


def test_docwise_entries_reject_bad_arguments_on_the_host(lib):
    p = _p(seq=1000, block=64, topk=4)
    rope = lib.msa_rope_docwise
    for n_docs, base, cu, q, k in [(0, 1e4, FAKE, FAKE, FAKE), (1, 1.0, FAKE, FAKE, FAKE),
                                   (1, float("inf"), FAKE, FAKE, FAKE), (1, 1e4, None, FAKE, FAKE),
                                   (1, 1e4, FAKE, None, FAKE), (1, 1e4, FAKE, FAKE,
                                                                ctypes.c_void_p(4100))]:
        assert rope(ctypes.byref(p), cu, n_docs, q, k, base, None) == _lib.MSA_ERR_INVALID_ARG
    var = lib.msa_prefill_varlen_fwd
    cu = (ctypes.c_int64 * 3)(0, 400, 1000)
    bad_cus = [(ctypes.c_int64 * 3)(1, 400, 1000), (ctypes.c_int64 * 3)(0, 400, 999),
               (ctypes.c_int64 * 3)(0, 1001, 1000)]
    for c in bad_cus:
        assert var(ctypes.byref(p), c, 2, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
                   None) == _lib.MSA_ERR_INVALID_ARG
    p2 = _p(batch=2, seq=1000, block=64, topk=4)
    assert var(ctypes.byref(p2), cu, 2, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 40,
               None) == _lib.MSA_ERR_INVALID_ARG
    # the workspace is sized for the longest document (600 tokens)
    p600 = _p(seq=600, block=64, topk=4)
    need = lib.msa_workspace_bytes(ctypes.byref(p600), _lib.OP_PREFILL_MIN, 0)
    assert var(ctypes.byref(p), cu, 2, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, need - 1,
               None) == _lib.MSA_ERR_WORKSPACE
