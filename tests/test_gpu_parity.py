"""GPU path vs the fp64 oracle, through the C ABI (via the ctypes binding).

Small cases compare every row; they span several kernel tiles and a ragged tail.
The full-size workloads are checked on a stratified sample of rows, with the same
launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import msa_inputs as mi
import oracle
from parity_util import (HostView, check_decode, check_prefill, pool_keys_chunked,
                         sample_tokens)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


def _inputs(w, seed=0):
    q, k, v = mi.prefill_inputs(w, device="cuda", seed=seed)
    return q, k, v


SMALL = [
    mi.WORKLOADS["prefill_tiny_s1k_f32"],
    mi.Workload("bf16_ragged_b128", "prefill", 1, 3000, 8, 2, 128, 128, 8, "bf16"),
    mi.Workload("bf16_ragged_b512", "prefill", 1, 5000, 8, 2, 128, 512, 8, "bf16"),
    mi.Workload("bf16_b256_g4", "prefill", 1, 4096, 16, 4, 128, 256, 6, "bf16"),
    mi.Workload("f32_d128_g8_b2", "prefill", 2, 700, 16, 2, 128, 64, 5, "f32"),
    mi.Workload("bf16_d64_g1", "prefill", 1, 2000, 4, 4, 64, 64, 4, "bf16"),
    mi.Workload("f32_topk1", "prefill", 1, 600, 4, 2, 64, 64, 1, "f32"),
    mi.Workload("f32_topk_all", "prefill", 1, 1000, 4, 1, 64, 64, 32, "f32"),
    mi.Workload("f32_one_partial_block", "prefill", 1, 50, 2, 1, 64, 64, 4, "f32"),
    mi.Workload("bf16_planted", "prefill", 1, 4096, 8, 2, 128, 128, 8, "bf16",
                planted_frac=0.02, planted_shift=3.0),
    mi.Workload("bf16_g8_b256", "prefill", 1, 2500, 16, 2, 128, 256, 5, "bf16"),
    mi.Workload("bf16_g1_b128", "prefill", 1, 1500, 4, 4, 128, 128, 4, "bf16"),
    mi.Workload("bf16_batch2_g2", "prefill", 2, 1000, 4, 2, 128, 128, 3, "bf16"),
    mi.Workload("bf16_b384_ragged", "prefill", 1, 2000, 8, 2, 128, 384, 4, "bf16"),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_prefill_small_all_rows(msa, w):
    q, k, v = _inputs(w)
    o, lse, idx = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    check_prefill(q, k, v, w.block, w.topk, w.scale, idx, o, lse)


@pytest.mark.parametrize("w", SMALL[:4], ids=lambda w: w.name)
def test_pool_keys_vs_oracle(msa, w):
    q, k, v = _inputs(w)
    kbar, hi, lo = msa.pool_keys(k, w.block, split=True)
    ref = oracle.pool_keys(k.float().cpu().numpy(), w.block)
    got = kbar.double().cpu().numpy()
    # fp32 sum of <= block terms of |x| < 6: error <= block * 2^-24 * 6
    assert np.abs(got - ref).max() <= w.block * 6 * 2.0 ** -24
    # split planes: hi = bf16(kbar), lo = bf16(kbar - hi)
    assert torch.equal(hi, kbar.to(torch.bfloat16))
    assert torch.equal(lo, (kbar - hi.float()).to(torch.bfloat16))


@pytest.mark.parametrize("w", SMALL[:3], ids=lambda w: w.name)
def test_block_scores_vs_oracle(msa, w):
    q, k, v = _inputs(w)
    kbar = msa.pool_keys(k, w.block)
    sc = msa.block_scores(q, kbar, w.block, w.hkv).double().cpu().numpy()
    kb = oracle.pool_keys(k.float().cpu().numpy(), w.block)
    Q = q.float().cpu().numpy()
    for t in range(0, w.seq, 97):
        i = t // w.block
        ref = oracle.prefill_block_scores(Q[0, t], kb[0], i)          # [hkv, i]
        got = sc[0, :, t, :]
        assert np.all(np.isinf(got[:, i:]))
        if i:
            np.testing.assert_allclose(got[:, :i], ref, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("w", SMALL[1:3], ids=lambda w: w.name)
def test_topk_select_and_attn_separately(msa, w):
    """Each step alone: the selection vs the oracle, and the attention fed the
    oracle's own selection vs the oracle."""
    q, k, v = _inputs(w)
    kbar = msa.pool_keys(k, w.block)
    idx = msa.topk_select(q, kbar, w.block, w.topk, w.hkv)
    rows = [(0, t) for t in range(0, w.seq, 7)]
    Q, K, V = HostView(q), HostView(k), HostView(v)
    ref = oracle.prefill_rows(Q, K, V, w.block, w.topk, w.scale, rows=rows)
    gi = idx.cpu().numpy()
    for r in ref:
        if r.gap > 1e-3:
            assert list(gi[0, r.g, r.t]) == r.idx
    oidx = torch.full_like(idx, -1)
    for r in oracle.prefill_rows(Q, K, V, w.block, w.topk, w.scale):
        oidx[0, r.g, r.t] = torch.tensor(r.idx)
    o, lse = msa.sparse_attn_fwd(q, k, v, oidx, w.block, w.scale)
    check_prefill(q, k, v, w.block, w.topk, w.scale, oidx, o, lse, rows=rows)


@pytest.mark.parametrize("w", [SMALL[1], SMALL[2], SMALL[3], SMALL[9], SMALL[10], SMALL[11],
                               SMALL[12]], ids=lambda w: w.name)
def test_topk_select_split_planes_vs_oracle(msa, w):
    """The selection fed the bf16 hi/lo planes (tensor-core path for bf16, d = 128)."""
    q, k, v = _inputs(w)
    kbar, hi, lo = msa.pool_keys(k, w.block, split=True)
    idx = msa.topk_select(q, kbar, w.block, w.topk, w.hkv, kbar_hi=hi, kbar_lo=lo)
    torch.cuda.synchronize()
    Q, K, V = HostView(q), HostView(k), HostView(v)
    kb = oracle.pool_keys(k.float().cpu().numpy(), w.block)
    rows = [(b, t) for b in range(w.batch) for t in range(0, w.seq, 3)]
    gi = idx.cpu().numpy()
    n_strict = 0
    for r in oracle.prefill_rows(Q, K, V, w.block, w.topk, w.scale, rows=rows, kbar=kb):
        sel = [int(x) for x in gi[r.b, r.g, r.t]]
        if r.gap > 1e-3:
            n_strict += 1
            assert sel == r.idx, (r.t, r.g, sel, r.idx)
        else:
            s = [j for j in sel if j >= 0]
            assert r.t // w.block in s and max(s) == r.t // w.block
    assert n_strict > 0


def test_selection_exact_ties_take_lowest_blocks(msa):
    """All-zero queries make every block score exactly 0: the tensor-core selection's
    candidate buffers overflow and its fallback must return the lowest block indices."""
    w = mi.Workload("bf16_all_ties", "prefill", 1, 16384, 8, 2, 128, 128, 8, "bf16")
    _, k, v = _inputs(w)
    q = torch.zeros(1, w.seq, w.hq, w.d, dtype=torch.bfloat16, device="cuda")
    kbar, hi, lo = msa.pool_keys(k, w.block, split=True)
    idx = msa.topk_select(q, kbar, w.block, w.topk, w.hkv, kbar_hi=hi, kbar_lo=lo)
    own = torch.arange(w.seq, device="cuda") // w.block
    n_past = torch.clamp(own, max=w.topk - 1)
    slot = torch.arange(w.topk, device="cuda")
    want = torch.where(slot[None] < n_past[:, None], slot[None], torch.full_like(slot[None], -1))
    want = torch.where(slot[None] == n_past[:, None], own[:, None], want)
    for g in range(w.hkv):
        assert torch.equal(idx[0, g].long(), want), g


def test_out_of_range_index_sets_error_word_and_skips(msa):
    w = SMALL[1]
    q, k, v = _inputs(w)
    kbar = msa.pool_keys(k, w.block)
    idx = msa.topk_select(q, kbar, w.block, w.topk, w.hkv)
    p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block, topk=w.topk,
                   scale=w.scale, dtype=q.dtype)
    ws = msa.workspace(p, msa.OP_SPARSE_ATTN)
    o_ref, _ = msa.sparse_attn_fwd(q, k, v, idx, w.block, w.scale, ws=ws)
    assert msa.read_device_error(ws) == 0
    bad = idx.clone()
    t = w.seq - 1
    bad[0, 0, t, 0] = 10_000          # beyond nb
    bad[0, 1, 5, 1] = 3               # a future block for token 5 (own block 0)
    o_bad, _ = msa.sparse_attn_fwd(q, k, v, bad, w.block, w.scale, ws=ws)
    assert msa.read_device_error(ws) & msa.DEVERR_IDX_RANGE
    msa.clear_device_error(ws)
    assert msa.read_device_error(ws) == 0
    # untouched rows are unchanged
    assert torch.equal(o_bad[0, :w.seq - 1, :w.hq // w.hkv], o_ref[0, :w.seq - 1, :w.hq // w.hkv])


def test_output_with_16_byte_alignment_only(msa):
    """The ABI promises 16-byte alignment; an output that is not 32-byte aligned must
    give the same result."""
    w = SMALL[1]
    q, k, v = _inputs(w)
    kbar = msa.pool_keys(k, w.block)
    idx = msa.topk_select(q, kbar, w.block, w.topk, w.hkv)
    o_ref, lse_ref = msa.sparse_attn_fwd(q, k, v, idx, w.block, w.scale)
    buf = torch.empty(q.numel() + 8, dtype=q.dtype, device="cuda")
    o = buf[8:].view(q.shape)                       # 16 bytes past a 32-byte boundary
    assert o.data_ptr() % 32 == 16
    p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block, topk=w.topk,
                   scale=w.scale, dtype=q.dtype)
    ws = msa.workspace(p, msa.OP_SPARSE_ATTN)
    import ctypes
    from block_sparse_top_mean_b200 import _lib
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib.load().msa_sparse_attn_fwd(ctypes.byref(p), P(q), P(k), P(v), P(idx), P(o), None,
                                         P(ws), ws.numel(),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)


def test_prefill_is_deterministic(msa):
    w = SMALL[3]
    q, k, v = _inputs(w)
    a = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    b = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("w", [
    mi.Workload("bf16_slabs_b128", "prefill", 2, 5000, 8, 2, 128, 128, 8, "bf16"),
    mi.Workload("bf16_slabs_b256_g4", "prefill", 1, 6500, 16, 4, 128, 256, 6, "bf16"),
], ids=lambda w: w.name)
def test_attention_in_token_slabs(msa, w):
    """With the minimum workspace the tensor-core attention walks the sequence in
    2048-token slabs (the last one ragged); every token's result is bitwise the one-pass
    result, and both match the oracle."""
    q, k, v = _inputs(w)
    o1, lse1, idx = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    p = msa._prefill_params(q, k, w.block, w.topk, w.scale)
    ws_min = msa.workspace(p, msa.OP_PREFILL_MIN, device=q.device)
    assert ws_min.numel() < msa.workspace(p, msa.OP_PREFILL, device=q.device).numel()
    o2, lse2, idx2 = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale, ws=ws_min)
    a_ws = msa.workspace(p, msa.OP_SPARSE_ATTN_MIN, device=q.device)
    o3, lse3 = msa.sparse_attn_fwd(q, k, v, idx, w.block, w.scale, ws=a_ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    for o, lse in [(o2, lse2), (o3, lse3)]:
        assert torch.equal(o, o1)
        assert torch.equal(lse, lse1)
    check_prefill(q, k, v, w.block, w.topk, w.scale, idx2, o2, lse2)
    assert msa.read_device_error(ws_min) == 0


DECODE_SMALL = [
    mi.Workload("decode_small_bf16", "decode", 1, 50_000, 32, 8, 128, 64, 32, "bf16", n_query=8),
    mi.Workload("decode_small_f32", "decode", 1, 9_000, 8, 2, 64, 64, 8, "f32", n_query=70),
    mi.Workload("decode_all_blocks", "decode", 1, 1000, 4, 1, 64, 64, 32, "f32", n_query=3),
]


@pytest.mark.parametrize("w", DECODE_SMALL, ids=lambda w: w.name)
def test_decode_small(msa, w):
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    kbar = msa.pool_keys(kb[None], w.block)[0]
    o, lse, idx = msa.decode_fwd(q, kbar, kb, vb, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    kbar_np = pool_keys_chunked(kb[None], w.block)[0]
    check_decode(q, kbar_np, kb, vb, w.block, w.topk, w.scale, idx, o, lse)


# Tensor-core bank scan (bf16 hi/lo planes of the pooled keys): several chunks per CTA,
# CTAs that span two groups, ragged last chunk, query tiles beyond 64, G = 1 / 2 / 4 / 8,
# topk below 32 and a bank with fewer blocks than topk.
DECODE_TC = [
    mi.Workload("dtc_b50k_g4", "decode", 1, 50_000, 32, 8, 128, 64, 32, "bf16", n_query=8),
    mi.Workload("dtc_b300k_q100", "decode", 1, 300_000, 32, 8, 128, 64, 32, "bf16",
                n_query=100),
    mi.Workload("dtc_g1_k7", "decode", 1, 200_003, 8, 8, 128, 64, 7, "bf16", n_query=65),
    mi.Workload("dtc_g2_b128", "decode", 1, 400_000, 16, 8, 128, 128, 16, "bf16", n_query=33),
    mi.Workload("dtc_g8_hkv4", "decode", 1, 1_000_000, 32, 4, 128, 64, 32, "bf16", n_query=64),
    mi.Workload("dtc_tiny_bank", "decode", 1, 1000, 32, 8, 128, 64, 32, "bf16", n_query=5),
    # >= 256 chunks of 128 blocks per group: a 1/16 sample pass seeds the thresholds
    mi.Workload("dtc_sampled_2p5m", "decode", 1, 2_500_000, 8, 2, 128, 64, 32, "bf16",
                n_query=40),
]


@pytest.mark.parametrize("w", DECODE_TC, ids=lambda w: w.name)
def test_decode_tc_scan(msa, w):
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    kbar, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    o, lse, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                 kbar_lo=klo)
    torch.cuda.synchronize()
    kbar_np = pool_keys_chunked(kb[None], w.block)[0]
    qs = list(range(w.n_query)) if w.n_query <= 16 else list(range(0, w.n_query, 3))
    check_decode(q, kbar_np, kb, vb, w.block, w.topk, w.scale, idx, o, lse, queries=qs)


@pytest.mark.parametrize("w", DECODE_TC, ids=lambda w: w.name)
def test_decode_tiled_bank_matches_natural_layout(msa, w):
    # the encoded bank changes where the bytes live and how the selection gets there (a
    # certified hi-plane pre-selection, then the three-term scores of the candidates):
    # selection and outputs are bitwise those of the natural layout, which the oracle
    # checks
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    o, lse, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                 kbar_lo=klo)
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    o2, lse2, idx2 = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(o, o2)
    assert torch.equal(lse, lse2)
    if w.name == "dtc_sampled_2p5m":
        kbar_np = pool_keys_chunked(kb[None], w.block)[0]
        check_decode(q, kbar_np, kb, vb, w.block, w.topk, w.scale, idx2, o2, lse2,
                     queries=list(range(0, w.n_query, 5)))


def test_decode_attn_tiled_given_selection(msa):
    # the attention step alone: -1 entries are skipped, an out-of-range entry is skipped
    # and reported, and every other row is the oracle's attention over its given blocks
    w = mi.Workload("dattn", "decode", 1, 80_000, 32, 8, 128, 64, 16, "bf16", n_query=6)
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    p = msa._bank_params(q, w.seq, w.hkv, w.block, w.topk, w.scale)
    ws = msa.workspace(p, msa.OP_DECODE, w.n_query)
    idx = msa.decode_select_tiled(q, bt, w.seq, w.hkv, w.block, w.topk, ws=ws)
    gen = torch.Generator().manual_seed(3)
    given = idx.clone()
    given[0, 0, 5:] = -1                                   # a shorter set, padded
    given[1, 2] = torch.randperm(w.nb, generator=gen)[:w.topk].sort().values.to(given)
    o, lse = msa.decode_attn_tiled(q, kt, vt, given, w.seq, w.hkv, w.block, w.scale, ws=ws)
    torch.cuda.synchronize()
    assert msa.read_device_error(ws) == 0
    kbar_np = pool_keys_chunked(kb[None], w.block)[0]
    Qd = q.float().cpu().numpy()
    gi = given.cpu().numpy()
    override = {(n, g): [int(x) for x in gi[n, g]] for n in range(w.n_query) for g in range(w.hkv)}
    ref = oracle.decode_rows(Qd, kbar_np, HostView(kb), HostView(vb), w.seq, w.block, w.topk,
                             w.scale, idx_override=override)
    G = w.hq // w.hkv
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    for r in ref:
        assert np.abs(og[r.n, r.g * G:(r.g + 1) * G] - r.O).max() <= 2e-2, (r.n, r.g)
        assert np.abs(lg[r.n, r.g * G:(r.g + 1) * G] - r.lse).max() <= 2e-3, (r.n, r.g)
    bad = given.clone()
    bad[3, 1, 0] = w.nb + 7
    o2, _ = msa.decode_attn_tiled(q, kt, vt, bad, w.seq, w.hkv, w.block, w.scale, ws=ws)
    assert msa.read_device_error(ws) & msa.DEVERR_IDX_RANGE
    msa.clear_device_error(ws)
    keep = torch.ones(w.n_query, w.hq, dtype=torch.bool)
    keep[3, G:2 * G] = False
    assert torch.equal(o2[keep], o[keep])


def test_encode_bank_layout(msa):
    # spot-check the documented image layout against the natural tensors
    w = mi.Workload("enc", "decode", 1, 1000, 8, 2, 128, 64, 8, "bf16", n_query=1)
    _, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    ntile = -(-w.seq // 64)
    img = kt.view(torch.bfloat16).view(w.hkv, ntile, 2, 64, 8, 8)   # [g][t][half][row][chunk][8]
    for g, tok, dim in [(0, 0, 0), (1, 5, 77), (0, 999, 127), (1, 640, 8)]:
        t, r = divmod(tok, 64)
        h, c, e = dim // 64, (dim % 64) // 8, dim % 8
        assert img[g, t, h, r, c ^ (r % 8), e].item() == kb[tok, g, dim].item()
    assert int(img[0, ntile - 1, 0, (w.seq % 64):].abs().sum().float().item()) == 0   # rows past S
    nch = -(-w.nb // 128)
    plane = w.hkv * nch * 2 * 128 * 64 * 2
    assert bt.numel() == 2 * plane + 256
    bimg = bt[:2 * plane].view(torch.bfloat16).view(2, w.hkv, nch, 2, 128, 8, 8)
    # the bounds after the planes: max over blocks of ||lo_j||_2 and ||hi_j||_2 per head
    bounds = bt[2 * plane:2 * plane + 8 * w.hkv].view(torch.float32).view(2, w.hkv)
    want = torch.stack([klo.float().norm(dim=-1).amax(dim=0), khi.float().norm(dim=-1).amax(dim=0)])
    torch.testing.assert_close(bounds, want, rtol=1e-6, atol=0)
    for g, j, dim in [(0, 0, 0), (1, 15, 100)]:
        h, c, e, r = dim // 64, (dim % 64) // 8, dim % 8, j % 128
        assert bimg[0, g, j // 128, h, r, c ^ (r % 8), e].item() == khi[j, g, dim].item()
        assert bimg[1, g, j // 128, h, r, c ^ (r % 8), e].item() == klo[j, g, dim].item()


def test_decode_tc_scan_exact_ties(msa):
    # zero queries: every score is exactly 0, so the lowest block indices win
    w = mi.Workload("dtc_ties", "decode", 1, 100_000, 32, 8, 128, 64, 32, "bf16", n_query=4)
    _, kb, vb = mi.decode_inputs(w, device="cuda")
    q = torch.zeros(w.n_query, w.hq, w.d, dtype=torch.bfloat16, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    _, _, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                               kbar_lo=klo)
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda").expand_as(idx)
    assert torch.equal(idx, want)


@pytest.mark.parametrize("seq,hkv", [(250_000, 8), (2_500_000, 2)])
def test_decode_tc_scan_rising_scores(msa, seq, hkv):
    # pooled keys that grow along the bank: for queries aligned with the drift every
    # block beats the running 32nd best, so every chunk refills the candidate lists
    # (the longer bank also runs the sample pass, whose thresholds then lag far behind)
    w = mi.Workload("dtc_rising", "decode", 1, seq, 4 * hkv, hkv, 128, 64, 32, "bf16",
                    n_query=6)
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    u = mi.normal((w.hkv, w.d), 5, mi.STREAM_PLANT, "cuda", torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    ramp = (torch.arange(w.seq, device="cuda", dtype=torch.float32) // w.block) * (8.0 / w.nb)
    kb = (kb.float() + ramp[:, None, None] * u[None]).to(torch.bfloat16)
    q = (q.float() + 0.5 * u.repeat_interleave(w.hq // w.hkv, 0)[None]).to(torch.bfloat16)
    kbar, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    o, lse, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                 kbar_lo=klo)
    torch.cuda.synchronize()
    kbar_np = pool_keys_chunked(kb[None], w.block)[0]
    check_decode(q, kbar_np, kb, vb, w.block, w.topk, w.scale, idx, o, lse)


def test_decode_tc_matches_fp32_scan(msa):
    w = DECODE_TC[1]
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    kbar, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    _, _, i_tc = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                kbar_lo=klo)
    _, _, i_f32 = msa.decode_fwd(q, kbar, kb, vb, w.block, w.topk, w.scale)
    # both exact up to fp32 rounding of near-ties: nearly every row agrees
    agree = (i_tc == i_f32).all(dim=-1).float().mean().item()
    assert agree > 0.95, agree


# ------------------------------------------------------------------ full-size workloads

FULL_PREFILL = ["prefill_tiny_s1k_f32", "prefill_32k_b512_k8", "prefill_128k_b128_k16_planted",
                "prefill_1m_b256_k16"]


@pytest.mark.parametrize("name", FULL_PREFILL)
def test_prefill_full_size_sampled(msa, name):
    w = mi.WORKLOADS[name]
    q, k, v = _inputs(w)
    o, lse, idx = msa.prefill_fwd(q, k, v, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    rows = [(0, t) for t in sample_tokens(w.seq, w.block, 192)]
    rep = {}
    check_prefill(q, k, v, w.block, w.topk, w.scale, idx, o, lse, rows=rows, report=rep)
    print(name, rep)
    # properties at every row: own block present, nothing in the future, ascending
    own = (torch.arange(w.seq, device="cuda") // w.block).view(1, 1, -1)
    sel = idx.long()
    assert bool((sel.max(dim=-1).values == own).all())
    valid = sel >= 0
    assert bool((sel[..., 1:] > sel[..., :-1])[valid[..., 1:]].all())
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("scan", ["tiled", "tc", "fp32"])
def test_decode_full_size_sampled(msa, scan):
    """The 10M-token bank: "tiled" is the path the bench times (encoded bank, the two
    tiled calls), "tc" and "fp32" the natural-layout scans."""
    w = mi.WORKLOADS["decode_bank10m_b64_k32"]
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    kbar, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    if scan == "tiled":
        kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
        del kbar, khi, klo
        torch.cuda.empty_cache()
        idx = msa.decode_select_tiled(q, bt, w.seq, w.hkv, w.block, w.topk)
        o, lse = msa.decode_attn_tiled(q, kt, vt, idx, w.seq, w.hkv, w.block, w.scale)
        del kt, vt, bt
    elif scan == "tc":
        o, lse, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                     kbar_lo=klo)
    else:
        o, lse, idx = msa.decode_fwd(q, kbar, kb, vb, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    kbar_np = pool_keys_chunked(kb[None], w.block, tokens_per_chunk=1 << 21)[0]
    rep = check_decode(q, kbar_np, kb, vb, w.block, w.topk, w.scale, idx, o, lse,
                       queries=list(range(0, w.n_query, 4)))
    print(rep)
