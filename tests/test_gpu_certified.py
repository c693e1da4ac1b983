"""The certified selection of an encoded bank (banks of at least ~8.4M tokens at block
64, where the sample pass bounds the hi-plane filter tightly): a hi-plane scan proposes
64 candidates per (query, group), the candidates are scored with the three-term split
product, and each row's result is accepted only when the bound on the dropped lo-plane
term shows that no other block can reach its top k; otherwise the whole bank is scanned
exactly.  Either way the selection must be bitwise that of the natural-layout scan.
The 10M-token cases below make the certificate fail (all rows, or some groups' rows) or
the filter overflow, so that the exact rescan is the path that decides; smaller banks
take the exact scan directly and are checked the same way."""
import pytest
import torch

import msa_inputs as mi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import block_sparse_top_mean_b200 as m
    from block_sparse_top_mean_b200 import build
    build.build()
    return m


def _both(msa, w, q, kb, vb, khi, klo):
    o, lse, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                 kbar_lo=klo)
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    o2, lse2, idx2 = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk, w.scale)
    torch.cuda.synchronize()
    return (o, lse, idx), (o2, lse2, idx2)


def test_exact_ties_take_lowest_blocks(msa):
    # zero queries: every score is exactly 0, no row can be certified (a zero-width
    # bound cannot separate equal scores), and the exact rescan picks the lowest blocks
    w = mi.Workload("cert_ties", "decode", 1, 300_000, 32, 8, 128, 64, 32, "bf16", n_query=4)
    _, kb, vb = mi.decode_inputs(w, device="cuda")
    q = torch.zeros(w.n_query, w.hq, w.d, dtype=torch.bfloat16, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    _, _, idx = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk, w.scale)
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda").expand_as(idx)
    assert torch.equal(idx, want)


@pytest.mark.parametrize("groups", ["all", "half"])
def test_equal_hi_planes_fall_back_to_the_exact_scan(msa, groups):
    # planes whose hi rows are one row repeated: the hi-plane scores of a group are all
    # equal, its candidates are arbitrary and only the lo plane orders the blocks, so
    # those rows fail the certificate ("half": the other group keeps its own planes and
    # certifies)
    w = mi.Workload("cert_hi", "decode", 1, 10_000_000, 8, 2, 128, 64, 32, "bf16", n_query=20)
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    sel = slice(None) if groups == "all" else slice(0, 1)
    khi[:, sel] = khi[:1, sel]
    a, b = _both(msa, w, q, kb, vb, khi, klo)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("seq,hkv", [(250_000, 8), (2_500_000, 2)])
def test_rising_scores(msa, seq, hkv):
    # pooled keys that grow along the bank (every chunk refills the candidate lists,
    # and the sample thresholds lag far behind): still the natural-layout selection
    w = mi.Workload("cert_rising", "decode", 1, seq, 4 * hkv, hkv, 128, 64, 32, "bf16",
                    n_query=6)
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    u = mi.normal((w.hkv, w.d), 5, mi.STREAM_PLANT, "cuda", torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    ramp = (torch.arange(w.seq, device="cuda", dtype=torch.float32) // w.block) * (8.0 / w.nb)
    kb = (kb.float() + ramp[:, None, None] * u[None]).to(torch.bfloat16)
    q = (q.float() + 0.5 * u.repeat_interleave(w.hq // w.hkv, 0)[None]).to(torch.bfloat16)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    a, b = _both(msa, w, q, kb, vb, khi, klo)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_repeated_calls_reset_the_fallback(msa):
    # a failing call, then a certifying one on the same workspace, then the failing one
    # again: each gives the natural-layout selection
    w = mi.Workload("cert_seq", "decode", 1, 10_000_000, 4, 1, 128, 64, 32, "bf16", n_query=8)
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    p = msa._bank_params(q, w.seq, w.hkv, w.block, w.topk, w.scale)
    ws = msa.workspace(p, msa.OP_DECODE, w.n_query, device=q.device)
    zero = torch.zeros_like(q)
    for qq in (zero, q, zero):
        _, _, i_nat = msa.decode_fwd(qq, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                                     kbar_lo=klo)
        _, _, i_t = msa.decode_fwd_tiled(qq, bt, kt, vt, w.seq, w.hkv, w.block, w.topk, w.scale,
                                         ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(i_nat, i_t)


# One KV head keeps these 10M-token banks small.
FILTER_BANK = mi.Workload("cert_filter_10m", "decode", 1, 10_000_000, 4, 1, 128, 64, 32, "bf16",
                          n_query=8)


def test_filtered_scan_exact_ties_overflow_to_the_exact_scan(msa):
    # zero queries: every block reaches the bound, the rows' buffers overflow, and the
    # list scan of the whole bank decides: the lowest blocks
    w = FILTER_BANK
    _, kb, vb = mi.decode_inputs(w, device="cuda")
    q = torch.zeros(w.n_query, w.hq, w.d, dtype=torch.bfloat16, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    want = torch.arange(w.topk, dtype=torch.int32, device="cuda").expand(w.n_query, w.hkv, w.topk)
    _, _, idx = msa.decode_fwd(q, None, kb, vb, w.block, w.topk, w.scale, kbar_hi=khi,
                               kbar_lo=klo)
    assert torch.equal(idx, want)
    kt, vt, bt = msa.encode_bank(kb, vb, khi, klo, w.block)
    _, _, idx = msa.decode_fwd_tiled(q, bt, kt, vt, w.seq, w.hkv, w.block, w.topk, w.scale)
    assert torch.equal(idx, want)


def test_filtered_scan_rising_scores(msa):
    w = FILTER_BANK
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    u = mi.normal((w.hkv, w.d), 5, mi.STREAM_PLANT, "cuda", torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    ramp = (torch.arange(w.seq, device="cuda", dtype=torch.float32) // w.block) * (8.0 / w.nb)
    kb = (kb.float() + ramp[:, None, None] * u[None]).to(torch.bfloat16)
    del ramp
    q = (q.float() + 0.5 * u.repeat_interleave(w.hq // w.hkv, 0)[None]).to(torch.bfloat16)
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    a, b = _both(msa, w, q, kb, vb, khi, klo)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_near_ties_at_the_cut_fail_the_certificate(msa):
    # 100 blocks with one and the same hi row, pointing along the queries' mean: they
    # top every row's hi-plane scores with equal values, so a row's 64 candidates are
    # some of them and only the lo plane orders them; the bound cannot separate the k-th
    # best from the blocks left out, the rows fail, and the exact rescan decides
    w = FILTER_BANK
    q, kb, vb = mi.decode_inputs(w, device="cuda")
    _, khi, klo = (t[0] for t in msa.pool_keys(kb[None], w.block, split=True))
    qs = q.float().view(w.n_query, w.hkv, -1, w.d).sum(dim=2)[:, 0]     # group-summed
    u = qs.mean(dim=0)
    u = u / u.norm()
    khi[1000:1100, 0] = (3.0 * khi[:, 0].float().norm(dim=-1).mean() * u).to(torch.bfloat16)
    a, b = _both(msa, w, q, kb, vb, khi, klo)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    sel = b[2]
    assert bool(((sel >= 1000) & (sel < 1100)).all())      # the planted blocks win
