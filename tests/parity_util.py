"""Helpers for GPU-vs-oracle parity tests (test code; imports the oracle, never the reverse).

Comparison rules:
  * selection: rows whose oracle gap between the last taken and the first left-out score
    exceeds 1e-3 relative ("strict" rows) must match the oracle's index list exactly;
    on the other ("tie") rows any valid selection whose every block scores within
    1e-3 relative of the cut is accepted, and its attention output is checked against
    the oracle run on that same selection;
  * outputs: |O_gpu - O_oracle| <= 1e-4 for fp32 inputs, 2e-2 for bf16 inputs;
  * lse: |lse_gpu - lse_oracle| <= 1e-4 (fp32) or 2e-3 (bf16).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

GAP = 1e-3
O_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
LSE_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-3}


class HostView:
    """Read-only numpy view of a (GPU) tensor: indexing copies just the indexed part to
    the host as fp32 (exact for bf16/fp32 values).  Lets the oracle walk full-size
    inputs without materialising them on the host."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, key):
        if not isinstance(key, tuple):
            key = (key,)
        key = tuple(torch.as_tensor(k, device=self.t.device) if isinstance(k, np.ndarray) else k
                    for k in key)
        return self.t[key].float().cpu().numpy()


def pool_keys_chunked(k: torch.Tensor, block: int, tokens_per_chunk: int = 1 << 20) -> np.ndarray:
    """oracle.pool_keys over block-aligned chunks of a large K ([b, S, hkv, d])."""
    b, S, hkv, d = k.shape
    step = max(block, (tokens_per_chunk // block) * block)
    parts = []
    for lo in range(0, S, step):
        parts.append(oracle.pool_keys(k[:, lo:lo + step].float().cpu().numpy(), block))
    return np.concatenate(parts, axis=1)


def sample_tokens(S: int, block: int, n: int, seed: int = 0) -> list[int]:
    """Stratified token sample: first tokens, block edges, the last token, random ones."""
    rng = np.random.default_rng(seed)
    nb = -(-S // block)
    pick = {0, 1, min(S - 1, block - 1), min(S - 1, block), S - 1}
    for j in rng.integers(0, nb, size=n // 4):
        pick.add(int(j * block))
        pick.add(int(min(S - 1, j * block + block - 1)))
    pick.update(int(x) for x in rng.integers(0, S, size=max(0, n - len(pick))))
    return sorted(t for t in pick if 0 <= t < S)


def _valid_prefill_set(sel, i, topk):
    s = [j for j in sel if j >= 0]
    return (i in s and max(s) == i and s == sorted(set(s)) and len(s) == min(topk, i + 1)
            and list(sel[len(s):]) == [-1] * (topk - len(s)))


def check_prefill(q, k, v, block, topk, scale, idx_gpu, o_gpu, lse_gpu, rows=None, kbar=None,
                  report=None):
    """Compares GPU prefill outputs (tensors on any device) with the oracle on `rows`
    ((b, t) pairs; all when None).  Returns a dict of counts; raises AssertionError."""
    dt = q.dtype
    Q, K, V = HostView(q), HostView(k), HostView(v)
    if kbar is None:
        kbar = pool_keys_chunked(k, block)
    bsz, S, hq, d = q.shape
    hkv = k.shape[2]
    G = hq // hkv
    if rows is None:
        rows = [(b, t) for b in range(bsz) for t in range(S)]
    ref = oracle.prefill_rows(Q, K, V, block, topk, scale, rows=rows, kbar=kbar)
    gi = idx_gpu.cpu().numpy()
    override, n_tie, n_strict = {}, 0, 0
    for r in ref:
        sel = [int(x) for x in gi[r.b, r.g, r.t]]
        if r.gap > GAP:
            n_strict += 1
            assert sel == r.idx, f"strict row b={r.b} t={r.t} g={r.g}: gpu {sel} oracle {r.idx}"
        else:
            n_tie += 1
            i = r.t // block
            assert _valid_prefill_set(sel, i, topk), (r.t, r.g, sel)
            qs = oracle.group_query_sum(Q[r.b, r.t], hkv)[r.g]
            cut = r.last_taken - GAP * max(abs(r.last_taken), abs(r.first_left))
            for j in sel:
                if 0 <= j < i:
                    assert float(qs @ kbar[r.b, j, r.g]) >= cut, (r.t, r.g, j)
            if sel != r.idx:
                override[(r.b, r.t, r.g)] = sel
    if override:
        keys = sorted({(b, t) for (b, t, g) in override})
        redo = oracle.prefill_rows(Q, K, V, block, topk, scale, rows=keys, kbar=kbar,
                                   idx_override=override)
        rmap = {(r.b, r.t, r.g): r for r in redo}
        ref = [rmap.get((r.b, r.t, r.g), r) for r in ref]
    max_err = max_lse = 0.0
    bt = sorted({(r.b, r.t) for r in ref})
    bi = torch.tensor([x[0] for x in bt], device=o_gpu.device)
    ti = torch.tensor([x[1] for x in bt], device=o_gpu.device)
    og = o_gpu[bi, ti].float().cpu().numpy()                       # [n, hq, d]
    lg = lse_gpu[bi, :, ti].float().cpu().numpy() if lse_gpu is not None else None
    pos = {x: n for n, x in enumerate(bt)}
    for r in ref:
        n = pos[(r.b, r.t)]
        err = np.abs(og[n, r.g * G:(r.g + 1) * G] - r.O).max()
        max_err = max(max_err, float(err))
        if lg is not None:
            max_lse = max(max_lse, float(np.abs(lg[n, r.g * G:(r.g + 1) * G] - r.lse).max()))
    out = dict(rows=len(ref), strict=n_strict, tie=n_tie, overridden=len(override),
               max_abs_err=max_err, max_lse_err=max_lse)
    if report is not None:
        report.update(out)
    assert max_err <= O_TOL[dt], out
    assert max_lse <= LSE_TOL[dt], out
    return out


def check_decode(q, kbar_np, k_bank, v_bank, block, topk, scale, idx_gpu, o_gpu, lse_gpu,
                 queries=None):
    dt = q.dtype
    Qd = q.float().cpu().numpy()
    S, hkv, d = k_bank.shape
    hq = q.shape[1]
    G = hq // hkv
    K, V = HostView(k_bank), HostView(v_bank)
    ref = oracle.decode_rows(Qd, kbar_np, K, V, S, block, topk, scale, queries=queries)
    gi = idx_gpu.cpu().numpy()
    override, n_tie = {}, 0
    for r in ref:
        sel = [int(x) for x in gi[r.n, r.g]]
        if r.gap > GAP:
            assert sel == r.idx, f"strict decode row n={r.n} g={r.g}: gpu {sel} oracle {r.idx}"
        else:
            n_tie += 1
            s = [j for j in sel if j >= 0]
            assert s == sorted(set(s)) and len(s) == min(topk, kbar_np.shape[0])
            qs = oracle.group_query_sum(Qd[r.n], hkv)[r.g]
            cut = r.last_taken - GAP * max(abs(r.last_taken), abs(r.first_left))
            for j in s:
                assert float(qs @ kbar_np[j, r.g]) >= cut
            if sel != r.idx:
                override[(r.n, r.g)] = sel
    if override:
        ns = sorted({n for (n, g) in override})
        redo = oracle.decode_rows(Qd, kbar_np, K, V, S, block, topk, scale, queries=ns,
                                  idx_override=override)
        rmap = {(r.n, r.g): r for r in redo}
        ref = [rmap.get((r.n, r.g), r) for r in ref]
    og = o_gpu.float().cpu().numpy()
    lg = lse_gpu.float().cpu().numpy() if lse_gpu is not None else None
    max_err = max_lse = 0.0
    for r in ref:
        max_err = max(max_err, float(np.abs(og[r.n, r.g * G:(r.g + 1) * G] - r.O).max()))
        if lg is not None:
            max_lse = max(max_lse, float(np.abs(lg[r.n, r.g * G:(r.g + 1) * G] - r.lse).max()))
    out = dict(rows=len(ref), tie=n_tie, overridden=len(override), max_abs_err=max_err,
               max_lse_err=max_lse)
    assert max_err <= O_TOL[dt], out
    assert max_lse <= LSE_TOL[dt], out
    return out
