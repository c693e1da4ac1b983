"""Seeded synthetic inputs for block-sparse top-k attention, and the workload shapes.

This module is shared by the CUDA path's tests/bench and by the CPU oracle. It holds
no arithmetic of the method itself (no pooling, scoring, selection or attention): it
only draws i.i.d. N(0,1) tensors from a counter-based generator and, for the planted
workload, adds a fixed shift so that block selection is non-uniform.

Generator (one published definition, evaluated with plain integer / fp64 tensor ops):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014): state_n = base + n * 0x9E3779B97F4A7C15 (mod 2^64), output_n =
    mix64(state_n) with the finaliser z ^= z>>>30; z *= 0xBF58476D1CE4E5B9;
    z ^= z>>>27; z *= 0x94D049BB133111EB; z ^= z>>>31.
  * base(seed, stream) = mix64(mix64(seed) XOR stream), one stream per tensor.
  * element i of a tensor (row-major flat index) takes outputs n = 2i+1 and n = 2i+2:
    u1 = ((out >>> 11) + 1) * 2^-53 in (0, 1], u2 = (out >>> 11) * 2^-53 in [0, 1),
    x = sqrt(-2 ln u1) * cos(2 pi u2)   (Box-Muller, in fp64).
  * x is rounded fp64 -> fp32 (RNE) and, for bf16 tensors, fp32 -> bf16 (RNE).
Any element depends only on (seed, stream, i), so a tensor can be generated in chunks
on any device.  The last bits of log/cos may differ between CPU and CUDA libraries, so
a consumer never regenerates a tensor on another device: the oracle reads a host copy
of the very tensor the GPU path consumed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "LazyBank", "lazy_decode_bank",
    "Workload", "WORKLOADS", "normal", "planted_blocks", "planted_directions",
    "prefill_inputs", "decode_inputs", "normal_rows", "decode_bank_rows", "doc_lengths",
    "cu_seqlens", "STREAM_Q", "STREAM_K", "STREAM_V",
    "STREAM_U", "STREAM_PLANT", "STREAM_DECODE_Q",
]

STREAM_Q, STREAM_K, STREAM_V, STREAM_U, STREAM_PLANT, STREAM_DECODE_Q = 1, 2, 3, 4, 5, 6

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _signed(x: int) -> int:
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z ^= z >> 30
    z = (z * _M1) & _MASK64
    z ^= z >> 27
    z = (z * _M2) & _MASK64
    z ^= z >> 31
    return z


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns (torch's >> is arithmetic)."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64_t(z: torch.Tensor) -> torch.Tensor:
    z = z ^ _srl(z, 30)
    z = z * _signed(_M1)
    z = z ^ _srl(z, 27)
    z = z * _signed(_M2)
    z = z ^ _srl(z, 31)
    return z


def stream_base(seed: int, stream: int) -> int:
    return _mix64_int(_mix64_int(seed + _GAMMA) ^ stream)


def _normal_chunk(base: int, start: int, count: int, device) -> torch.Tensor:
    return _normal_idx(base, torch.arange(start, start + count, dtype=torch.int64, device=device))


def _normal_idx(base: int, i: torch.Tensor) -> torch.Tensor:
    g = _signed(_GAMMA)
    b = _signed(base)
    a = _mix64_t(b + (2 * i + 1) * g)
    c = _mix64_t(b + (2 * i + 2) * g)
    u1 = (_srl(a, 11) + 1).to(torch.float64) * (2.0 ** -53)
    u2 = _srl(c, 11).to(torch.float64) * (2.0 ** -53)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


_CHUNK = 1 << 24


def normal(shape, seed: int, stream: int, device="cpu", dtype=torch.float32,
           shift=None) -> torch.Tensor:
    """i.i.d. N(0,1) tensor of `shape`; element i from the counter-based generator.

    `shift`, if given, is called as shift(x_fp64_chunk, flat_start) and returns the
    fp64 chunk with a deterministic offset added before rounding (planted workload).
    """
    shape = tuple(int(s) for s in shape)
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=dtype, device=device)
    base = stream_base(seed, stream)
    for start in range(0, n, _CHUNK):
        cnt = min(_CHUNK, n - start)
        x = _normal_chunk(base, start, cnt, device)
        if shift is not None:
            x = shift(x, start)
        out[start:start + cnt] = x.to(torch.float32).to(dtype)
    return out.view(shape)


def normal_rows(shape, row_lo: int, row_hi: int, seed: int, stream: int, device="cpu",
                dtype=torch.float32) -> torch.Tensor:
    """Rows [row_lo, row_hi) along the first axis of normal(shape, seed, stream, ...),
    generated alone (the same values: element i depends only on its flat index)."""
    shape = tuple(int(s) for s in shape)
    row = 1
    for s in shape[1:]:
        row *= s
    n = (row_hi - row_lo) * row
    out = torch.empty(n, dtype=dtype, device=device)
    base = stream_base(seed, stream)
    for start in range(0, n, _CHUNK):
        cnt = min(_CHUNK, n - start)
        out[start:start + cnt] = _normal_chunk(base, row_lo * row + start, cnt,
                                               device).to(torch.float32).to(dtype)
    return out.view((row_hi - row_lo,) + shape[1:])


def decode_bank_rows(w: "Workload", lo: int, hi: int, device="cpu", seed: int = 0):
    """Tokens [lo, hi) of the bank K and V of decode_inputs(w, seed=seed)."""
    dt = w.torch_dtype
    shape = (w.seq, w.hkv, w.d)
    return (normal_rows(shape, lo, hi, seed, STREAM_K, device, dt),
            normal_rows(shape, lo, hi, seed, STREAM_V, device, dt))


class LazyBank:
    """The bank tensor normal((S, hkv, d), seed, stream) of a decode workload, generated on
    demand: bank[p, g] returns the rows p (index array) of head g as fp32 numpy values of
    the `dtype`-rounded elements, identical to the materialised tensor's.  Lets host-side
    code read a few selected blocks of a 10M-token bank without building 20 GB."""

    def __init__(self, shape, seed: int, stream: int, dtype=torch.bfloat16):
        self.shape = tuple(int(s) for s in shape)
        self.base = stream_base(seed, stream)
        self.dtype = dtype

    def __getitem__(self, key):
        p, g = key
        S, hkv, d = self.shape
        p = torch.as_tensor(np.asarray(p), dtype=torch.int64).reshape(-1)
        flat = (p[:, None] * hkv + int(g)) * d + torch.arange(d, dtype=torch.int64)[None, :]
        x = _normal_idx(self.base, flat.reshape(-1)).to(torch.float32).to(self.dtype)
        return x.float().reshape(len(p), d).numpy()


def lazy_decode_bank(w: "Workload", seed: int = 0):
    """(K, V) of decode_inputs(w, seed=seed) as LazyBank views."""
    return (LazyBank((w.seq, w.hkv, w.d), seed, STREAM_K, w.torch_dtype),
            LazyBank((w.seq, w.hkv, w.d), seed, STREAM_V, w.torch_dtype))


@dataclass(frozen=True)
class Workload:
    """Shapes of one synthetic workload.

    prefill: Q [batch, seq, hq, d], K/V [batch, seq, hkv, d].
    decode:  Q [n_query, hq, d] against a bank K/V [seq, hkv, d] (seq = bank tokens).
    """
    name: str
    kind: str
    batch: int
    seq: int
    hq: int
    hkv: int
    d: int
    block: int
    topk: int
    dtype: str
    n_query: int = 0
    planted_frac: float = 0.0
    planted_shift: float = 0.0
    n_docs: int = 0            # packed documents (kind "prefill_docs")
    rope_base: float = 0.0     # document-wise RoPE base (kind "prefill_docs")
    host_bank: bool = False    # decode bank content in pinned host memory
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def nb(self) -> int:
        return -(-self.seq // self.block)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    w.name: w for w in [
        Workload("prefill_tiny_s1k_f32", "prefill", 1, 1024, 2, 1, 64, 64, 4, "f32",
                 note="tiny causal prefill, fp32, 16 blocks of 64, top-4"),
        Workload("prefill_32k_b512_k8", "prefill", 1, 32768, 32, 8, 128, 512, 8, "bf16",
                 note="causal prefill bf16, 64 blocks of 512, top-8"),
        Workload("prefill_128k_b128_k16_planted", "prefill", 1, 131072, 32, 8, 128, 128, 16,
                 "bf16", planted_frac=0.01, planted_shift=3.0,
                 note="causal prefill bf16, 1024 blocks of 128, top-16, 1% planted blocks"),
        Workload("prefill_1m_b256_k16", "prefill", 1, 1048576, 32, 8, 128, 256, 16, "bf16",
                 note="causal prefill bf16, 4096 blocks of 256, top-16"),
        Workload("decode_bank10m_b64_k32", "decode", 1, 10_000_000, 32, 8, 128, 64, 32, "bf16",
                 n_query=64,
                 note="64 decode queries against a 10M-token bank, 156250 blocks of 64, top-32"),
        Workload("decode_bank10m_b64_k32_hostbank", "decode", 1, 10_000_000, 32, 8, 128, 64, 32,
                 "bf16", n_query=64, host_bank=True,
                 note="the 10M-token decode with the bank's K/V in pinned host memory"),
        Workload("prefill_1m_b256_k16_bwd", "prefill_bwd", 1, 1048576, 32, 8, 128, 256, 16,
                 "bf16", note="backward of the 1M causal prefill's sparse attention"),
        Workload("prefill_128k_b128_k16_planted_bwd", "prefill_bwd", 1, 131072, 32, 8, 128, 128,
                 16, "bf16", planted_frac=0.01, planted_shift=3.0,
                 note="backward of the 128K planted prefill's sparse attention"),
        Workload("prefill_docs_1m_b256_k16_rope", "prefill_docs", 1, 1048576, 32, 8, 128, 256,
                 16, "bf16", n_docs=64, rope_base=1_000_000.0,
                 note="1M packed tokens in 64 documents (log-uniform lengths 2K-64K), "
                      "document-wise RoPE, each document its own causal prefill"),
    ]
}


def doc_lengths(total: int, n_docs: int, seed: int = 0, lo: int = 2048, hi: int = 65536):
    """n_docs document lengths summing to `total`: log-uniform draws in [lo, hi] from a
    seeded numpy generator, scaled to the total (the last one takes the rounding)."""
    rng = np.random.default_rng(seed + 1000)
    x = np.exp(rng.uniform(math.log(lo), math.log(hi), n_docs))
    n = np.floor(x / x.sum() * total).astype(np.int64)
    n = np.maximum(n, 1)
    n[-1] = total - n[:-1].sum()
    assert n[-1] >= 1
    return [int(v) for v in n]


def cu_seqlens(lengths) -> list[int]:
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return out


def planted_blocks(nb: int, frac: float, seed: int) -> list[int]:
    """floor(frac*nb) distinct block ids: the blocks with the smallest stream-5 draws."""
    n = int(math.floor(frac * nb))
    base = stream_base(seed, STREAM_PLANT)
    keyed = sorted((_mix64_int(base + (j + 1) * _GAMMA), j) for j in range(nb))
    return sorted(j for _, j in keyed[:n])


def planted_directions(hkv: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    """One unit vector per KV head, fp64 [hkv, d] (a normalised stream-4 Gaussian)."""
    base = stream_base(seed, STREAM_U)
    u = _normal_chunk(base, 0, hkv * d, device).view(hkv, d)
    return u / torch.linalg.vector_norm(u, dim=1, keepdim=True)


def prefill_inputs(w: Workload, device="cpu", seed: int = 0):
    """Q, K, V for a prefill workload, in the workload's dtype, on `device` (packed
    documents: the batch-1 tensors of all their tokens)."""
    assert w.kind in ("prefill", "prefill_docs", "prefill_bwd")
    b, s, hq, hkv, d = w.batch, w.seq, w.hq, w.hkv, w.d
    dt = w.torch_dtype
    qshift = kshift = None
    if w.planted_frac > 0:
        g_size = hq // hkv
        u = planted_directions(hkv, d, seed, device) * w.planted_shift      # [hkv, d]
        uq = u.repeat_interleave(g_size, dim=0).reshape(-1)                  # [hq*d]
        mark = torch.zeros(w.nb, dtype=torch.bool, device=device)
        pl = planted_blocks(w.nb, w.planted_frac, seed)
        if pl:
            mark[torch.tensor(pl, device=device)] = True
        uk = u.reshape(-1)                                                   # [hkv*d]

        def qshift(x, start):
            pos = torch.arange(start, start + x.numel(), device=device) % (hq * d)
            return x + uq[pos]

        def kshift(x, start):
            flat = torch.arange(start, start + x.numel(), device=device)
            tok = (flat // (hkv * d)) % s
            hit = mark[tok // w.block]
            return x + torch.where(hit, uk[flat % (hkv * d)], torch.zeros((), dtype=x.dtype,
                                                                          device=device))
    q = normal((b, s, hq, d), seed, STREAM_Q, device, dt, qshift)
    k = normal((b, s, hkv, d), seed, STREAM_K, device, dt, kshift)
    v = normal((b, s, hkv, d), seed, STREAM_V, device, dt)
    return q, k, v


def decode_inputs(w: Workload, device="cpu", seed: int = 0, bank: bool = True):
    """Decode queries [n_query, hq, d] and (optionally) the bank K/V [seq, hkv, d]."""
    assert w.kind == "decode"
    dt = w.torch_dtype
    q = normal((w.n_query, w.hq, w.d), seed, STREAM_DECODE_Q, device, dt)
    if not bank:
        return q, None, None
    k = normal((w.seq, w.hkv, w.d), seed, STREAM_K, device, dt)
    v = normal((w.seq, w.hkv, w.d), seed, STREAM_V, device, dt)
    return q, k, v
