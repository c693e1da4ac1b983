#!/usr/bin/env python
"""Benchmark of the block-sparse top-k attention hot path on B200; prints ONE JSON line.

A step is one pass of the whole hot path over one synthetic sequence resident in HBM:
pool keys -> fused block scoring + top-k -> sparse attention, each through the C ABI.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent sequence
(weak scaling, no collective on the data path); the time is the max over ranks and
`value` counts the work of all ranks.  `--impl reference` times the fp64 CPU oracle on
a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import msa_inputs as mi  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ workload arithmetic

def prefill_flops(w: mi.Workload) -> tuple[float, float]:
    """(attention FLOPs, scoring FLOPs) of one causal prefill pass, as the method counts
    them: 4*d per (query head, attended key) and 2*d per (token, group, past block)."""
    t = np.arange(w.seq, dtype=np.int64)
    i = t // w.block
    keys = (np.minimum(w.topk, i + 1) - 1) * w.block + (t - i * w.block + 1)
    attn = float(keys.sum()) * w.hq * 4 * w.d * w.batch
    score = float(i.sum()) * w.hkv * 2 * w.d * w.batch
    return attn, score


def decode_work(w: mi.Workload) -> dict:
    nb = w.nb
    full = min(w.topk, nb) * w.block
    return dict(
        attn_flops=float(w.n_query * w.hq * 4 * w.d * full),
        score_flops=float(w.n_query * w.hkv * 2 * w.d * nb),
        # bytes the two phases must read at least: the pooled-key bank once (as bf16), and
        # the selected K/V blocks once per (query, group)
        score_bytes=float(nb * w.hkv * w.d * 2),
        attn_bytes=float(w.n_query * w.hkv * full * w.d * 2 * 2),
    )


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

CLOCK_Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
           "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
           "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """Samples SM clock, power and clock-event reasons of one GPU while the timed region
    runs: NVML from a host thread every 2 ms (short regions such as a decode step get
    samples too), else nvidia-smi every 200 ms.  Reads only; changes no setting."""

    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.thread = None
        self.rows = []
        self.path = os.path.join("/tmp", f"msa_clocks_{os.getpid()}.csv")

    def _nvml_loop(self, nv, h):
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((float(sm), float(mx), pw,
                                  [name for bit, name in self.REASONS.items() if rs & bit]))
            except Exception:  # noqa: BLE001 - sampling is best effort
                pass
            self.stop.wait(0.002)

    def __enter__(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:  # noqa: BLE001 - fall back to nvidia-smi
            self.thread = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    self.rows.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                      [names[k] for k, x in enumerate(parts[5:9])
                                       if x.lower().startswith("active")]))
                except ValueError:
                    continue

    def summary(self):
        rows = self.rows
        if not rows:
            return None
        reasons = sorted({n for r in rows for n in r[3]})
        busy = [r[0] for r in rows if r[2] > 300.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": round(max(r[2] for r in rows), 1),
                "source": "nvml 2 ms" if self.thread is not None else "nvidia-smi 200 ms"}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our implementation

class PrefillRunner:
    """Holds device buffers and issues one step through the C ABI."""

    def __init__(self, w: mi.Workload, seed: int):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        self.q, self.k, self.v = mi.prefill_inputs(w, device="cuda", seed=seed)
        dev = self.q.device
        self.p = msa.params(batch=w.batch, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                            topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.kbar = torch.empty(w.batch, w.nb, w.hkv, w.d, dtype=torch.float32, device=dev)
        # bf16 hi/lo planes of the pooled keys feed the tensor-core selection
        self.khi = torch.empty(w.batch, w.nb, w.hkv, w.d, dtype=torch.bfloat16, device=dev)
        self.klo = torch.empty_like(self.khi)
        self.idx = torch.empty(w.batch, w.hkv, w.seq, w.topk, dtype=torch.int32, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(w.batch, w.hq, w.seq, dtype=torch.float32, device=dev)
        n = max(self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_TOPK_SELECT, 0),
                self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_SPARSE_ATTN, 0))
        self.ws = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.check = _lib.check
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        self.ptr = {k: P(getattr(self, k)) for k in ("q", "k", "v", "kbar", "khi", "klo", "idx", "o",
                                                     "lse", "ws")}
        self.pp = ctypes.byref(self.p)
        # own kernels per step (memsets excluded): pool 1; selection: tensor-core pass +
        # exact pass over flagged tiles = 2; attention, per token slab: count, scan, fill,
        # tile table, tiles, merge = 6
        slab = msa.attn_slab_tokens(self.p, _lib.OP_SPARSE_ATTN, n)
        self.n_slabs = -(-w.seq // slab)
        self.launches_per_step = 3 + 6 * self.n_slabs

    def step(self, events=None):
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        P, lib = self.ptr, self.lib
        if events:
            events[0].record()
        self.check("msa_pool_keys", lib.msa_pool_keys(self.pp, P["k"], P["kbar"], P["khi"],
                                                      P["klo"], s))
        if events:
            events[1].record()
        self.check("msa_topk_select", lib.msa_topk_select(
            self.pp, P["q"], P["kbar"], P["khi"], P["klo"], P["idx"], P["ws"], self.ws.numel(),
            s))
        if events:
            events[2].record()
        self.check("msa_sparse_attn_fwd", lib.msa_sparse_attn_fwd(
            self.pp, P["q"], P["k"], P["v"], P["idx"], P["o"], P["lse"], P["ws"],
            self.ws.numel(), s))
        if events:
            events[3].record()


class DecodeRunner:
    """Decode of n_query queries against a bank resident in HBM, through the C ABI.  The
    bank's pooled keys are computed once up front (offline encoding, not timed)."""

    def __init__(self, w: mi.Workload, seed: int):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        self.q, self.k, self.v = mi.decode_inputs(w, device="cuda", seed=seed)
        # offline bank preparation (not timed): the routing keys as bf16 hi/lo planes, then
        # the encoded images the decode kernels stream with one bulk copy per tile
        _, khi, klo = (t[0] for t in msa.pool_keys(self.k[None], w.block, split=True))
        self.kt, self.vt, self.bt = msa.encode_bank(self.k, self.v, khi, klo, w.block)
        del khi, klo                            # the step reads only the encoded bank
        dev = self.q.device
        self.p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                            topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(w.n_query, w.hq, dtype=torch.float32, device=dev)
        self.idx = torch.empty(w.n_query, w.hkv, w.topk, dtype=torch.int32, device=dev)
        n = self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_DECODE, w.n_query)
        self.ws = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.check = _lib.check
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        self.ptr = {k: P(getattr(self, k)) for k in ("q", "kt", "vt", "bt", "idx", "o", "lse",
                                                     "ws")}
        self.pp = ctypes.byref(self.p)
        # own kernels per step: sample scan, sample threshold, bank scan, list merge,
        # attention, combine
        self.launches_per_step = 6

    def step(self, events=None):
        # msa_decode_fwd_tiled as its two calls, so the phases can be timed apart
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        P, w = self.ptr, self.w
        if events:
            events[0].record()
        self.check("msa_decode_select_tiled", self.lib.msa_decode_select_tiled(
            self.pp, w.n_query, P["q"], P["bt"], P["idx"], P["ws"], self.ws.numel(), s))
        if events:
            events[1].record()
        self.check("msa_decode_attn_tiled", self.lib.msa_decode_attn_tiled(
            self.pp, w.n_query, P["q"], P["kt"], P["vt"], P["idx"], P["o"], P["lse"], P["ws"],
            self.ws.numel(), s))
        if events:
            events[2].record()


def run_decode(args, world, rank, local):
    w = workload_of(args)
    from block_sparse_top_mean_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    r = DecodeRunner(w, seed=rank)
    work = decode_work(w)
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the bank (41 GB) is far larger than L2; the pooled keys (0.6 GB) too
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        start.record()
        for i in range(args.steps):
            r.step(ev[i])
        end.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, world)
    peaks, peak_src = load_peaks()
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    # algorithmic bytes: the selection reads the pooled-key bank once at 4 bytes per element
    # (bf16 hi + lo planes, as exact as fp32 for the selection); the attention reads the
    # selected K/V blocks once per (query, group)
    kbar_bytes = float(w.nb * w.hkv * w.d * 4)
    phases = {
        "select": {"ms": sel_ms, "bytes": kbar_bytes,
                   "kernel": "msa_decode_select_tiled (sample scan + threshold + full "
                             "tensor-core scan + list merge)",
                   # DRAM bytes of its scan kernels in one ncu capture of a 1.2M-token bank
                   # (sample 10.5 MB + scan 79.5 MB for 18,750 blocks), scaled by blocks
                   "traffic": (10.52e6 + 79.46e6) * w.nb / 18750},
        "attend": {"ms": att_ms, "bytes": float(work["attn_bytes"]),
                   "kernel": "msa_decode_attn_tiled (streamed attention + split combine)",
                   # the attention kernel's DRAM bytes in the same capture (526.3 MB read,
                   # 16.8 MB written); they depend on the selection, not on the bank size
                   "traffic": 543.09e6 * w.n_query * w.hkv * w.topk / (64 * 8 * 32)},
    }
    dom = max(phases.values(), key=lambda x: x["ms"])
    gbs = dom["bytes"] / (dom["ms"] * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": dom["kernel"], "achieved": round(gbs, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
            "peak_source": f"hbm_gbs of {peak_src}", "traffic": round(dom["traffic"]),
            "traffic_source": "ncu capture of a 1.2M-token bank, scaled (see profiles/)",
            "algorithmic_per_launch": dom["bytes"]}
    phase_line = {k: {"us": round(v["ms"] * 1e3, 1),
                      "gbs": round(v["bytes"] / (v["ms"] * 1e-3) / 1e9, 1)} for k, v in phases.items()}
    e2e = None
    if not args.no_e2e:
        hq_ = r.q.cpu().pin_memory()
        ho = torch.empty(r.o.shape, dtype=r.o.dtype).pin_memory()

        def one():
            r.q.copy_(hq_, non_blocking=True)
            r.step()
            ho.copy_(r.o, non_blocking=True)
        for _ in range(args.warmup):
            one()
        torch.cuda.synchronize()
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_.record()
        for _ in range(args.steps):
            one()
        e_.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(s_.elapsed_time(e_) / args.steps, world)
        e2e = {"value": round(ems * 1e3, 1), "unit": "us/step", "ms_per_step": round(ems, 4),
               "h2d_bytes_per_step": hq_.numel() * hq_.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size()}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_decode(w, r.q, seed=rank)
    line = {
        "metric": "decode us/step", "value": round(ms * 1e3, 1), "unit": "us/step",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "l2": "bank and pooled keys larger than L2, no flush",
                   "parallelism": f"{world} independent banks, one per GPU"},
        "phases": phase_line, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clk.summary(),
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    w = workload_of(args)
    if w.kind != "prefill":
        return run_decode(args, world, rank, local)
    from block_sparse_top_mean_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    r = PrefillRunner(w, seed=rank)
    attn_flops, score_flops = prefill_flops(w)
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()

    # device-timed region: K steps, inputs resident in HBM (Q alone is larger than L2)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        start.record()
        for i in range(args.steps):
            r.step(ev[i])
        end.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = start.elapsed_time(end) / args.steps
    ms_max = max_over_ranks(ms, world)
    phase = {n: statistics.mean(e[a].elapsed_time(e[a + 1]) for e in ev)
             for a, n in enumerate(["pool_keys", "topk_select", "sparse_attn"])}
    err = r.msa.read_device_error(r.ws)

    peaks, peak_src = load_peaks()
    value = world * (attn_flops + score_flops) / (ms_max * 1e-3) / 1e12
    tokens_s = world * w.seq * w.batch / (ms_max * 1e-3)
    attn_tflops = attn_flops / (phase["sparse_attn"] * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    roof = {"bound": "tensor", "kernel": "sparse_attn", "achieved": round(attn_tflops, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(attn_tflops / peak, 4),
            "peak_source": f"bf16_tflops_sustained of {peak_src}", "traffic": None,
            "algorithmic_per_launch": attn_flops}

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(r, args, world, attn_flops + score_flops)
    cpu = None
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        cpu = cpu_baseline_prefill(w, r, attn_flops + score_flops)

    line = {
        "metric": "sparse-attn prefill TFLOP/s", "value": round(value, 3), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "seq": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "l2": f"inputs larger than L2 (Q alone {w.batch * w.seq * w.hq * w.d * 2 / 2**30:.2f} GiB), no flush",
                   "workspace_gib": round(r.ws.numel() / 2**30, 2),
                   "attn_token_slabs": r.n_slabs,
                   "parallelism": f"{world} independent sequences, one per GPU"},
        "tokens_per_s": round(tokens_s, 1),
        "flops_per_step": {"attention": attn_flops, "scoring": score_flops},
        "phases_ms": {k: round(v, 3) for k, v in phase.items()},
        "attn_phase_tflops": round(attn_tflops, 2),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": r.launches_per_step * args.steps,
        "clocks": clk.summary(),
        "device_error_bits": err,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_e2e(r: PrefillRunner, args, world, flops):
    """Same step through the C ABI from pinned HOST buffers: H2D of q/k/v, the three
    calls, D2H of o, all inside the device-timed region."""
    hq_, hk_, hv_ = (x.cpu().pin_memory() for x in (r.q, r.k, r.v))
    ho = torch.empty(r.o.shape, dtype=r.o.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_))
    d2h = ho.numel() * ho.element_size()

    def one():
        r.q.copy_(hq_, non_blocking=True)
        r.k.copy_(hk_, non_blocking=True)
        r.v.copy_(hv_, non_blocking=True)
        r.step()
        ho.copy_(r.o, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        one()
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        one()
    e.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / args.steps, world)
    return {"value": round(world * flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# ------------------------------------------------------------------ the oracle on the host

def _oracle_rates(w: mi.Workload, K_host, Qv, Kv, Vv, kbar, n_blocks: int, n_tokens: int,
                  seed: int):
    """Times the oracle on a sample: pooling of n_blocks blocks and selection+attention of
    n_tokens tokens (all groups; they read `kbar`, the oracle's own pooled keys computed
    once outside the timing).  Returns (s_per_block, s_per_token, sample text)."""
    import oracle
    from threadpoolctl import threadpool_limits
    rng = np.random.default_rng(seed)
    blocks = rng.choice(w.nb, size=min(n_blocks, w.nb), replace=False)
    toks = sorted(rng.choice(w.seq, size=min(n_tokens, w.seq), replace=False).tolist())
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for j in blocks:
            lo, hi = int(j) * w.block, min(w.seq, (int(j) + 1) * w.block)
            oracle.pool_keys(K_host[:, lo:hi], w.block)
        t1 = time.perf_counter()
        t2 = time.perf_counter()
        oracle.prefill_rows(Qv, Kv, Vv, w.block, w.topk, w.scale,
                            rows=[(0, t) for t in toks], kbar=kbar)
        t3 = time.perf_counter()
    sample = (f"pooling of {len(blocks)} random blocks + selection and attention of "
              f"{len(toks)} random tokens x {w.hkv} groups, extrapolated to the full "
              f"workload ({w.nb} blocks, {w.seq} tokens); numpy fp64, 1 thread")
    return (t1 - t0) / len(blocks), (t3 - t2) / len(toks), sample


def cpu_baseline_prefill(w, r, flops, n_blocks=64, n_tokens=96):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity_util import HostView
    import oracle
    K_host = r.k.float().cpu().numpy()
    kbar = oracle.pool_keys(K_host, w.block)
    spb, spt, sample = _oracle_rates(w, K_host, HostView(r.q), K_host, HostView(r.v), kbar,
                                     n_blocks, n_tokens, 0)
    t_full = spb * w.nb * w.batch + spt * w.seq * w.batch
    return {"value": round(flops / t_full / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
            "kind": "oracle", "sample": sample, "extrapolated_s_per_step": round(t_full, 1)}


def cpu_baseline_decode(w, q, seed=0, n_s=2):
    """Oracle decode of n_s queries (all groups) on one host core, extrapolated to
    n_query.  The fp64 pooled keys of a 10M-token bank would take minutes to build on the
    host; random values of the right shape stand in (only the time is measured), while
    K and V are the workload's bank, generated block by block as the oracle reads them."""
    import oracle
    from threadpoolctl import threadpool_limits
    kbar = mi.normal((w.nb, w.hkv, w.d), 7, 7, "cpu", torch.float32).numpy().astype(np.float64)
    Qd = q.float().cpu().numpy()
    K, V = mi.lazy_decode_bank(w, seed)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle.decode_rows(Qd, kbar, K, V, w.seq, w.block, w.topk, w.scale,
                           queries=list(range(n_s)))
        t = (time.perf_counter() - t0) / n_s * w.n_query
    sample = (f"{n_s} of {w.n_query} queries (all {w.hkv} groups), extrapolated to "
              f"{w.n_query}; numpy fp64, 1 thread; random stand-in pooled keys")
    return {"value": round(t * 1e6, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
            "sample": sample}


def run_reference_decode(args, world, w):
    """The oracle arm for decode: a bounded sample of the queries per step."""
    q, _, _ = mi.decode_inputs(w, device="cpu", seed=0, bank=False)
    times = []
    for s_ in range(args.warmup + args.steps):
        qs = torch.roll(q, shifts=-2 * s_, dims=0)
        cb = cpu_baseline_decode(w, qs)
        if s_ >= args.warmup:
            times.append(cb["value"] * 1e-6)
    t = statistics.mean(times)
    line = {
        "impl": "reference", "metric": "decode us/step", "value": round(t * 1e6, 1),
        "unit": "us/step", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "parallelism": "host oracle, rank 0 only"},
        "cpu_baseline": dict(cb, value=round(t * 1e6, 1)),
        "e2e": {"value": round(t * 1e6, 1), "unit": "us/step", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The base contract's reference arm for this method: the fp64 CPU oracle, timed on the
    host cores on a bounded sample of the same workload."""
    if rank != 0:
        return
    w = workload_of(args)
    if w.kind == "decode":
        return run_reference_decode(args, world, w)
    attn, score = prefill_flops(w)
    # inputs generated on the host in the same way (bounded: only what the sample touches)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    q, k, v = mi.prefill_inputs(w, device=dev, seed=0)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity_util import HostView
    import oracle
    K_host = k.float().cpu().numpy()
    kbar = oracle.pool_keys(K_host, w.block)
    times = []
    sample = ""
    for s in range(args.warmup + args.steps):
        spb, spt, sample = _oracle_rates(w, K_host, HostView(q), K_host, HostView(v), kbar,
                                         16, 24, s)
        if s >= args.warmup:
            times.append(spb * w.nb * w.batch + spt * w.seq * w.batch)
    t = statistics.mean(times)
    value = (attn + score) / t / 1e12
    line = {
        "impl": "reference", "metric": "sparse-attn prefill TFLOP/s", "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "seq": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "parallelism": "host oracle, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_of(args) -> mi.Workload:
    w = mi.WORKLOADS[args.workload]
    if args.seq is not None:
        w = w.with_(name=f"{w.name}@seq{args.seq}", seq=args.seq)
    return w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_1m_b256_k16", choices=list(mi.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq", type=int, default=None,
                    help="override the workload's sequence / bank length (small profiling "
                         "captures only; the JSON line then names the changed workload)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
