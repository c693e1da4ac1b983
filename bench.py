#!/usr/bin/env python
"""Benchmark of the block-sparse top-k attention hot path on B200; prints ONE JSON line.

A prefill step is one pass of the whole hot path over one synthetic sequence resident
in HBM: pool keys -> fused block scoring + top-k -> sparse attention, each through the C
ABI.  A decode step is the selection and the attention of 64 queries against an encoded
10M-token bank resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With no --workload the line's headline is the 1M-token prefill, and the 128K planted
prefill and the 10M-token decode are timed the same way (K steps after W warm-ups) under
"workloads".  Multi-GPU (torchrun, one rank per GPU): every rank
takes a part of the same problems (strong scaling): the prefill sequence split by KV group (no
collective on the data path), the decode bank split into block shards (Memory Parallel:
two all-gathers per step); the time is the max over ranks and `value` counts the work of
all ranks.  The CPU baseline and `--impl reference` time
the fp64 oracle on the host's cores (worker processes forked before the first CUDA call)
on a bounded sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import time
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import msa_inputs as mi  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_EXTRAS = ("prefill_128k_b128_k16_planted", "decode_bank10m_b64_k32")


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


def prefill_entries(w: mi.Workload) -> int:
    """Selected (token, group, block) entries of one pass (past blocks + the own block)."""
    t = np.arange(w.seq, dtype=np.int64)
    return int(np.minimum(w.topk, t // w.block + 1).sum()) * w.hkv * w.batch


def decode_work(w: mi.Workload) -> dict:
    nb = w.nb
    full = min(w.topk, nb) * w.block
    return dict(
        attn_flops=float(w.n_query * w.hq * 4 * w.d * full),
        score_flops=float(w.n_query * w.hkv * 2 * w.d * nb),
        # bytes the two phases must read at least: the pooled-key bank once as one bf16
        # plane, and the selected K/V blocks once per (query, group)
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


# ------------------------------------------------------------------ the oracle on host cores
# Worker processes are forked before the first CUDA call of this process (a process
# forked after CUDA is initialised can hang) and read the sampled workload's inputs from
# host memory-mapped files; each returns the perf_counter interval of its oracle work.

def _to_f32(x: np.ndarray) -> np.ndarray:
    """fp32 values of a host array holding fp32 values or bf16 bit patterns (exact)."""
    if x.dtype == np.uint16:
        return (np.asarray(x).astype(np.uint32) << 16).view(np.float32)
    return np.asarray(x, dtype=np.float32)


class _HostRows:
    """Read-only view of a memory-mapped [b, S, h, d] input: indexing returns fp32."""

    def __init__(self, arr):
        self.a = arr
        self.shape = arr.shape

    def __getitem__(self, key):
        return _to_f32(self.a[key])


class _QRows:
    """The query rows of the sampled tokens only, indexed like Q[b, t] / Q[b, t, heads]."""

    def __init__(self, rows: np.ndarray, keys, shape):
        self.rows = rows
        self.pos = {k: i for i, k in enumerate(keys)}
        self.shape = shape

    def __getitem__(self, key):
        r = self.rows[self.pos[(key[0], key[1])]]
        return r if len(key) == 2 else r[key[2]]


def _w_init():
    torch.set_num_threads(1)


def _w_noop(_):
    return os.getpid()


def _w_pool(spec):
    import oracle
    from threadpoolctl import threadpool_limits
    K = np.memmap(spec["k"], dtype=spec["k_dtype"], mode="r", shape=spec["k_shape"])
    kbar = np.memmap(spec["kbar"], dtype=np.float64, mode="r+", shape=spec["kbar_shape"])
    block, S = spec["block"], spec["k_shape"][1]
    j0, j1 = spec["blocks"]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for b in range(spec["k_shape"][0]):
            x = _to_f32(K[b:b + 1, j0 * block:min(S, j1 * block)])
            kbar[b:b + 1, j0:j1] = oracle.pool_keys(x, block)
        t1 = time.perf_counter()
    kbar.flush()
    return t0, t1


def _w_prefill(spec):
    import oracle
    from threadpoolctl import threadpool_limits
    K = _HostRows(np.memmap(spec["k"], dtype=spec["k_dtype"], mode="r", shape=spec["k_shape"]))
    V = _HostRows(np.memmap(spec["v"], dtype=spec["k_dtype"], mode="r", shape=spec["k_shape"]))
    kbar = np.memmap(spec["kbar"], dtype=np.float64, mode="r", shape=spec["kbar_shape"])
    Q = _QRows(spec["q_rows"], spec["rows"], spec["q_shape"])
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle.prefill_rows(Q, K, V, spec["block"], spec["topk"], spec["scale"],
                            rows=spec["rows"], kbar=kbar)
        t1 = time.perf_counter()
    return t0, t1


def _w_decode(spec):
    import oracle
    from threadpoolctl import threadpool_limits
    w = spec["w"]
    K, V = mi.lazy_decode_bank(w, spec["seed"])
    kbar = np.memmap(spec["kbar"], dtype=np.float64, mode="r", shape=spec["kbar_shape"])
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        oracle.decode_rows(spec["qd"], kbar, K, V, w.seq, w.block, w.topk, w.scale,
                           queries=spec["queries"])
        t1 = time.perf_counter()
    return t0, t1


class OraclePool:
    """Host worker processes for the oracle timings (see above)."""

    def __init__(self, n: int):
        self.n = n
        self.ex = ProcessPoolExecutor(n, mp_context=mp.get_context("fork"), initializer=_w_init)
        list(self.ex.map(_w_noop, range(n)))          # every worker exists from here on
        shm = "/dev/shm"
        self.dir = shm if os.path.isdir(shm) and os.access(shm, os.W_OK) else "/tmp"
        self.files = []

    @staticmethod
    def cores() -> int:
        try:
            n = len(os.sched_getaffinity(0))
        except AttributeError:
            n = os.cpu_count() or 1
        return max(1, min(n, 64))

    def file(self, tag: str, shape, dtype) -> tuple[str, np.memmap]:
        path = os.path.join(self.dir, f"msa_bench_{os.getpid()}_{tag}_{len(self.files)}.bin")
        self.files.append(path)
        return path, np.memmap(path, dtype=dtype, mode="w+", shape=tuple(shape))

    def host_copy(self, tag: str, t: torch.Tensor) -> tuple[str, str]:
        """A host file holding t's values (bf16 as bit patterns); returns (path, dtype)."""
        if t.dtype == torch.bfloat16:
            arr, dt = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16), "uint16"
        else:
            arr, dt = t.float().contiguous().cpu().numpy(), "float32"
        path, mm = self.file(tag, arr.shape, dt)
        mm[...] = arr
        mm.flush()
        del mm
        return path, dt

    def run(self, fn, specs) -> float:
        """Runs the specs on the workers; returns the wall time of their work."""
        spans = list(self.ex.map(fn, specs))
        return max(s[1] for s in spans) - min(s[0] for s in spans)

    def clear_files(self):
        for p in self.files:
            try:
                os.remove(p)
            except OSError:
                pass
        self.files = []

    def close(self):
        self.clear_files()
        self.ex.shutdown(cancel_futures=True)


def _split(n: int, parts: int):
    base, extra = divmod(n, parts)
    lo = 0
    for r in range(parts):
        hi = lo + base + (1 if r < extra else 0)
        if hi > lo:
            yield lo, hi
        lo = hi


class PrefillOracle:
    """The oracle's pooling (all blocks) and selection + attention (a token sample) of a
    prefill workload, on the pool's workers."""

    def __init__(self, pool: OraclePool, w: mi.Workload, q, k, v):
        self.pool, self.w, self.q = pool, w, q
        self.kpath, self.kdt = pool.host_copy("k", k)
        self.vpath, _ = pool.host_copy("v", v)
        self.kbar_shape = (w.batch, w.nb, w.hkv, w.d)
        self.kbar_path, mm = pool.file("kbar", self.kbar_shape, np.float64)
        del mm

    def pool_keys(self) -> float:
        w = self.w
        specs = [dict(k=self.kpath, k_dtype=self.kdt, k_shape=(w.batch, w.seq, w.hkv, w.d),
                      kbar=self.kbar_path, kbar_shape=self.kbar_shape, block=w.block,
                      blocks=r) for r in _split(w.nb, self.pool.n)]
        return self.pool.run(_w_pool, specs)

    def rows(self, tokens_per_worker: int, seed: int) -> tuple[float, int]:
        w = self.w
        rng = np.random.default_rng(seed)
        n = min(w.seq * w.batch, tokens_per_worker * self.pool.n)
        flat = np.sort(rng.choice(w.seq * w.batch, size=n, replace=False))
        rows = [(int(f // w.seq), int(f % w.seq)) for f in flat]
        bi = torch.tensor([r[0] for r in rows], device=self.q.device)
        ti = torch.tensor([r[1] for r in rows], device=self.q.device)
        q_rows = self.q[bi, ti].float().cpu().numpy()
        specs = []
        for lo, hi in _split(len(rows), self.pool.n):
            specs.append(dict(k=self.kpath, v=self.vpath, k_dtype=self.kdt,
                              k_shape=(w.batch, w.seq, w.hkv, w.d), kbar=self.kbar_path,
                              kbar_shape=self.kbar_shape, q_rows=q_rows[lo:hi],
                              rows=rows[lo:hi], q_shape=tuple(self.q.shape), block=w.block,
                              topk=w.topk, scale=w.scale))
        return self.pool.run(_w_prefill, specs), len(rows)

    def step_seconds(self, tokens_per_worker: int, seed: int) -> tuple[float, str]:
        """Oracle seconds of one whole prefill step: the pooling of every block, and the
        selection + attention of a token sample extrapolated to every token."""
        t_pool = self.pool_keys()
        t_rows, n = self.rows(tokens_per_worker, seed)
        w = self.w
        t = t_pool + t_rows * (w.seq * w.batch) / n
        sample = (f"pooling of all {w.nb * w.batch} blocks + selection and attention of {n} "
                  f"random tokens x {w.hkv} groups (of {w.seq * w.batch}), extrapolated to "
                  f"every token; numpy fp64, {self.pool.n} worker processes, 1 thread each")
        return t, sample


class DecodeOracle:
    """The oracle's decode of a query sample against the workload's bank (regenerated
    block by block from the seeded generator as the oracle reads it).  The fp64 pooled
    keys of a 10M-token bank would take minutes to build on the host, so random values of
    the right shape stand in for them: only the time is measured."""

    def __init__(self, pool: OraclePool, w: mi.Workload, q, seed: int = 0):
        self.pool, self.w, self.seed = pool, w, seed
        self.qd = q.float().cpu().numpy()
        self.kbar_shape = (w.nb, w.hkv, w.d)
        self.kbar_path, mm = pool.file("dkbar", self.kbar_shape, np.float64)
        rng = np.random.default_rng(7)
        for lo in range(0, w.nb, 1 << 14):
            hi = min(w.nb, lo + (1 << 14))
            mm[lo:hi] = rng.standard_normal((hi - lo, w.hkv, w.d)) * 0.125
        mm.flush()
        del mm

    def step_seconds(self, queries_per_worker: int, seed: int) -> tuple[float, str]:
        w = self.w
        n = min(w.n_query, queries_per_worker * self.pool.n)
        qs = [int(x) for x in np.sort(np.random.default_rng(seed).choice(w.n_query, n,
                                                                          replace=False))]
        specs = [dict(w=w, seed=self.seed, kbar=self.kbar_path, kbar_shape=self.kbar_shape,
                      qd=self.qd, queries=qs[lo:hi]) for lo, hi in _split(n, self.pool.n)]
        t = self.pool.run(_w_decode, specs) * w.n_query / n
        sample = (f"{n} of {w.n_query} queries (all {w.hkv} groups)"
                  + (f", extrapolated to {w.n_query}" if n < w.n_query else "")
                  + f"; numpy fp64, {self.pool.n} worker processes, 1 thread each; random "
                  "stand-in pooled keys")
        return t, sample


# ------------------------------------------------------------------ our implementation

def kv_group_split(w: mi.Workload, rank: int, world: int) -> mi.Workload:
    """Rank `rank`'s part of one sequence split by KV group: KV heads
    [rank * hkv / world, (rank + 1) * hkv / world) and their query heads."""
    if w.hkv % world != 0:
        raise SystemExit(f"{w.name}: {w.hkv} KV heads do not split over {world} ranks")
    return w.with_(hq=w.hq // world, hkv=w.hkv // world)


class PrefillRunner:
    """Holds device buffers and issues one step through the C ABI.  With world > 1 the
    rank holds its KV-group slice of the one sequence (contiguous tensors of its heads, as
    a head-sharded QKV projection produces them) and runs the same calls on it."""

    def __init__(self, w: mi.Workload, seed: int, rank: int = 0, world: int = 1,
                 select_only: bool = False):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib = msa, _lib.load()
        self.select_only = select_only
        q, k, v = mi.prefill_inputs(w, device="cuda", seed=seed)
        if select_only:
            v = torch.empty(0, dtype=q.dtype, device=q.device)
        if world > 1:
            wl = kv_group_split(w, rank, world)
            g0, g1 = rank * wl.hkv, (rank + 1) * wl.hkv
            G = w.hq // w.hkv
            q = q[:, :, g0 * G:g1 * G].contiguous()
            k = k[:, :, g0:g1].contiguous()
            v = v[:, :, g0:g1].contiguous()
            w = wl
            torch.cuda.empty_cache()
        self.w = w
        self.q, self.k, self.v = q, k, v
        dev = self.q.device
        self.p = msa.params(batch=w.batch, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                            topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.kbar = torch.empty(w.batch, w.nb, w.hkv, w.d, dtype=torch.float32, device=dev)
        # bf16 hi/lo planes of the pooled keys feed the tensor-core selection
        self.khi = torch.empty(w.batch, w.nb, w.hkv, w.d, dtype=torch.bfloat16, device=dev)
        self.klo = torch.empty_like(self.khi)
        self.idx = torch.empty(w.batch, w.hkv, w.seq, w.topk, dtype=torch.int32, device=dev)
        self.o = torch.empty(0 if select_only else self.q.numel(), dtype=self.q.dtype, device=dev)
        self.lse = torch.empty(0 if select_only else w.batch * w.hq * w.seq, dtype=torch.float32,
                               device=dev)
        n = self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_TOPK_SELECT, 0)
        if not select_only:
            n = max(n, self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_SPARSE_ATTN, 0))
        self.ws = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.check = _lib.check
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        self.ptr = {k: P(getattr(self, k)) for k in ("q", "k", "v", "kbar", "khi", "klo", "idx", "o",
                                                     "lse", "ws")}
        self.pp = ctypes.byref(self.p)
        # own kernels per step (memsets excluded): pool 1; selection: tensor-core pass +
        # exact pass over flagged tiles = 2; attention, per token slab: count, scan, fill,
        # tile table, tiles, merge = 6
        if select_only:
            self.n_slabs = 0
            self.launches_per_step = 3
            return
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
        if self.select_only:
            return
        self.check("msa_sparse_attn_fwd", lib.msa_sparse_attn_fwd(
            self.pp, P["q"], P["k"], P["v"], P["idx"], P["o"], P["lse"], P["ws"],
            self.ws.numel(), s))
        if events:
            events[3].record()


def select_launches(nb: int) -> int:
    """Own kernels of one selection over an encoded bank of nb blocks: [sample scan,
    threshold,] hi-plane scan, candidate select or merge, exact rescoring, and the two
    launches of the exact rescan (which exit at once when every row is certified).  The
    sample pass runs from 128 chunks of 128 blocks per group."""
    return 7 if -(-nb // 128) >= 128 else 5


class DecodeRunner:
    """Decode of n_query queries against a bank resident in HBM, through the C ABI.  The
    bank's pooled keys and encoded images are built once up front (the offline encoding
    of a bank, not timed); the step reads only the encoded images."""

    def __init__(self, w: mi.Workload, seed: int, rank: int = 0, world: int = 1):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        self.rank, self.world = rank, world
        self.q, _, _ = mi.decode_inputs(w, device="cuda", seed=seed, bank=False)
        dev = self.q.device
        if world > 1:
            # Memory Parallel: this rank holds only its contiguous shard of the bank
            from block_sparse_top_mean_b200.memory_parallel import BankShard, shard_ranges
            begin, count = shard_ranges(w.nb, world)[rank]
            t0, t1 = begin * w.block, min(w.seq, (begin + count) * w.block)
            k, v = mi.decode_bank_rows(w, t0, t1, device="cuda", seed=seed)
            self.shard = BankShard(k, v, w.block, begin)
            del k, v
            self.kt, self.vt, self.bt = (self.shard.k_tiles, self.shard.v_tiles,
                                         self.shard.kbar_tiles)
            seq_local = t1 - t0
        else:
            self.shard = None
            _, k, v = mi.decode_inputs(w, device="cuda", seed=seed)
            _, khi, klo = (t[0] for t in msa.pool_keys(k[None], w.block, split=True))
            self.kt, self.vt, self.bt = msa.encode_bank(k, v, khi, klo, w.block)
            del k, v, khi, klo                  # the natural layout is not needed any more
            seq_local = w.seq
            if w.host_bank:
                # the content images move to pinned host memory; only the routing planes
                # (bt) stay in HBM
                self.kt, self.vt = self.kt.cpu().pin_memory(), self.vt.cpu().pin_memory()
        torch.cuda.empty_cache()
        self.p = msa.params(batch=1, seq=seq_local, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                            topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(w.n_query, w.hq, dtype=torch.float32, device=dev)
        self.idx = torch.empty(w.n_query, w.hkv, w.topk, dtype=torch.int32, device=dev)
        op = _lib.OP_DECODE_OFFLOAD if w.host_bank else _lib.OP_DECODE
        n = self.lib.msa_workspace_bytes(ctypes.byref(self.p), op, w.n_query)
        self.ws = torch.zeros(n, dtype=torch.uint8, device=dev)
        self.check = _lib.check
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        self.ptr = {k: P(getattr(self, k)) for k in ("q", "kt", "vt", "bt", "idx", "o", "lse",
                                                     "ws")}
        self.pp = ctypes.byref(self.p)
        # own kernels per step: the selection's, then attention and split combine
        self.nb_local = -(-seq_local // w.block)
        self.launches_per_step = select_launches(self.nb_local) + 2

    def step(self, events=None):
        if self.shard is not None:
            return self.step_sharded(events)
        if self.w.host_bank:
            return self.step_host_bank(events)
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


    def step_host_bank(self, events=None):
        """msa_decode_fwd_offload: selection, staging of the selected K/V tiles from host
        memory over PCIe, attention on the staged copy."""
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        P, w = self.ptr, self.w
        if events:
            events[0].record()
        self.check("msa_decode_fwd_offload", self.lib.msa_decode_fwd_offload(
            self.pp, w.n_query, P["q"], P["bt"], P["kt"], P["vt"], P["idx"], P["o"], P["lse"],
            P["ws"], self.ws.numel(), s))
        if events:
            events[1].record()
            events[2].record()

    def step_sharded(self, events=None):
        """Memory Parallel decode step: shard scan, all-gather of the keys, merge, owned-block
        attention, all-gather of the partials, combine (block_sparse_top_mean_b200.
        memory_parallel.decode_step)."""
        from block_sparse_top_mean_b200.memory_parallel import decode_step
        if events:
            events[0].record()
        self.o, self.lse, self.idx = decode_step(self.q, self.shard, self.w.topk, self.w.scale,
                                                 ws=self.ws)
        if events:
            events[1].record()
            events[2].record()


class DocsRunner:
    """Packed documents: document-wise RoPE of q and k in place, then the causal prefill of
    every document (msa_rope_docwise + msa_prefill_varlen_fwd).  Each step rotates q and k
    again; the work per step is the same."""

    def __init__(self, w: mi.Workload, seed: int):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        q, k, v = mi.prefill_inputs(w, device="cuda", seed=seed)
        self.q, self.k, self.v = q[0], k[0], v[0]
        self.lengths = mi.doc_lengths(w.seq, w.n_docs, seed)
        self.cu = mi.cu_seqlens(self.lengths)
        self.cu_dev = torch.tensor(self.cu, dtype=torch.int32, device="cuda")
        self.ws = msa.varlen_workspace(self.q, self.k, self.cu, w.block, w.topk)
        # own kernels per step: the rotation, then per document pool + 2 selection + 6 per
        # attention token slab
        slabs = sum(-(-L // max(1, msa.attn_slab_tokens(
            msa.params(batch=1, seq=L, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block, topk=w.topk,
                       scale=w.scale, dtype=self.q.dtype), _lib.OP_PREFILL, self.ws.numel())))
            for L in self.lengths)
        self.launches_per_step = 1 + 3 * len(self.lengths) + 6 * slabs

    def step(self, events=None):
        w = self.w
        if events:
            events[0].record()
        self.msa.rope_docwise(self.q, self.k, self.cu_dev, w.rope_base)
        if events:
            events[1].record()
        self.o, self.lse, self.idx = self.msa.prefill_varlen_fwd(
            self.q, self.k, self.v, self.cu, w.block, w.topk, w.scale, ws=self.ws)
        if events:
            events[2].record()


class BwdRunner:
    """The backward of the sparse attention for a fixed selection: the forward runs once
    (untimed) for o, lse and idx; a step is msa_sparse_attn_bwd."""

    def __init__(self, w: mi.Workload, seed: int):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        self.q, self.k, self.v = mi.prefill_inputs(w, device="cuda", seed=seed)
        self.o, self.lse, self.idx = msa.prefill_fwd(self.q, self.k, self.v, w.block, w.topk,
                                                     w.scale)
        self.dout = mi.normal(self.q.shape, seed + 7, mi.STREAM_DECODE_Q, "cuda", torch.bfloat16)
        self.dq = torch.empty(self.q.shape, dtype=torch.float32, device="cuda")
        self.dk = torch.empty(self.k.shape, dtype=torch.float32, device="cuda")
        self.dv = torch.empty(self.v.shape, dtype=torch.float32, device="cuda")
        p = msa.params(batch=w.batch, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                       topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.ws = msa.workspace(p, _lib.OP_SPARSE_ATTN_BWD)
        torch.cuda.empty_cache()

    def step(self, events=None):
        if events:
            events[0].record()
        self.msa.sparse_attn_bwd(self.q, self.k, self.v, self.o, self.lse, self.dout, self.idx,
                                 self.w.block, self.w.scale, ws=self.ws,
                                 out=(self.dq, self.dk, self.dv))
        if events:
            events[1].record()


def bench_bwd(w, args, world, rank, local, pool):
    if world > 1:
        raise SystemExit(f"{w.name}: one GPU only")
    r = BwdRunner(w, seed=0)
    attn, _ = prefill_flops(w)
    flops = attn * 10 / 4          # S, dP, dV, dK, dQ: five 2*d contractions per (head, key)
    ms, ev, clocks = timed_steps(r, args, world, local, 2)
    peaks, peak_src = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "sparse-attn backward TFLOP/s", "value": round(tf, 3), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "seq": w.seq, "hq": w.hq, "hkv": w.hkv, "d": w.d,
                   "block": w.block, "topk": w.topk, "planted_frac": w.planted_frac,
                   "workspace_gib": round(r.ws.numel() / 2**30, 2), "parallelism": "one GPU"},
        "flops_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": "msa_sparse_attn_bwd (whole call)",
                     "achieved": round(tf, 2), "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops_sustained"], 4),
                     "peak_source": f"bf16_tflops_sustained of {peak_src}", "traffic": None,
                     "algorithmic_per_launch": flops},
        "cpu_baseline": None, "e2e": None, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_docs(w, args, world, rank, local, pool):
    if world > 1:
        raise SystemExit(f"{w.name}: one GPU only")
    r = DocsRunner(w, seed=0)
    attn = score = 0.0
    for L in r.lengths:
        a, s_ = prefill_flops(w.with_(seq=L))
        attn += a
        score += s_
    ms, ev, clocks = timed_steps(r, args, world, local, 3)
    rope_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    pre_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    peaks, peak_src = load_peaks()
    rope_bytes = float(w.seq * (w.hq + w.hkv) * w.d * 2 * 2)
    rope_gbs = rope_bytes / (rope_ms * 1e-3) / 1e9
    line = {
        "metric": "sparse-attn prefill TFLOP/s", "value": round((attn + score) / (ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.seq, "n_docs": w.n_docs,
                   "doc_len_min": min(r.lengths), "doc_len_max": max(r.lengths), "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "rope_base": w.rope_base, "parallelism": "one GPU"},
        "phases_ms": {"rope_docwise": round(rope_ms, 3), "prefill_varlen": round(pre_ms, 3)},
        "flops_per_step": {"attention": attn, "scoring": score},
        "roofline": {"bound": "tensor", "kernel": "msa_prefill_varlen_fwd (all documents)",
                     "achieved": round((attn + score) / (pre_ms * 1e-3) / 1e12, 2),
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round((attn + score) / (pre_ms * 1e-3) / 1e12
                                   / peaks["bf16_tflops_sustained"], 4),
                     "peak_source": f"bf16_tflops_sustained of {peak_src}", "traffic": None},
        "rope_roofline": {"bound": "hbm", "kernel": "rope_docwise_kernel",
                          "achieved": round(rope_gbs, 1), "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": round(rope_gbs / peaks["hbm_gbs"], 4),
                          "algorithmic_per_launch": rope_bytes},
        "cpu_baseline": None, "e2e": None,
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


E2E_OVERLAP = ("double-buffered: per step H2D of the inputs, the calls and D2H of the "
               "output on their own streams; step i's D2H overlaps step i+1's H2D and compute")


def set_io_of(self, **tensors):
    """Points a runner's step at other device tensors of the same shapes."""
    for name, t in tensors.items():
        setattr(self, name, t)
        self.ptr[name] = ctypes.c_void_p(t.data_ptr())


PrefillRunner.set_io = set_io_of
DecodeRunner.set_io = set_io_of


def timed_steps(r, args, world, local, n_events):
    """W warm-ups, then exactly K steps between barriers and synchronisations, with the
    SM clock sampled meanwhile.  Returns (ms per step max over ranks, per-step phase
    events, clock summary)."""
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
          for _ in range(args.steps)]
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
    ms = max_over_ranks(start.elapsed_time(end) / args.steps, world)
    return ms, ev, clk.summary()


def e2e_steps(r, args, world, in_names, out_name):
    """The same step through the C ABI from pinned HOST buffers: every step copies its
    inputs host -> device, runs the calls and copies its output device -> host, all inside
    the device-timed region.  Double-buffered over three streams (copies in, compute,
    copies out) with two device buffer sets, so step i's device -> host copy overlaps
    step i+1's host -> device copy and compute.  Returns (ms per step, h2d, d2h bytes)."""
    ins = [getattr(r, n) for n in in_names]
    out = getattr(r, out_name)
    hosts = [x.cpu().pin_memory() for x in ins]
    ho = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    sets = [ins + [out], [torch.empty_like(x) for x in ins] + [torch.empty_like(out)]]
    names = list(in_names) + [out_name]
    s_cmp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i & 1
        bufs = sets[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_cmp[b])         # step i-2's compute is done with set b
            for d_, h_ in zip(bufs[:-1], hosts):
                d_.copy_(h_, non_blocking=True)
            ev_in[b].record(s_in)
        s_cmp.wait_event(ev_in[b])
        if used[b]:
            s_cmp.wait_event(ev_out[b])            # step i-2's output has left set b
        r.set_io(**dict(zip(names, bufs)))
        r.step()
        ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            ho[b].copy_(bufs[-1], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(max(1, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(s_in)
    for i in range(args.steps):
        one(i)
    e.record(s_out)
    torch.cuda.synchronize()
    r.set_io(**dict(zip(names, sets[0])))
    ms = max_over_ranks(s.elapsed_time(e) / args.steps, world)
    return ms, sum(x.numel() * x.element_size() for x in hosts), ho[0].numel() * ho[0].element_size()


# DRAM bytes (read + write) of the prefill attention phase per selected (token, group,
# block) entry, from one ncu capture of the 1M workload shortened to 32K tokens (Q 256 MiB,
# larger than L2; 3,948,544 entries): tiles kernel 2006.0, partial merge 1112.4, index
# inversion 8.9 (profiles/prefill_32k_b256_k16_attn_dram.md).  The per-entry traffic does
# not depend on the sequence length at this block size: every block is selected by about
# 4096 entries per group at 32K and at 1M alike.
PREFILL_ATTN_DRAM_PER_ENTRY = {"attn_tiles_kernel": 2006.0, "merge_partials_kernel": 1112.4,
                               "index inversion": 8.9}


def bench_prefill(w, args, world, rank, local, pool):
    r = PrefillRunner(w, seed=0, rank=rank, world=world)
    w_full, w = w, r.w
    attn_flops, score_flops = prefill_flops(w)
    ms, ev, clocks = timed_steps(r, args, world, local, 4)
    phase = {n: statistics.mean(e[a].elapsed_time(e[a + 1]) for e in ev)
             for a, n in enumerate(["pool_keys", "topk_select", "sparse_attn"])}
    err = r.msa.read_device_error(r.ws)
    peaks, peak_src = load_peaks()
    # every rank holds 1/world of the sequence's KV groups: world x its work = the sequence
    value = world * (attn_flops + score_flops) / (ms * 1e-3) / 1e12
    tokens_s = w_full.seq * w_full.batch / (ms * 1e-3)
    attn_tflops = attn_flops / (phase["sparse_attn"] * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    entries = prefill_entries(w)
    per_entry = sum(PREFILL_ATTN_DRAM_PER_ENTRY.values())
    traffic = round(per_entry * entries)
    roof = {"bound": "tensor",
            "kernel": "msa_sparse_attn_fwd (index inversion, tcgen05 tiles, partial merge)",
            "achieved": round(attn_tflops, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(attn_tflops / peak, 4),
            "peak_source": f"bf16_tflops_sustained of {peak_src}", "traffic": traffic,
            "traffic_source": "ncu dram bytes of the phase's kernels on the 1M workload "
                              "shortened to 32K tokens, per selected (token, group, block) "
                              "entry, times this workload's entries",
            "traffic_per_entry": PREFILL_ATTN_DRAM_PER_ENTRY,
            "traffic_floor_ms": round(traffic / (peaks["hbm_gbs"] * 1e9) * 1e3, 2),
            "algorithmic_bytes": float(w.batch * w.seq * (2 * w.hq + 2 * w.hkv) * w.d * 2),
            "algorithmic_per_launch": attn_flops, "selected_entries": entries}
    e2e = None
    if not args.no_e2e:
        ems, h2d, d2h = e2e_steps(r, args, world, ["q", "k", "v"], "o")
        e2e = {"value": round(world * (attn_flops + score_flops) / (ems * 1e-3) / 1e12, 3),
               "unit": "TFLOP/s", "ms_per_step": round(ems, 3), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "overlap": E2E_OVERLAP}
    cpu = None
    if pool is not None:
        orc = PrefillOracle(pool, w, r.q, r.k, r.v)
        t, sample = orc.step_seconds(192, 0)
        pool.clear_files()
        cpu = {"value": round((attn_flops + score_flops) / t / 1e12, 6), "unit": "TFLOP/s",
               "cores": pool.n, "kind": "oracle", "sample": sample,
               "extrapolated_s_per_step": round(t, 1)}
    line = {
        "metric": "sparse-attn prefill TFLOP/s", "value": round(value, 3), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w_full.name, "batch": w.batch, "seq": w.seq, "hq": w_full.hq,
                   "hkv": w_full.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "kv_heads_per_gpu": w.hkv,
                   "planted_frac": w.planted_frac,
                   "l2": f"inputs larger than L2 (Q alone {w.batch * w.seq * w.hq * w.d * 2 / 2**30:.2f} GiB), no flush",
                   "workspace_gib": round(r.ws.numel() / 2**30, 2),
                   "attn_token_slabs": r.n_slabs,
                   "parallelism": ("one GPU" if world == 1 else
                                   f"one sequence split by KV group over {world} GPUs "
                                   f"({w.hkv} KV heads each), no collective on the data path")},
        "tokens_per_s": round(tokens_s, 1),
        "flops_per_step": {"attention": attn_flops, "scoring": score_flops},
        "phases_ms": {k: round(v, 3) for k, v in phase.items()},
        "attn_phase_tflops": round(attn_tflops, 2),
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks,
        "device_error_bits": err,
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_decode(w, args, world, rank, local, pool):
    r = DecodeRunner(w, seed=0, rank=rank, world=world)
    work = decode_work(w)
    # the encoded bank (41 GB) and its pooled-key planes (0.6 GB) are larger than L2
    ms, ev, clocks = timed_steps(r, args, world, local, 3)
    peaks, peak_src = load_peaks()
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    # what the selection streams: the hi plane, every 8th chunk of it again for the sample
    # bounds, and the hi + lo rows of 64 candidates per (query, group) for the rescoring
    nch = -(-w.nb // 128)
    planes_read = float(w.nb * w.hkv * w.d * 2 + -(-nch // 8) * 128 * w.hkv * w.d * 2 +
                        w.n_query * w.hkv * 64 * w.d * 2 * 2)
    if world > 1:
        return bench_decode_sharded(w, r, args, world, ms, clocks, peaks, peak_src, work)
    if w.host_bank:
        return bench_decode_host_bank(w, r, args, ms, clocks, work)
    phases = {
        "select": {"ms": sel_ms, "bytes": work["score_bytes"],
                   "kernel": "msa_decode_select_tiled (hi-plane sample scan + threshold + "
                             "hi-plane filter scan + candidate select + exact rescoring "
                             "with certificate; the exact rescan launches exit at once)",
                   # DRAM bytes (read + write) of its kernels in one ncu capture of this
                   # 10M-token bank's planes (profiles/decode_bank10m_b64_k32_select_dram.md):
                   # the two scans (40.70 + 322.04 MB) scale with the bank's blocks; the
                   # threshold, select, rescoring and the two exiting launches (1.26 + 2.83
                   # + 17.14 + 0.10 MB) with the 512 (query, group) rows
                   "traffic": (40.70e6 + 322.04e6) * w.nb / 156250 +
                              (1.26e6 + 2.83e6 + 17.14e6 + 0.10e6) * w.n_query * w.hkv / 512},
        "attend": {"ms": att_ms, "bytes": work["attn_bytes"],
                   "kernel": "msa_decode_attn_tiled (streamed attention + split combine)",
                   # the attention kernel's DRAM bytes in the same capture (526.3 MB read,
                   # 16.8 MB written); they depend on the selection, not on the bank size
                   "traffic": 543.09e6 * w.n_query * w.hkv * w.topk / (64 * 8 * 32)},
    }
    dom = phases["select"]
    gbs = dom["bytes"] / (dom["ms"] * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": dom["kernel"], "achieved": round(gbs, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
            "peak_source": f"hbm_gbs of {peak_src}", "traffic": round(dom["traffic"]),
            "traffic_source": "ncu dram bytes of the selection's kernels on the 10M-token "
                              "bank's planes (see profiles/)",
            "algorithmic_per_launch": dom["bytes"],
            "algorithmic_note": "one bf16 plane of the pooled keys: the scan streams the hi "
                                "plane; the lo plane is read only for each row's 64 "
                                "candidates",
            "planes_read_bytes": planes_read,
            "planes_read_gbs": round(planes_read / (dom["ms"] * 1e-3) / 1e9, 1)}
    phase_line = {k: {"us": round(v["ms"] * 1e3, 1),
                      "gbs": round(v["bytes"] / (v["ms"] * 1e-3) / 1e9, 1)}
                  for k, v in phases.items()}
    e2e = None
    if not args.no_e2e:
        ems, h2d, d2h = e2e_steps(r, args, world, ["q"], "o")
        e2e = {"value": round(ems * 1e3, 1), "unit": "us/step", "ms_per_step": round(ems, 4),
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "overlap": E2E_OVERLAP}
    cpu = None
    if pool is not None:
        t, sample = DecodeOracle(pool, w, r.q, seed=rank).step_seconds(2, 0)
        pool.clear_files()
        cpu = {"value": round(t * 1e6, 1), "unit": "us/step", "cores": pool.n,
               "kind": "oracle", "sample": sample}
    line = {
        "metric": "decode us/step", "value": round(ms * 1e3, 1), "unit": "us/step",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "strong",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "l2": "bank and pooled keys larger than L2, no flush",
                   "parallelism": "one GPU"},
        "phases": phase_line, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


class SelectOnlyRunner:
    """The decode selection alone over a bank's encoded pooled-key image: the bank's keys
    are generated and pooled in slices, only the routing image is kept (no K/V images)."""

    def __init__(self, w: mi.Workload, seed: int):
        import block_sparse_top_mean_b200 as msa
        from block_sparse_top_mean_b200 import _lib
        self.msa, self.lib, self.w = msa, _lib.load(), w
        self.q, _, _ = mi.decode_inputs(w, device="cuda", seed=seed, bank=False)
        khi = torch.empty(w.nb, w.hkv, w.d, dtype=torch.bfloat16, device="cuda")
        klo = torch.empty_like(khi)
        step = 1 << 20                                   # tokens per slice (whole blocks)
        for t0 in range(0, w.seq, step):
            t1 = min(w.seq, t0 + step)
            k, _ = mi.decode_bank_rows(w, t0, t1, device="cuda", seed=seed)
            _, h, l = (t[0] for t in msa.pool_keys(k[None], w.block, split=True))
            b0 = t0 // w.block
            khi[b0:b0 + h.shape[0]], klo[b0:b0 + h.shape[0]] = h, l
            del k, h, l
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        pe = msa.params(batch=1, seq=w.seq, hq=w.hkv, hkv=w.hkv, d=w.d, block=w.block, topk=1,
                        scale=1.0, dtype=torch.bfloat16)
        self.bt = torch.empty(self.lib.msa_bank_tiles_bytes(ctypes.byref(pe), 1),
                              dtype=torch.uint8, device="cuda")
        _lib.check("msa_encode_bank", self.lib.msa_encode_bank(
            ctypes.byref(pe), None, None, P(khi), P(klo), None, None, P(self.bt), None))
        del khi, klo
        torch.cuda.empty_cache()
        self.p = msa.params(batch=1, seq=w.seq, hq=w.hq, hkv=w.hkv, d=w.d, block=w.block,
                            topk=w.topk, scale=w.scale, dtype=self.q.dtype)
        self.idx = torch.empty(w.n_query, w.hkv, w.topk, dtype=torch.int32, device="cuda")
        n = self.lib.msa_workspace_bytes(ctypes.byref(self.p), _lib.OP_DECODE, w.n_query)
        self.ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        self.check = _lib.check
        self.ptr = {k: P(getattr(self, k)) for k in ("q", "bt", "idx", "ws")}
        self.launches_per_step = select_launches(w.nb)

    def step(self, events=None):
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        P, w = self.ptr, self.w
        if events:
            events[0].record()
        self.check("msa_decode_select_tiled", self.lib.msa_decode_select_tiled(
            ctypes.byref(self.p), w.n_query, P["q"], P["bt"], P["idx"], P["ws"],
            self.ws.numel(), s))
        if events:
            events[1].record()


def bench_prefill_select_only(w, args, local):
    """Pooling and selection of a prefill workload alone (no V, O or attention workspace)."""
    r = PrefillRunner(w, seed=0, select_only=True)
    ms, ev, clocks = timed_steps(r, args, 1, local, 3)
    _, score_flops = prefill_flops(w)
    sel_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    line = {
        "metric": "prefill selection ms/step", "value": round(sel_ms, 3), "unit": "ms/step",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "scope": "msa_pool_keys + msa_topk_select alone"},
        "scoring_tflops": round(score_flops / (sel_ms * 1e-3) / 1e12, 2),
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_decode_select_only(w, args, local):
    r = SelectOnlyRunner(w, seed=0)
    ms, _, clocks = timed_steps(r, args, 1, local, 2)
    work = decode_work(w)
    line = {
        "metric": "decode selection us/step", "value": round(ms * 1e3, 1), "unit": "us/step",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "scope": "msa_decode_select_tiled alone (no K/V images)"},
        "gbs_one_plane": round(work["score_bytes"] / (ms * 1e-3) / 1e9, 1),
        "gpu_launches": r.launches_per_step * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_decode_host_bank(w, r, args, ms, clocks, work):
    """The decode line with the bank's K/V in pinned host memory: the step is bound by the
    PCIe transfer of the selected tiles (each selected (group, block) once)."""
    idx = r.idx.view(w.n_query, w.hkv, w.topk)
    staged = sum(int(torch.unique(idx[:, g][idx[:, g] >= 0]).numel()) for g in range(w.hkv))
    fetched = staged * w.block * w.d * 2 * 2
    gbs = fetched / (ms * 1e-3) / 1e9
    line = {
        "metric": "decode us/step", "value": round(ms * 1e3, 1), "unit": "us/step",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": False, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "bank_content": "pinned host memory, read by the GPU over PCIe",
                   "parallelism": "one GPU"},
        "roofline": {"bound": "pcie", "kernel": "msa_decode_fwd_offload (whole step)",
                     "achieved": round(gbs, 2), "unit": "GB/s", "peak": None,
                     "frac": None, "traffic": None,
                     "algorithmic_per_launch": fetched,
                     "note": "K/V bytes of the distinct selected (group, block) pairs fetched "
                             "from host memory per step, over the step time"},
        "staged_blocks_per_step": staged,
        "cpu_baseline": None, "e2e": None,
        # selection, the four staging kernels, attention and split combine
        "gpu_launches": (select_launches(w.nb) + 6) * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_decode_sharded(w, r, args, world, ms, clocks, peaks, peak_src, work):
    """The Memory Parallel decode line: the bank split over the ranks, one step = shard
    scan + key all-gather + merge + owned-block attention + partial all-gather + combine."""
    per_rank = (work["score_bytes"] + work["attn_bytes"]) / world
    gbs = per_rank / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": "Memory Parallel decode step (one rank)",
            "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"hbm_gbs of {peak_src}",
            "traffic": None, "algorithmic_per_launch": per_rank,
            "algorithmic_note": "one bf16 plane of the rank's pooled keys and, on average, "
                                "1/world of the selected K/V blocks"}
    line = {
        "metric": "decode us/step", "value": round(ms * 1e3, 1), "unit": "us/step",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "strong",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
                   "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
                   "l2": "bank and pooled keys larger than L2, no flush",
                   "parallelism": f"Memory Parallel: the bank in {world} contiguous block "
                                  f"shards, two NCCL all-gathers per step"},
        "roofline": roof, "cpu_baseline": None, "e2e": None,
        # the shard's selection, key merge, attention, split combine, shard combine
        "gpu_launches": (select_launches(r.nb_local) + 5) * args.steps, "clocks": clocks,
        "device_error_bits": r.msa.read_device_error(r.ws),
    }
    del r
    torch.cuda.empty_cache()
    return line


def bench_one(name, args, world, rank, local, pool):
    w = workload_of(name, args.seq)
    if getattr(args, "select_only", False):
        assert world == 1 and w.kind in ("decode", "prefill"), \
            "--select-only: one GPU, a decode or prefill workload"
        if w.kind == "prefill":
            return bench_prefill_select_only(w, args, local)
        return bench_decode_select_only(w, args, local)
    fn = {"prefill": bench_prefill, "decode": bench_decode, "prefill_docs": bench_docs,
          "prefill_bwd": bench_bwd}[w.kind]
    return fn(w, args, world, rank, local, pool)


def run_ours(args, world, rank, local, pool):
    from block_sparse_top_mean_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    line = bench_one(args.workload, args, world, rank, local, pool)
    if args.default_set:
        line["workloads"] = {}
        for name in DEFAULT_EXTRAS:
            sub = bench_one(name, args, world, rank, local, pool)
            sub.pop("n_gpus", None)
            line["workloads"][name] = sub
        line["gpu_launches_all_workloads"] = line["gpu_launches"] + sum(
            s["gpu_launches"] for s in line["workloads"].values())
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the reference arm

def run_reference(args, world, rank, pool):
    """The base contract's reference arm for this method: the fp64 CPU oracle, timed on the
    host cores, each step a bounded sample of the same workload (rank 0 only)."""
    if rank != 0:
        return
    w = workload_of(args.workload, args.seq)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    times, sample = [], ""
    if w.kind == "decode":
        q, _, _ = mi.decode_inputs(w, device="cpu", seed=0, bank=False)
        orc = DecodeOracle(pool, w, q)
        for s_ in range(args.warmup + args.steps):
            t, sample = orc.step_seconds(1, s_)
            if s_ >= args.warmup:
                times.append(t)
        t = statistics.mean(times)
        value, unit, hib, metric = round(t * 1e6, 1), "us/step", False, "decode us/step"
        cfg = {"workload": w.name, "n_query": w.n_query, "bank_tokens": w.seq, "hq": w.hq,
               "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk}
    else:
        attn, score = prefill_flops(w)
        q, k, v = mi.prefill_inputs(w, device=dev, seed=0)
        orc = PrefillOracle(pool, w, q, k, v)
        del k, v
        for s_ in range(args.warmup + args.steps):
            t, sample = orc.step_seconds(12, s_)
            if s_ >= args.warmup:
                times.append(t)
        t = statistics.mean(times)
        value, unit, hib, metric = (attn + score) / t / 1e12, "TFLOP/s", True, \
            "sparse-attn prefill TFLOP/s"
        cfg = {"workload": w.name, "batch": w.batch, "seq": w.seq, "hq": w.hq,
               "hkv": w.hkv, "d": w.d, "block": w.block, "topk": w.topk,
               "planted_frac": w.planted_frac}
    cfg["parallelism"] = "host oracle, rank 0 only"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": hib, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": unit, "cores": pool.n, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_of(name: str, seq) -> mi.Workload:
    w = mi.WORKLOADS[name]
    if seq is not None:
        w = w.with_(name=f"{w.name}@seq{seq}", seq=seq)
    return w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None, choices=list(mi.WORKLOADS),
                    help="one workload only (default: the 1M prefill as the headline plus "
                         "the 128K planted prefill and the 10M-token decode)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq", type=int, default=None,
                    help="override the workload's sequence / bank length (small profiling "
                         "captures only; the JSON line then names the changed workload)")
    ap.add_argument("--select-only", action="store_true",
                    help="decode: build only the bank's pooled-key image and time the "
                         "selection alone; prefill: pooling and selection without V, O or the "
                         "attention workspace (small footprints for profiling captures; the "
                         "JSON line names it)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    args.default_set = args.workload is None
    if args.default_set:
        args.workload = "prefill_1m_b256_k16"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    # host workers for the oracle, forked before this process makes its first CUDA call
    pool = None
    if rank == 0 and (args.impl == "reference" or (world == 1 and not args.no_cpu_baseline)):
        pool = OraclePool(OraclePool.cores())
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank, pool)
        else:
            run_ours(args, world, rank, local, pool)
    finally:
        if pool is not None:
            pool.close()
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
