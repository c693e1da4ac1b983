"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): max-over-ranks timing,
one JSON line from rank 0, every rank exits cleanly."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    m = bench.max_over_ranks(float(rank + 1) * 1.5, w)
    bench.barrier(w)
    out[rank] = m
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert dict(out) == {0: 3.0, 1: 3.0}


@pytest.mark.parametrize("workload", [["prefill_tiny_s1k_f32"],
                                      ["decode_bank10m_b64_k32", "--seq", "100000"]],
                         ids=["prefill", "decode"])
def test_reference_arm_under_torchrun_prints_one_line(workload):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", *workload, "--steps", "1", "--warmup", "3",
           "--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _split_worker(rank, world, port, out):
    """One rank of the KV-group split: the oracle on this rank's head slice of one
    sequence, gathered over gloo in rank order."""
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import msa_inputs as mi
    import oracle
    from block_sparse_top_mean_b200.memory_parallel import _all_gather
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w = mi.Workload("split", "prefill", 1, 192, 8, 4, 16, 16, 4, "f32")
        q, k, v = mi.prefill_inputs(w)
        wl = bench.kv_group_split(w, rank, world)
        G = w.hq // w.hkv
        g0, g1 = rank * wl.hkv, (rank + 1) * wl.hkv
        ql, kl, vl = (x.numpy() for x in (q[:, :, g0 * G:g1 * G], k[:, :, g0:g1], v[:, :, g0:g1]))
        rows = oracle.prefill_rows(ql, kl, vl, w.block, w.topk, w.scale)
        O = np.zeros((w.seq, wl.hq, w.d))
        for r in rows:
            O[r.t, r.g * G:(r.g + 1) * G] = r.O
        allO = _all_gather(torch.from_numpy(O))           # [world, S, hq/world, d]
        full = torch.cat(list(allO), dim=1).numpy()       # heads in rank order
        ref = oracle.prefill_rows(q.numpy(), k.numpy(), v.numpy(), w.block, w.topk, w.scale)
        Ofull = np.zeros((w.seq, w.hq, w.d))
        for r in ref:
            Ofull[r.t, r.g * G:(r.g + 1) * G] = r.O
        af, sf = bench.prefill_flops(w)
        al, sl = bench.prefill_flops(wl)
        out[rank] = (float(np.abs(full - Ofull).max()), (al + sl) * world == af + sf)
    finally:
        dist.destroy_process_group()


def test_kv_group_split_reassembles_the_sequence():
    """bench.py --gpus N splits one sequence by KV group: the ranks' outputs, gathered in
    rank order, are the whole sequence's, and world x a rank's FLOPs is the sequence's."""
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_split_worker, args=(2, port, out), nprocs=2, join=True)
    for rank in range(2):
        err, flops_ok = out[rank]
        assert err == 0.0 and flops_ok
