"""The benchmark's work accounting, checked against brute-force counts on small shapes:
the attention and scoring FLOPs a prefill pass is credited with, its selected entries,
the decode byte and FLOP figures, the kernel-launch counts of a decode selection, and
the roofline denominators read from the measured peaks."""
import json
import os

import numpy as np

import bench
import msa_inputs as mi


def _brute_prefill(w):
    attn = score = entries = 0
    for t in range(w.seq):
        i = t // w.block
        past = min(w.topk - 1, i)                    # full past blocks attended
        keys = past * w.block + (t - i * w.block + 1)
        attn += keys * w.hq * 4 * w.d
        score += i * w.hkv * 2 * w.d                 # every past block is scored
        entries += (past + 1) * w.hkv                # past blocks + the own block
    return attn * w.batch, score * w.batch, entries * w.batch


def test_prefill_flops_and_entries_match_brute_force():
    for w in (mi.Workload("a", "prefill", 1, 1000, 8, 2, 64, 64, 4, "bf16"),
              mi.Workload("b", "prefill", 2, 777, 4, 4, 128, 128, 16, "bf16"),
              mi.Workload("c", "prefill", 1, 300, 2, 1, 64, 256, 1, "f32")):
        attn, score, entries = _brute_prefill(w)
        a, s = bench.prefill_flops(w)
        assert (a, s) == (float(attn), float(score))
        assert bench.prefill_entries(w) == entries


def test_headline_prefill_flops():
    # the 1M headline: 6.80e13 attention and 4.40e12 scoring FLOPs per pass
    a, s = bench.prefill_flops(mi.WORKLOADS["prefill_1m_b256_k16"])
    assert abs(a - 6.80e13) / 6.80e13 < 5e-3
    assert abs(s - 4.40e12) / 4.40e12 < 5e-3


def test_decode_work():
    w = mi.Workload("d", "decode", 1, 10_000, 32, 8, 128, 64, 32, "bf16", n_query=4)
    d = bench.decode_work(w)
    nb = -(-10_000 // 64)
    assert d["score_bytes"] == nb * 8 * 128 * 2                 # one bf16 plane
    assert d["attn_bytes"] == 4 * 8 * 32 * 64 * 128 * 2 * 2     # K and V of the selection
    assert d["score_flops"] == 4 * 8 * 2 * 128 * nb
    assert d["attn_flops"] == 4 * 32 * 4 * 128 * 32 * 64
    few = mi.Workload("e", "decode", 1, 640, 8, 2, 64, 64, 32, "bf16", n_query=1)
    assert bench.decode_work(few)["attn_bytes"] == 1 * 2 * 10 * 64 * 64 * 2 * 2   # 10 blocks


def test_decode_selection_launch_counts():
    # sample pass + threshold from 128 chunks of 128 blocks per group, else 5 launches
    assert bench.select_launches(127 * 128 + 1) == 7              # 128 chunks (the last partial)
    assert bench.select_launches(127 * 128) == 5
    assert bench.select_launches(156_250) == 7                  # the 10M-token bank


def test_peaks_come_from_the_measured_file():
    peaks, src = bench.load_peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        assert src == "measured"
        assert peaks["hbm_gbs"] == float(d["hbm_gbs"])
        assert peaks["bf16_tflops_sustained"] == float(d["bf16_tflops_sustained"])
    else:
        assert src == "fallback"
    assert all(np.isfinite(v) and v > 0 for v in peaks.values())
