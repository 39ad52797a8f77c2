"""The measurement's arithmetic, on CPU: the unmasked-pair counts and FLOP
totals the benchmark divides by, checked against a brute-force count of the
band mask and against the closed forms of the windowed causal mask; and the
bench's helpers that need no GPU."""
import json
import os
import sys

import numpy as np
import pytest

import causal_sliding_window_rope_b200 as cs

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def brute_pairs(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return int(((j <= i) & (j > i - W)).sum())


@pytest.mark.parametrize("T,W", [(16, 16), (16, 1), (37, 5), (2048, 1024), (2048, 2048), (300, 4000)])
def test_pairs_match_the_band_mask(T, W):
    w = cs.Workload(0, "t", B=1, T=T, H=1, Hk=1, D=8, windows=[W], ve=[False], dtype="bf16")
    assert w.pairs(W) == brute_pairs(T, W)


def test_d24_and_long_context_totals():
    # d24 SSSL: 3 layers of W=1024 and one of W=2048 at T=2048, B=4, H=12, D=128.
    w = cs.WORKLOADS[4]
    assert w.pairs(1024) == 1024 * 1025 // 2 + 1024 * 1024 == 1_573_376
    assert w.pairs(2048) == 2048 * 2049 // 2 == 2_098_176
    assert w.flops() == 12 * 128 * 4 * 12 * (3 * 1_573_376 + 2_098_176) == 502_699_917_312
    assert w.flops("flash") == w.flops() * 14 / 12
    # long context: W=2048 x3 and W=8192 at T=8192, B=1, H=16.
    w5 = cs.WORKLOADS[5]
    assert w5.pairs(2048) == 14_681_088 and w5.pairs(8192) == 33_558_528
    # the fp32 microgpt layer: full causal, T=16.
    assert cs.WORKLOADS[1].pairs(16) == 136


def test_bench_reduce_max_single_process():
    import torch
    assert bench.reduce_max([1.5, 2.0], None, torch.device("cpu")) == [1.5, 2.0]


def test_bench_peaks_and_workload_description():
    peaks, src = bench.load_peaks()
    assert peaks["hbm_gbs"] > 0 and peaks["bf16_tflops_sustained"] > 0
    if os.path.exists(os.path.join(os.path.dirname(bench.__file__), "MEASURED_PEAKS.json")):
        assert src == "measured"
    desc = bench.workload_desc(cs.WORKLOADS[4])
    assert "B=4" in desc and "T=2048" in desc and "H=12" in desc and "Hk=4" in desc


def test_traffic_table_is_keyed_by_kernel_sources():
    path = os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")
    table = json.load(open(path))
    for kind in ("fwd", "bwd", "prologue", "bwd_pre", "bwd_epi"):
        ent = table[kind]
        assert ent["bytes_per_launch"] == pytest.approx(ent["read"] + ent["write"])
        assert len(ent["source_sha"]) == 16
        # the table is used only while the kernel sources are unchanged
        assert bench.traffic_for(kind) in (None, ent["bytes_per_launch"])
