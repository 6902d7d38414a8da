"""Host-side arithmetic of bench.py (CPU): algorithmic bytes, the whole-job
throughput, and the rule that a stored DRAM-traffic figure is reported only while
the GEMM sources hash to the ones it was captured on."""
import torch

import bench
from sparse_moe_layer_noaux_b200.workloads import TINY, V3_DECODE, V3_PREFILL


def test_gate_up_algorithmic_bytes_at_v3_prefill():
    # Gate and up weights of 256 routed + 1 shared expert, the T*k gathered rows plus
    # the T shared rows read, h written for T*(k+S) rows (bf16 throughout).
    s = V3_PREFILL
    want = 257 * 2 * 2048 * 7168 * 2 + (16384 * 8 + 16384) * 7168 * 2 + 16384 * 9 * 2048 * 2
    assert bench.gate_up_algorithmic_bytes(s, 256) == want
    assert abs(want / 1e9 - 17.809) < 1e-3


def test_layer_bytes_count_touched_experts_router_and_io():
    s = V3_DECODE
    idx = torch.tensor([[0, 1, 2, 3, 4, 5, 6, 7], [0, 1, 2, 3, 4, 5, 6, 8]], dtype=torch.int32)
    b, touched = bench.layer_bytes(s, idx)
    assert touched == 9
    per_expert = 3 * s.H * s.I * 2
    assert b == 9 * per_expert + per_expert * s.S + 4 * s.E * s.H + 2 * s.T * s.H + 4 * s.T * s.H
    bm, tm = bench.layer_bytes_mx(s, idx)
    assert tm == 9 and bm < b   # E4M3 weights: about half the bytes


def test_job_throughput_counts_every_rank_over_the_slowest():
    assert bench.job_throughput(TINY.T, 1, 2.0) == TINY.T / 2e-3
    assert bench.job_throughput(100, 4, 10.0) == 400 / 10e-3
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    for prec in ("bf16", "mxfp8"):
        m = bench.MEASURED_TRAFFIC[(prec, "v3_prefill")]
        assert bench.measured_traffic("v3_prefill", prec) == m["dram_read"] + m["dram_write"]
        assert bench.measured_traffic("v3_decode", prec) is None     # never captured
    # A kernel source that changed since the capture voids the stored figure.
    monkeypatch.setitem(bench.GEMM_SOURCES, "bf16", ("grouped_gemm.cuh", "router.cuh"))
    assert bench.measured_traffic("v3_prefill", "bf16") is None
