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


def test_down_algorithmic_bytes_at_v3_prefill():
    # Down weights of 220 touched + 1 shared expert, h read for T*(k+S) rows, block-
    # scaled fp16 y_perm written for the T*k routed and T shared rows (2 bytes per
    # value, 224 scale bytes per row at H = 7168).
    s = V3_PREFILL
    want = 221 * 7168 * 2048 * 2 + 16384 * 9 * 2048 * 2 + (16384 * 8 + 16384) * (2 * 7168 + 224)
    assert bench.down_algorithmic_bytes(s, 220) == want


def test_load_stats():
    s = TINY
    idx = torch.zeros((s.T, s.k), dtype=torch.int32)
    idx[:, 1], idx[:, 2], idx[:, 3] = 1, 2, 3
    st = bench.load_stats(s, idx.numpy(), histogram=True)
    assert st["experts_touched"] == 4 and st["max_rows"] == s.T
    assert st["max_over_mean"] == s.T / (s.T * s.k / s.E)
    assert st["rows_per_expert"][:4] == [s.T] * 4 and sum(st["rows_per_expert"]) == s.T * s.k


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    sha = bench.gemm_sources_sha1("bf16")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("bf16", "gate_up"),
                        {"sources_sha1": sha, "case": "v3_e32", "dram_bytes": 1100, "algorithmic_bytes": 1000})
    f = bench.traffic_fields("gate_up", 5000, "bf16")
    assert f["traffic_ratio"] == 1.1 and f["traffic"] == 5500 and f["algorithmic_bytes"] == 5000
    monkeypatch.delitem(bench.MEASURED_TRAFFIC, ("bf16", "down"), raising=False)
    assert bench.traffic_fields("down", 5000, "bf16")["traffic"] is None     # never captured
    # A kernel source that changed since the capture voids the stored figure.
    monkeypatch.setitem(bench.GEMM_SOURCES, "bf16", ("grouped_gemm.cuh", "router.cuh"))
    assert bench.traffic_fields("gate_up", 5000, "bf16")["traffic"] is None


def test_stored_captures_match_the_current_sources():
    # The stored DRAM captures were taken on the kernels in the tree: the bench reports them.
    for (prec, kernel) in bench.MEASURED_TRAFFIC:
        assert bench.traffic_ratio(kernel, prec) is not None, (prec, kernel)


def test_host_cpu_reports_cores():
    h = bench.host_cpu()
    assert h["host_cores"] >= 1
