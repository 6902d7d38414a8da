"""Benchmark of the DeepSeekMoE layer forward (noaux_tc routing) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3_prefill]
    python bench.py --impl reference ...      # the float64 CPU oracle arm

One step = one pass of the whole layer (route, dispatch, gate/up GEMM with
SwiGLU, down GEMM, combine) over one batch of T synthetic tokens, inputs
resident in HBM.  Expert weights (22.5 GB at the V3 shape) exceed the 126 MB
L2 many times over, so every step streams them from HBM.  Under torchrun each
rank runs its own batch with replicated weights (weak scaling; no collective
on the data path); the time is the max over ranks.  Rank 0 prints ONE JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_moe_layer_noaux_b200 import MoELayer, MoELayerMX, abi  # noqa: E402
from sparse_moe_layer_noaux_b200.workloads import WORKLOADS, bf16_bits, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOP/s at V3 shape (T=128, 16384); % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of the expert GEMMs.  The V3 workloads hold 22.5 GB of expert weights,
# beyond the size of an ncu capture on this pool, so the counters
# (dram__bytes_read.sum + dram__bytes_write.sum, one pass) are taken on the 32-expert
# V3 case (v3_e32: T = 4096, 2.8 GB of weights), whose launches walk their segments
# in the same orders as the full workload (expert segments of a few row tiles column
# by column, the shared segment row by row).  A launch's traffic is reported as that
# case's measured traffic / algorithmic-bytes ratio times the launch's own algorithmic
# bytes, and only while the kernel sources hash to the value the capture was taken on
# (profiles/ holds the capture and its command).
GEMM_SOURCES = {"bf16": ("grouped_gemm.cuh", "sm100_ptx.cuh", "device_status.cuh"),
                "mxfp8": ("grouped_gemm_mx.cuh", "mx.cuh", "grouped_gemm.cuh", "sm100_ptx.cuh",
                          "device_status.cuh")}
# (precision, "gate_up" | "down") -> the capture: the kernel sources' hash, the case, DRAM read + write bytes
# of its second-pass launch and that launch's algorithmic bytes (profiles/grouped_gemm_dram_v3_e32.md).
MEASURED_TRAFFIC = {
    ("bf16", "gate_up"): {"sources_sha1": "dfe7b14e204d9c05afd92a3faf768704c4c2c7a3", "case": "v3_e32",
                          "dram_bytes": 2961000000, "algorithmic_bytes": 2617245696},
    ("bf16", "down"): {"sources_sha1": "dfe7b14e204d9c05afd92a3faf768704c4c2c7a3", "case": "v3_e32",
                       "dram_bytes": 1630800000, "algorithmic_bytes": 1656619008},
    ("mxfp8", "gate_up"): {"sources_sha1": "bb9dc3c4638fe4c5e2905a82c02fe5ac54182cb6", "case": "v3_e32",
                           "dram_bytes": 1367600000, "algorithmic_bytes": 1349517312},
}


def gemm_sources_sha1(precision="bf16"):
    import hashlib
    h = hashlib.sha1()
    for f in GEMM_SOURCES[precision]:
        with open(os.path.join(ROOT, "sparse_moe_layer_noaux_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_ratio(kernel, precision="bf16"):
    """Measured DRAM bytes / algorithmic bytes of a captured launch of `kernel`
    ("gate_up" or "down"), or None when no capture matches the current sources."""
    m = MEASURED_TRAFFIC.get((precision, kernel))
    if m is None or m["sources_sha1"] != gemm_sources_sha1(precision):
        return None
    return m["dram_bytes"] / m["algorithmic_bytes"]


def traffic_fields(kernel, algorithmic, precision="bf16"):
    """The roofline's traffic keys for one launch with `algorithmic` bytes."""
    r = traffic_ratio(kernel, precision)
    m = MEASURED_TRAFFIC.get((precision, kernel))
    return {"algorithmic_bytes": algorithmic,
            "traffic": None if r is None else int(r * algorithmic),
            "traffic_ratio": r,
            "traffic_source": None if r is None else
            f"ncu dram__bytes_read.sum + dram__bytes_write.sum on {m['case']}: "
            f"{m['dram_bytes']} B against {m['algorithmic_bytes']} algorithmic B, ratio x this launch's bytes"}


def _routed_rows(shape):
    return shape.T * shape.k + (shape.T if shape.S else 0)


def gate_up_algorithmic_bytes(shape, touched, elt=2.0):
    """Compulsory HBM bytes of one gate/up launch: gate and up weights of the touched
    routed experts and of the shared experts, the T*k gathered rows and the T token
    rows they read, and the h rows written (T*(k+S) x I).  `elt` is bytes per
    element (2 for bf16; 1 + 1/32 for MXFP8: E4M3 bytes plus one scale per 32)."""
    w = (touched + shape.S) * 2 * shape.I * shape.H * elt
    a = _routed_rows(shape) * shape.H * elt
    h = shape.T * (shape.k + shape.S) * shape.I * elt
    return int(w + a + h)


def down_algorithmic_bytes(shape, touched, elt=2.0):
    """Compulsory HBM bytes of one down launch: down weights of the touched routed
    experts and of the shared experts, the h rows read, and the block-scaled fp16
    y_perm rows written (2 bytes per value plus one scale byte per 32, rows padded
    to 8 scale bytes)."""
    w = (touched + shape.S) * shape.H * shape.I * elt
    h = shape.T * (shape.k + shape.S) * shape.I * elt
    y = _routed_rows(shape) * (2 * shape.H + (shape.H // 32 + 7) // 8 * 8)
    return int(w + h + y)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """Max of a per-rank scalar over all ranks (the step time the job is bound by)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(shape, rank, device):
    """Weights replicated on every rank (same seed); each rank its own tokens."""
    inp = make_inputs(shape, device)
    if rank:
        g = torch.Generator(device=device)
        g.manual_seed(shape.seed * 1000 + rank)
        inp["x"] = torch.randn((shape.T, shape.H), generator=g, device=device).to(torch.bfloat16)
    return inp


def job_throughput(tokens_per_rank, world, ms_max):
    """Whole-job tokens/s: the units all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.rows = []
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------- GPU arm
class StagedStep:
    """One layer step as its five C-ABI stages, with CUDA events between them
    on the launching stream (same kernels and order as moe_forward)."""

    NAMES = ("route", "dispatch", "gate_up", "down", "combine")

    def __init__(self, shape, inp):
        self.shape, self.inp = shape, inp
        T, k, E, H, I, S = shape.T, shape.k, shape.E, shape.H, shape.I, shape.S
        d = inp["x"].device
        self.cfg = abi.MoEConfig.from_shape(shape)
        self.ws = torch.empty(abi.workspace_size(self.cfg, T), dtype=torch.uint8, device=d)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=d)
        self.w = torch.empty((T, k), dtype=torch.float32, device=d)
        self.off = torch.empty(E + 1, dtype=torch.int32, device=d)
        self.x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=d)
        self.perm_src = torch.empty(T * k, dtype=torch.int32, device=d)
        self.row_of = torch.empty((T, k), dtype=torch.int32, device=d)
        self.h_r = torch.empty((T * k, I), dtype=torch.bfloat16, device=d)
        self.h_s = torch.empty((T, max(S * I, 8)), dtype=torch.bfloat16, device=d)
        self.y_perm = torch.empty((T * k + T, H), dtype=torch.float16, device=d)
        self.y_sc = torch.empty((T * k + T, abi.y_perm_scale_cols(H)), dtype=torch.uint8, device=d)
        self.y = torch.empty((T, H), dtype=torch.float32, device=d)

    def run(self, events=None):
        s, i, T = self.shape, self.inp, self.shape.T
        ev = events or [None] * 6

        def rec(j):
            if ev[j] is not None:
                ev[j].record()
        rec(0)
        abi.moe_route(self.cfg, i["x"], i["router_w"], i["e_bias"], self.idx, self.w, self.ws)
        rec(1)
        abi.moe_dispatch(self.cfg, i["x"], self.idx, self.off, self.x_perm, self.perm_src, self.row_of, self.ws)
        rec(2)
        abi.moe_experts_gate_up(self.cfg, T, i["x"], self.x_perm, self.off, i["w_gate"], i["w_up"],
                                i["ws_gate"], i["ws_up"], self.h_r, self.h_s)
        rec(3)
        abi.moe_experts_down(self.cfg, T, self.h_r, self.h_s, self.off, self.perm_src, self.w, i["w_down"],
                             i["ws_down"], self.y_perm, self.y_sc)
        rec(4)
        abi.moe_combine(self.cfg, T, self.y_perm, self.y_sc, self.row_of, self.y)
        rec(5)


class StagedStepMX:
    """The MXFP8 layer step as its C-ABI stages (route, dispatch with quantisation,
    gate/up, down, combine), events between them; the weights are quantised once
    at construction, outside any timed region."""

    NAMES = StagedStep.NAMES

    def __init__(self, shape, inp):
        self.shape, self.inp = shape, inp
        T, k, E, H, I, S = shape.T, shape.k, shape.E, shape.H, shape.I, shape.S
        d = inp["x"].device
        self.cfg = abi.MoEConfig.from_shape(shape)
        self.layer = MoELayerMX.from_inputs(shape, inp)
        rp, tp = abi.mx_routed_rows(self.cfg, T), (T + 127) // 128 * 128
        self.rp = rp
        n_ws = max(abi.workspace_size_mx(self.cfg, T), abi.workspace_size(self.cfg, T))
        self.ws = torch.empty(n_ws, dtype=torch.uint8, device=d)
        u8 = lambda *sh: torch.empty(sh, dtype=torch.uint8, device=d)
        i32 = lambda *sh: torch.empty(sh, dtype=torch.int32, device=d)
        self.idx, self.w = i32(T, k), torch.empty((T, k), dtype=torch.float32, device=d)
        self.off, self.cnt, self.perm_src, self.row_of = i32(E + 1), i32(E), i32(rp), i32(T, k)
        self.xq, self.xsf = u8(rp, H), u8(abi.mx_scale_bytes(rp, H))
        self.xqs, self.xssf = u8(tp, H), u8(max(abi.mx_scale_bytes(tp, H), 16))
        self.hq, self.hsf = u8(rp, I), u8(abi.mx_scale_bytes(rp, I))
        self.hqs, self.hssf = u8(tp, max(S * I, 128)), u8(max(abi.mx_scale_bytes(tp, max(S * I, 128)), 16))
        self.y_perm = torch.empty((rp + T, H), dtype=torch.float16, device=d)
        self.y_sc = u8(rp + T, abi.y_perm_scale_cols(H))
        self.y = torch.empty((T, H), dtype=torch.float32, device=d)

    def run(self, events=None):
        i, T, L = self.inp, self.shape.T, self.layer
        ev = events or [None] * 6

        def rec(j):
            if ev[j] is not None:
                ev[j].record()
        rec(0)
        abi.moe_route(self.cfg, i["x"], i["router_w"], i["e_bias"], self.idx, self.w, self.ws)
        rec(1)
        abi.moe_dispatch_mx(self.cfg, i["x"], self.idx, self.off, self.cnt, self.xq, self.xsf, self.xqs, self.xssf,
                            self.perm_src, self.row_of, self.ws)
        rec(2)
        abi.moe_experts_gate_up_mx(self.cfg, T, self.xq, self.xsf, self.xqs, self.xssf, self.off, self.cnt,
                                   L.weights, self.hq, self.hsf, self.hqs, self.hssf)
        rec(3)
        abi.moe_experts_down_mx(self.cfg, T, self.hq, self.hsf, self.hqs, self.hssf, self.off, self.cnt,
                                self.perm_src, self.w, L.weights, self.y_perm, self.y_sc)
        rec(4)
        abi.moe_combine_mx(self.cfg, T, self.y_perm, self.y_sc, self.row_of, self.y)
        rec(5)


def layer_bytes_mx(shape, idx):
    """Algorithmic bytes of one MXFP8 step: E4M3 weights of the touched routed experts
    and the shared experts (1 byte per element + one scale byte per 32), the fp32
    router, and x (bf16) in and y (fp32) out."""
    touched = int(torch.unique(idx).numel())
    b = (touched + shape.S) * 3 * shape.H * shape.I * (1 + 1 / 32)
    b += 4 * shape.E * shape.H + 2 * shape.T * shape.H + 4 * shape.T * shape.H
    return int(b), touched


def time_gpu_mx(shape, steps, warmup, world, rank, peaks, inp=None):
    """The MXFP8 layer: staged step timed like the bf16 one, and moe_forward_mx alone."""
    inp = inp if inp is not None else rank_inputs(shape, rank, "cuda")
    st = StagedStepMX(shape, inp)
    for _ in range(warmup):
        st.run()
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    torch.cuda.synchronize()
    for j in range(steps):
        st.run(evs[j])
    torch.cuda.synchronize()
    stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i, name in enumerate(StagedStepMX.NAMES)}
    staged_ms = statistics.mean(e[0].elapsed_time(e[5]) for e in evs)
    assert abi.device_status() == 0
    y = torch.empty(inp["x"].shape, dtype=torch.float32, device=inp["x"].device)
    ms, launches, clk = time_steps(lambda: st.layer(inp["x"], y), steps, warmup, world)
    fwd_ms = ms
    fp8_peak = 2.0 * peaks["bf16_tflops"]  # nominal dense fp8 / bf16 ratio (4.5 / 2.25) x measured bf16
    flops = shape.flops()
    lbytes, touched = layer_bytes_mx(shape, st.idx)
    t_roof = max(flops / (fp8_peak * 1e12), lbytes / (peaks["hbm_gbs"] * 1e9))
    gu_ms = stage_ms["gate_up"]
    gu_flops = 4.0 * shape.H * shape.I * shape.T * (shape.k + shape.S)
    out = {
        "ms_per_step": ms, "tokens_per_s": job_throughput(shape.T, world, ms), "stage_ms": stage_ms,
        "staged_ms": staged_ms, "forward_ms": fwd_ms, "tflops": flops / (ms * 1e-3) / 1e12 * world, "gpu_launches": launches,
        "experts_touched": touched, "layer_bytes": lbytes,
        "layer_roofline": {"bound": "tensor" if flops / (fp8_peak * 1e12) >= lbytes / (peaks["hbm_gbs"] * 1e9)
                           else "hbm", "roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms},
        "roofline": {"kernel": "grouped_gemm_mx_kernel<kSwiGLU> (MXFP8 gate/up + SwiGLU + h quantisation)",
                     "bound": "tensor", "achieved": gu_flops / (gu_ms * 1e-3) / 1e12, "peak": fp8_peak,
                     "unit": "TFLOP/s", "frac": gu_flops / (gu_ms * 1e-3) / 1e12 / fp8_peak,
                     "peak_source": "measured bf16 burst x 2 (nominal dense fp8/bf16 ratio)",
                     **traffic_fields("gate_up", gate_up_algorithmic_bytes(shape, touched, 1 + 1 / 32), "mxfp8"),
                     "ms_per_launch": gu_ms},
        "clocks": clk,
    }
    del st
    return out


def time_backward(shape, steps, warmup, world, rank, peaks, inp):
    """moe_backward (gradients of sum(y * dy) for x, the router weight and every
    expert weight) on the same workload, K calls timed like the forward."""
    layer = MoELayer.from_inputs(shape, inp)
    g = torch.Generator(device="cuda").manual_seed(shape.seed + 99)
    dy = torch.randn((shape.T, shape.H), device="cuda", generator=g).bfloat16()
    grads = layer.backward(inp["x"], dy)  # allocates the gradients and the workspace once
    cfg = layer.cfg
    ws = layer._ws_bwd

    def step():
        abi.moe_backward(cfg, inp["x"], layer.router_w, layer.e_bias, layer.w_gate, layer.w_up, layer.w_down,
                         layer.ws_gate, layer.ws_up, layer.ws_down, dy, grads["x"], grads["router_w"],
                         grads["w_gate"], grads["w_up"], grads["w_down"], grads.get("ws_gate"), grads.get("ws_up"),
                         grads.get("ws_down"), ws)
    ms, launches, clk = time_steps(step, steps, warmup, world)

    # Training step: moe_forward_train (keeps routing, rows, g | u) + moe_backward_train.
    y = torch.empty(inp["x"].shape, dtype=torch.float32, device="cuda")
    layer.forward_train(inp["x"], y)

    def train_step():
        layer.forward_train(inp["x"], y)
        layer.backward_train(inp["x"], dy, grads)
    train_ms, train_launches, train_clk = time_steps(train_step, steps, warmup, world)
    # recompute g,u (4), dh (2), dx (4), dWd (2), dWg + dWu (4): 16 H I per (token, expert) pair
    flops = 16.0 * shape.H * shape.I * shape.T * (shape.k + shape.S) + 4.0 * shape.T * shape.E * shape.H
    # weights read (gate/up twice, down twice), weight gradients written (bf16)
    touched = int(torch.unique(layer_route_idx(shape, inp)).numel())
    wbytes = (touched + shape.S) * 3 * shape.H * shape.I * 2
    bytes_ = 2 * wbytes + wbytes + 2 * 2 * shape.T * shape.H + 4 * shape.T * shape.H
    t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9))
    out = {"ms_per_step": ms, "tokens_per_s": job_throughput(shape.T, world, ms),
           "tflops": flops / (ms * 1e-3) / 1e12 * world, "flops": flops, "gpu_launches": launches,
           "layer_roofline": {"bound": "tensor" if flops / (peaks["bf16_tflops"] * 1e12) >= bytes_ / (peaks["hbm_gbs"] * 1e9)
                              else "hbm", "roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms},
           "clocks": clk,
           "training_step": {"ms_per_step": train_ms, "tokens_per_s": job_throughput(shape.T, world, train_ms),
                             "what": "moe_forward_train + moe_backward_train (g, u kept, not recomputed)",
                             "tflops": (6.0 * shape.H * shape.I * shape.T * (shape.k + shape.S) + flops
                                        - 4.0 * shape.H * shape.I * shape.T * (shape.k + shape.S))
                             / (train_ms * 1e-3) / 1e12 * world,
                             "gpu_launches": train_launches, "clocks": train_clk}}
    del grads, layer
    return out


def time_ep(shape, steps, warmup, world, rank, inp):
    """The expert-parallel layer (MoELayerEP): each rank holds E/world of the routed
    experts and its own T tokens; a token's row goes once to each rank holding one of
    its experts and its sum comes back, by the process group's all-to-all.  At world 1 (no torchrun) a one-rank NCCL group is
    formed here, so the same code path runs with the exchanges as local copies."""
    import datetime
    import socket
    import torch.distributed as dist
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP, expert_block
    own = not dist.is_initialized()
    if own:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
        dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                                device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        layer = MoELayerEP(shape, world, rank, inp["router_w"], inp["e_bias"],
                           expert_block(inp["w_gate"], world, rank), expert_block(inp["w_up"], world, rank),
                           expert_block(inp["w_down"], world, rank), inp["ws_gate"], inp["ws_up"], inp["ws_down"])
        ms, launches, clk = time_steps(lambda: layer(inp["x"]), steps, warmup, world)
        st = layer.send(inp["x"])
        torch.cuda.synchronize()
        sent_rows = int(st.send_counts.sum().item())
    finally:
        if own:
            dist.destroy_process_group()
    return {"ms_per_step": ms, "tokens_per_s": job_throughput(shape.T, world, ms), "world": world,
            "experts_per_rank": shape.E // world, "gpu_launches": launches, "clocks": clk,
            "rows_sent_per_rank": sent_rows, "rows_sent_per_token": round(sent_rows / max(shape.T, 1), 3),
            "what": "MoELayerEP.forward: route, send rows (one per token and destination rank), all-to-all "
                    "of counts and rows, local sort and expert GEMMs on the received rows, per-row sums, "
                    "all-to-all of the sums back, combine"}


def layer_route_idx(shape, inp):
    cfg = abi.MoEConfig.from_shape(shape)
    ws = torch.empty(abi.workspace_size(cfg, shape.T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    return idx


def layer_bytes(shape, idx):
    """Algorithmic bytes of one step: bf16 weights of the touched routed experts and the
    shared experts, the fp32 router, and x (bf16) in and y (fp32) out."""
    touched = int(torch.unique(idx).numel())
    b = touched * 3 * shape.H * shape.I * 2 + 3 * shape.H * shape.S * shape.I * 2
    b += 4 * shape.E * shape.H + 2 * shape.T * shape.H + 4 * shape.T * shape.H
    return b, touched


def load_stats(shape, idx, histogram=False):
    """Per-expert load of one routed batch: rows per expert against the mean T*k/E."""
    counts = np.bincount(idx.reshape(-1).astype(np.int64), minlength=shape.E)
    mean = shape.T * shape.k / shape.E
    out = {"experts_touched": int((counts > 0).sum()), "max_rows": int(counts.max()),
           "mean_rows": mean, "max_over_mean": float(counts.max() / mean),
           "min_rows_touched": int(counts[counts > 0].min()) if counts.any() else 0,
           "segments_le_112_rows": int(((counts > 0) & (counts <= 112)).sum())}
    if histogram:
        out["rows_per_expert"] = counts.tolist()
    return out


def time_gpu(shape, steps, warmup, world, rank, peaks, flush_note=True):
    inp = rank_inputs(shape, rank, "cuda")
    st = StagedStep(shape, inp)
    for _ in range(warmup):
        st.run()
    torch.cuda.synchronize()
    assert abi.device_status() == 0

    # Stage breakdown: the five C-ABI stages in sequence, events between them.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    torch.cuda.synchronize()
    for j in range(steps):
        st.run(evs[j])
    torch.cuda.synchronize()
    stage_ms = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i, name in enumerate(StagedStep.NAMES)}
    staged_ms = statistics.mean(e[0].elapsed_time(e[5]) for e in evs)
    assert abi.device_status() == 0

    # The step: one moe_forward call (the public entry point).
    layer = MoELayer.from_inputs(shape, inp)
    y = torch.empty(inp["x"].shape, dtype=torch.float32, device=inp["x"].device)
    ms, launches, clk = time_steps(lambda: layer(inp["x"], y), steps, warmup, world)
    fwd_ms = ms
    # Small batches are launch-bound: the same call replayed from a CUDA graph.
    graph_ms = time_graph(lambda: layer(inp["x"], y), steps, world) if shape.T <= 4096 else None

    flops = shape.flops()
    lbytes, touched = layer_bytes(shape, st.idx)
    t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), lbytes / (peaks["hbm_gbs"] * 1e9))
    idx_h = st.idx.cpu().numpy()
    res = {
        "ms": ms, "stage_ms": stage_ms, "staged_ms": staged_ms, "forward_ms": fwd_ms, "launches": launches,
        "tflops": flops / (ms * 1e-3) / 1e12, "layer_bytes": lbytes, "experts_touched": touched,
        "layer_roofline": {"bound": "tensor" if flops / (peaks["bf16_tflops"] * 1e12) >=
                           lbytes / (peaks["hbm_gbs"] * 1e9) else "hbm",
                           "roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms,
                           "hbm_gbs_achieved": lbytes / (ms * 1e-3) / 1e9},
        "graph_ms": graph_ms, "clocks": clk, "st": st, "inp": inp, "layer": layer, "idx": idx_h,
        "load": load_stats(shape, idx_h, histogram=shape.bias_kind == "zipf"),
        "routing_inputs": (bf16_bits(inp["x"]), inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()),
    }
    return res


def time_graph(step, steps, world):
    """step() captured once in a CUDA graph (after a warm-up call on the capture's
    side stream) and replayed exactly `steps` times between synchronizes; CUDA events,
    max over ranks.  The launches of a serving loop that replays a fixed shape."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    assert abi.device_status() == 0
    del g
    return max_over_ranks(e0.elapsed_time(e1) / steps, world)


def time_steps(step, steps, warmup, world):
    """Exactly `steps` calls of step() between a barrier + synchronize on both sides,
    CUDA events on the current stream, clocks sampled meanwhile; max over ranks."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    n0 = abi.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    launches = abi.launch_count() - n0
    barrier(world)
    assert abi.device_status() == 0
    return max_over_ranks(e0.elapsed_time(e1) / steps, world), launches, clk.summary()


E2E_CHUNKS = 2  # chunks of the batch in the host-buffer forward (copies overlap the layer)


def time_e2e(layer, shape, steps, chunks=E2E_CHUNKS):
    """The public host-buffer call: pinned x on the host -> moe_forward_host (the batch
    in `chunks` chunks, each chunk's copy in and the previous chunk's copy out
    overlapping its computation) -> y back in pinned host memory, every step."""
    x_host = torch.empty((shape.T, shape.H), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(layer_inputs_host(shape))
    y_host = torch.empty(x_host.shape, dtype=torch.float32, pin_memory=True)
    chunk = (shape.T + chunks - 1) // chunks if chunks > 1 else 0
    for _ in range(2):
        layer.forward_host(x_host, y_host, chunk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        layer.forward_host(x_host, y_host, chunk)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return ms, x_host.numel() * x_host.element_size(), y_host.numel() * y_host.element_size()


def layer_inputs_host(shape):
    g = torch.Generator().manual_seed(shape.seed + 77)
    return torch.randn((shape.T, shape.H), generator=g).to(torch.bfloat16)


# ----------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(shape, inp, n_tokens, seed):
    """Time the float64 oracle (routing + shared + routed experts) on n_tokens rows.
    Expert weights are copied from the device one expert at a time; that copy time
    is excluded.  Returns (seconds of oracle work, rows)."""
    import oracle
    oracle.build()
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(shape.T, n_tokens, replace=False))
    x_bits = bf16_bits(inp["x"][torch.as_tensor(rows, device=inp["x"].device)])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    shared = None
    if shape.S:
        shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    fetch_s = [0.0]

    def fetch(e):
        t0 = time.perf_counter()
        r = (bf16_bits(inp["w_gate"][e]), bf16_bits(inp["w_up"][e]), bf16_bits(inp["w_down"][e]))
        fetch_s[0] += time.perf_counter() - t0
        return r
    t0 = time.perf_counter()
    oracle.moe_layer(shape, x_bits, rw, bias, fetch, shared)
    return time.perf_counter() - t0 - fetch_s[0], rows


def oracle_tokens_per_step(shape):
    per_token_macs = shape.E * shape.H + 3 * shape.H * shape.I * (shape.k + shape.S)
    # About half a second of float64 work, never more rows than the batch has.
    return max(1, min(shape.T, int(4e8 // per_token_macs)))


def host_cpu():
    """Host core count and CPU model (from /proc/cpuinfo when there is one)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def cpu_baseline(shape, inp, budget_tokens=None):
    n = budget_tokens or max(1, min(shape.T, 24 * oracle_tokens_per_step(shape)))
    secs, rows = oracle_sample(shape, inp, n, seed=99)
    return {"value": len(rows) / secs, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(rows)} of the {shape.T} tokens of the {shape.name} batch (seeded): "
                      f"routing, shared and routed SwiGLU experts in float64, 1 thread; "
                      f"expert-weight copies from the device excluded", **host_cpu()}


NEAR_TIE = 1e-4  # oracle margin below which two expert sets are equally correct in fp32


def oracle_routing_report(shape, routing_inputs, gpu_idx):
    """The float64 oracle router on every token of a workload (row blocks in spawned
    processes): its throughput, the near-tie count (tokens whose margin at the
    group-keep or top-k boundary is below 1e-4) and how many GPU expert sets differ
    from the oracle's (each allowed only on a near tie)."""
    import oracle
    from oracle.pool import route_rows
    oracle.build()
    x_bits, rw, bias = routing_inputs
    workers = max(1, min(16, os.cpu_count() or 1))
    t0 = time.perf_counter()
    ref_idx, _, margin, _ = route_rows(shape, x_bits, rw, bias, workers=workers)
    secs = time.perf_counter() - t0
    near = margin < NEAR_TIE
    differ = np.array([set(a.tolist()) != set(b.tolist()) for a, b in zip(gpu_idx, ref_idx)])
    return {"tokens": int(shape.T), "near_ties": int(near.sum()), "gpu_sets_differing": int(differ.sum()),
            "gpu_sets_differing_off_near_tie": int((differ & ~near).sum()),
            "oracle_routing_tokens_per_s": shape.T / secs, "oracle_processes": workers}


def bias_balancing(shape, inp, steps=60, gamma=0.05, every=10):
    """The aux-loss-free balancing loop on one batch: route (moe_route), nudge the bias
    by its load (moe_bias_update), repeat; the max / mean expert load every `every`
    steps.  Works on a copy of the bias."""
    cfg = abi.MoEConfig.from_shape(shape)
    bias = inp["e_bias"].clone()
    ws = torch.empty(abi.workspace_size(cfg, shape.T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    load = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    mean = shape.T * shape.k / shape.E
    trace = []
    for step in range(steps + 1):
        abi.moe_route(cfg, inp["x"], inp["router_w"], bias, idx, w, ws)
        abi.moe_bias_update(cfg, idx, bias, gamma if step < steps else 0.0, load)
        if step % every == 0:
            trace.append(round(float(load.max().item()) / mean, 3))
    assert abi.device_status() == 0
    return {"gamma": gamma, "steps": steps, "max_over_mean_every_10_steps": trace,
            "what": "moe_route + moe_bias_update repeated on the batch (the bias nudged down where an expert is "
                    "over the mean load, up where under)"}


def workload_summary(shape, r, world):
    """The nested bench object of one workload's forward."""
    return {"T": shape.T, "ms_per_step": r["ms"], "tokens_per_s": job_throughput(shape.T, world, r["ms"]),
            "tflops": r["tflops"] * world, "stage_ms": r["stage_ms"], "forward_ms": r["forward_ms"],
            "layer_roofline": r["layer_roofline"], "layer_bytes": r["layer_bytes"],
            "experts_touched": r["experts_touched"], "load": r["load"], "gpu_launches": r["launches"],
            "graph_ms_per_step": r["graph_ms"], "clocks": r["clocks"]}


def run_reference(args, shape, world, rank):
    """The oracle arm: the float64 oracle as it stands, timed on this host's cores on
    a bounded token sample per step (rank 0 only)."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(shape, dev)
    per = oracle_tokens_per_step(shape)
    for j in range(args.warmup):
        oracle_sample(shape, inp, per, seed=1000 + j)
    secs = 0.0
    for j in range(args.steps):
        s, _ = oracle_sample(shape, inp, per, seed=2000 + j)
        secs += s
    value = per * args.steps / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(shape, world),
        "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": "tokens/s",
                         "sample": f"{per} seeded tokens of the {shape.T}-token {shape.name} batch per "
                                   f"step: routing + shared + routed experts in float64, 1 thread"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(shape, world):
    return {"workload": f"{shape.name}: DeepSeekMoE layer, T={shape.T} tokens per GPU, hidden {shape.H}, "
                        f"{shape.E} routed experts (top-{shape.k}, {shape.n_group} groups keep "
                        f"{shape.topk_group}), intermediate {shape.I}, {shape.S} shared",
            "T": shape.T, "hidden_size": shape.H, "n_routed_experts": shape.E,
            "num_experts_per_tok": shape.k, "n_group": shape.n_group, "topk_group": shape.topk_group,
            "moe_intermediate_size": shape.I, "n_shared_experts": shape.S,
            "global_batch": shape.T * world, "parallelism": f"replicas x{world} (token-sharded)",
            "l2": "inputs larger than L2: 22.5 GB of expert weights streamed per step"
            if shape.H == 7168 else "no L2 flush (weights may stay in L2)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="v3_prefill", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mx", action="store_true", help="skip the MXFP8 variant of the layer")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward pass")
    ap.add_argument("--no-ep", action="store_true", help="skip the expert-parallel layer")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only the headline workload, not the other four shapes")
    ap.add_argument("--precision", default="bf16", choices=["bf16", "mxfp8", "backward"],
                    help="what --profile-only runs: the bf16 or MXFP8 forward stages, or the backward")
    ap.add_argument("--profile-only", action="store_true",
                    help="run warmup + steps layer passes and exit without timing (for profilers)")
    args = ap.parse_args()
    shape = WORKLOADS[args.workload]
    if args.impl == "reference" and not args.profile_only:
        # The oracle arm runs on rank 0 alone and needs no collective: no process
        # group is formed, so the other ranks exit at once without waiting for it.
        if int(os.environ.get("RANK", "0")) != 0:
            return
        if torch.cuda.is_available():
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        args.warmup = max(args.warmup, 3)
        run_reference(args, shape, int(os.environ.get("WORLD_SIZE", "1")), 0)
        return
    world, rank, local = dist_setup(args.gpus)
    if args.profile_only:
        inp0 = rank_inputs(shape, rank, "cuda")
        if args.precision == "backward":
            layer = MoELayer.from_inputs(shape, inp0)
            dy = torch.randn((shape.T, shape.H), device="cuda").bfloat16()

            class _B:
                def run(self):
                    layer.backward(inp0["x"], dy)
            st = _B()
        else:
            stepper = StagedStepMX if args.precision == "mxfp8" else StagedStep
            st = stepper(shape, inp0)
        for _ in range(args.warmup + args.steps):
            st.run()
        torch.cuda.synchronize()
        assert abi.device_status() == 0
        print(f"profile-only: {args.warmup + args.steps} passes of {shape.name}", flush=True)
        if args.precision != "backward":
            # The algorithmic bytes of this workload's GEMM launches, for the traffic ratio.
            touched = int(torch.unique(st.idx).numel())
            elt = 2.0 if args.precision == "bf16" else 1 + 1 / 32
            print(json.dumps({"workload": shape.name, "precision": args.precision, "experts_touched": touched,
                              "gate_up_algorithmic_bytes": gate_up_algorithmic_bytes(shape, touched, elt),
                              "down_algorithmic_bytes": down_algorithmic_bytes(shape, touched, elt)}),
                  flush=True)
        finish(world)
        return
    args.warmup = max(args.warmup, 3)

    peaks, peak_src = load_peaks()
    res = time_gpu(shape, args.steps, args.warmup, world, rank, peaks)
    ms = res["ms"]
    value = job_throughput(shape.T, world, ms)

    # Dominant kernel: the gate/up grouped GEMM with the SwiGLU epilogue.
    k4_ms = res["stage_ms"]["gate_up"]
    k4_flops = 4.0 * shape.H * shape.I * shape.T * (shape.k + shape.S)
    achieved = k4_flops / (k4_ms * 1e-3) / 1e12
    roofline = {"kernel": "grouped_gemm_kernel<kSwiGLU> (gate/up + SwiGLU)", "bound": "tensor",
                "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "flops_per_launch": k4_flops, "ms_per_launch": k4_ms}

    k5_ms = res["stage_ms"]["down"]
    k5_flops = 2.0 * shape.H * shape.I * shape.T * (shape.k + shape.S)
    roofline.update(traffic_fields("gate_up", gate_up_algorithmic_bytes(shape, res["experts_touched"])))
    down_roofline = {"kernel": "grouped_gemm_kernel<kDown> (down + routing weight, block-scaled fp16 out)",
                     "bound": "tensor", "achieved": k5_flops / (k5_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": k5_flops / (k5_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     **traffic_fields("down", down_algorithmic_bytes(shape, res["experts_touched"])),
                     "flops_per_launch": k5_flops, "ms_per_launch": k5_ms}

    e2e_ms, h2d, d2h = time_e2e(res["layer"], shape, max(3, args.steps // 2))
    e2e_ms = max_over_ranks(e2e_ms, world)
    routing_inputs = {shape.name: (shape, res["routing_inputs"], res["idx"])}
    load = res["load"]

    extra = {}
    if shape.name == "v3_prefill":
        del res["st"], res["layer"]
        torch.cuda.empty_cache()
        # The other four workload shapes, each timed the same way (their own inputs).
        workloads = {}
        for name in ([] if args.no_workloads else ["tiny", "mid", "v3_decode", "v3_skewed"]):
            ws = WORKLOADS[name]
            r = time_gpu(ws, max(args.steps, 20), args.warmup, world, rank, peaks)
            workloads[name] = workload_summary(ws, r, world)
            if name == "v3_skewed":
                workloads[name]["bias_balancing"] = bias_balancing(ws, r["inp"])
            routing_inputs[name] = (ws, r["routing_inputs"], r["idx"])
            del r
            torch.cuda.empty_cache()
        if workloads:
            extra["workloads"] = workloads
    if not args.no_mx and shape.name == "v3_prefill":
        # The MXFP8 expert FFNs on the same workload (fine-grained FP8 of the pages'
        # FP8 notes): a second precision of the same layer, reported beside it.
        torch.cuda.empty_cache()
        extra["mxfp8"] = time_gpu_mx(shape, args.steps, args.warmup, world, rank, peaks, inp=res["inp"])
        dec = WORKLOADS["v3_decode"]
        extra["mxfp8_decode"] = time_gpu_mx(dec, max(args.steps, 20), args.warmup, world, rank, peaks)
        torch.cuda.empty_cache()
    if not args.no_bwd and shape.name == "v3_prefill":
        extra["backward"] = time_backward(shape, max(3, args.steps // 4), args.warmup, world, rank, peaks,
                                          res["inp"])
        torch.cuda.empty_cache()
    if not args.no_ep and shape.name == "v3_prefill":
        extra["expert_parallel"] = time_ep(shape, max(3, args.steps // 2), args.warmup, world, rank, res["inp"])
        torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights)",
        "config": workload_config(shape, world),
        "tflops": res["tflops"] * world, "stage_ms": res["stage_ms"], "staged_ms": res["staged_ms"],
        "forward_ms": res["forward_ms"],
        "layer_roofline": res["layer_roofline"], "experts_touched": res["experts_touched"], "load": load,
        "roofline": roofline, "down_roofline": down_roofline,
        "clocks": res["clocks"],
        "e2e": {"value": job_throughput(shape.T, world, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": res["launches"],
    }
    line.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(shape, res["inp"])
        # The oracle router over every token of each workload: near ties and the
        # GPU's agreement with it.
        cb["routing"] = {name: oracle_routing_report(ws, ri, gi) for name, (ws, ri, gi) in routing_inputs.items()}
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    finish(world)


def finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
