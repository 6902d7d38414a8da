"""Workload shapes and seeded synthetic inputs for the DeepSeekMoE layer.

This module is shared by the CUDA path's tests/benchmark and by the float64
oracle's tests.  It holds no arithmetic of the method itself: it only names the
layer shapes and draws random tensors in a fixed, documented order.

Shapes follow the DeepSeek-V3 MoE dimensions printed on the
"DeepSeekV3.2-Tiered-Implementations" README (§ Architecture, § Key Dimensions:
hidden_size 7168, 256 routed experts, top-8, 1 shared expert, n_group=8,
topk_group=4, moe_intermediate_size 2048).

Draw order for a workload (one ``torch.Generator`` seeded with ``seed`` on the
target device):
  1. x        [T, H]      ~ N(0, 1)            -> bf16
  2. router_w [E, H]      ~ N(0, 0.02)         fp32
  3. e_bias   [E]         ~ U(-b, b)           fp32   (uniform workloads)
                          or, for the skewed workload, a random permutation of
                          the experts followed by 0.5 * ln(Zipf(s) popularity)
  4. w_gate   [E, I, H]   ~ N(0, 0.02)  -> bf16, drawn expert by expert
  5. w_up     [E, I, H]   ~ N(0, 0.02)  -> bf16, expert by expert
  6. w_down   [E, H, I]   ~ N(0, 0.02)  -> bf16, expert by expert
  7. ws_gate  [S*I, H], ws_up [S*I, H], ws_down [H, S*I] ~ N(0, 0.02) -> bf16
The torch CPU and CUDA generators give different streams for the same seed, so a
parity test draws once on its device and hands the same bits to both sides.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class MoEShape:
    """One layer configuration, with the DeepSeek-V3 config field names."""

    name: str
    T: int
    hidden_size: int
    n_routed_experts: int
    n_group: int
    topk_group: int
    num_experts_per_tok: int
    moe_intermediate_size: int
    n_shared_experts: int
    routed_scaling_factor: float
    norm_topk_prob: bool
    bias_kind: str = "uniform"     # "uniform" or "zipf"
    bias_range: float = 0.1        # half-width b of U(-b, b)
    zipf_s: float = 1.2
    seed: int = 0

    @property
    def H(self) -> int:
        return self.hidden_size

    @property
    def E(self) -> int:
        return self.n_routed_experts

    @property
    def I(self) -> int:  # noqa: E743 - the intermediate size's usual name
        return self.moe_intermediate_size

    @property
    def k(self) -> int:
        return self.num_experts_per_tok

    @property
    def S(self) -> int:
        return self.n_shared_experts

    def with_(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)

    def routed_weight_bytes(self) -> int:
        return 3 * self.E * self.I * self.H * 2

    def flops(self) -> float:
        """Algorithmic FLOPs of one forward: router GEMM + (k + S) SwiGLU experts per token."""
        return float(self.T) * (2.0 * self.H * self.E
                                + 6.0 * self.H * self.I * (self.k + self.S))


# The five workloads: tiny, mid (V2-lite-like), V3 decode, V3 prefill, V3 skewed.
TINY = MoEShape("tiny", T=64, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                num_experts_per_tok=4, moe_intermediate_size=128, n_shared_experts=1,
                routed_scaling_factor=2.5, norm_topk_prob=True, bias_range=0.1, seed=0)
MID = MoEShape("mid", T=4096, hidden_size=2048, n_routed_experts=64, n_group=8, topk_group=4,
               num_experts_per_tok=6, moe_intermediate_size=1408, n_shared_experts=2,
               routed_scaling_factor=1.0, norm_topk_prob=False, bias_range=0.05, seed=1)
V3_DECODE = MoEShape("v3_decode", T=128, hidden_size=7168, n_routed_experts=256, n_group=8,
                     topk_group=4, num_experts_per_tok=8, moe_intermediate_size=2048,
                     n_shared_experts=1, routed_scaling_factor=2.5, norm_topk_prob=True,
                     bias_range=0.1, seed=2)
V3_PREFILL = V3_DECODE.with_(name="v3_prefill", T=16384, seed=3)
V3_SKEWED = V3_DECODE.with_(name="v3_skewed", T=8192, bias_kind="zipf", seed=4)

# V3 dimensions with 32 experts (2.8 GB of weights, still 22x the L2): the case
# for detailed profiler captures, which must stay a few GB on the device.
V3_E32 = V3_DECODE.with_(name="v3_e32", T=4096, n_routed_experts=32, seed=5)
# The same 32 experts under a prefill-sized batch (16384 tokens, top-2: ~1024 rows per
# expert, and the shared expert's 16384 rows = 235 MB of A, as at the V3 prefill):
# a capture case for the DRAM traffic of the prefill's tile orders (about 4.5 GB on
# the device).
V3_E32_T16K = V3_E32.with_(name="v3_e32_t16k", T=16384, num_experts_per_tok=2, seed=6)

# The V3 router, dispatch and combine at their full widths (256 experts, top-8, hidden
# 7168) on 8192 tokens, with a narrow intermediate (128) so that the expert weights
# take 1.4 GB: the capture case for the DRAM traffic of the kernels around the expert
# GEMMs (x_perm and y_perm 0.94 GB each, beyond the L2; about 4 GB on the device).
V3_IO = V3_DECODE.with_(name="v3_io", T=8192, moe_intermediate_size=128, seed=7)
# 16 experts at V3 dimensions on 1024 tokens (top-8 of the 8 experts in the 4 kept
# groups: ~512 rows per expert, as at the V3 prefill): the capture case for the
# backward's weight-gradient GEMMs, whose contraction runs over an expert's rows
# (about 3 GB on the device).
V3_E16_T1K = V3_E32.with_(name="v3_e16_t1k", T=1024, n_routed_experts=16, seed=8)

WORKLOADS: Dict[str, MoEShape] = {w.name: w for w in
                                  (TINY, MID, V3_DECODE, V3_PREFILL, V3_SKEWED, V3_E32, V3_E32_T16K, V3_IO,
                                   V3_E16_T1K)}


def _normal(shape, std, gen, device, dtype):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(dtype)


def make_inputs(shape: MoEShape, device="cpu", seed: Optional[int] = None,
                weight_std: float = 0.02) -> Dict[str, torch.Tensor]:
    """Draw every input of one workload in the documented order.

    Returns a dict of contiguous tensors on ``device``: x, router_w, e_bias,
    w_gate, w_up, w_down, ws_gate, ws_up, ws_down (shared tensors have zero
    rows when n_shared_experts == 0).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(shape.seed if seed is None else seed)
    T, H, E, I, S = shape.T, shape.H, shape.E, shape.I, shape.S
    bf = torch.bfloat16
    out: Dict[str, torch.Tensor] = {}
    out["x"] = _normal((T, H), 1.0, gen, device, bf)
    out["router_w"] = _normal((E, H), weight_std, gen, device, torch.float32)
    if shape.bias_kind == "uniform":
        u = torch.rand((E,), generator=gen, device=device, dtype=torch.float32)
        out["e_bias"] = (u * 2.0 - 1.0) * shape.bias_range
    elif shape.bias_kind == "zipf":
        perm = torch.randperm(E, generator=gen, device=device)
        out["e_bias"] = zipf_bias(E, shape.zipf_s, perm.cpu()).to(device)
    else:
        raise ValueError(f"unknown bias kind {shape.bias_kind!r}")
    for name, rows, cols in (("w_gate", I, H), ("w_up", I, H), ("w_down", H, I)):
        t = torch.empty((E, rows, cols), device=device, dtype=bf)
        for e in range(E):
            t[e] = _normal((rows, cols), weight_std, gen, device, bf)
        out[name] = t
    out["ws_gate"] = _normal((S * I, H), weight_std, gen, device, bf)
    out["ws_up"] = _normal((S * I, H), weight_std, gen, device, bf)
    out["ws_down"] = _normal((H, S * I), weight_std, gen, device, bf)
    return out


def zipf_bias(E: int, s: float, perm: torch.Tensor) -> torch.Tensor:
    """Skewed correction bias: expert perm[r-1] gets 0.5 * ln(p_r), p_r ∝ r^-s, Σp = 1."""
    p = [r ** (-s) for r in range(1, E + 1)]
    z = sum(p)
    bias = torch.empty(E, dtype=torch.float32)
    for r in range(E):
        bias[int(perm[r])] = 0.5 * math.log(p[r] / z)
    return bias


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bits (copied to the CPU)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
