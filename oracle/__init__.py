"""Float64 CPU oracle of the DeepSeekMoE layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, the package's ``smoke()`` check and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python
binding) never imports, links or calls anything here, and this package imports
nothing from the product.

The arithmetic lives in ``moe_oracle.c`` (plain C, float64, single thread); this
module builds it with gcc, wraps it with ctypes, and composes the layer's
forward the way the teaching code of "The Evolving Transformer · 07 — DeepSeek
V2 & V3" (§ 02 DeepSeekMoE, § 03 Shared Expert) defines it: the shared expert
runs on every token; the router gives each token its top-k experts and their
weights; each routed expert runs on the tokens sent to it; a token's output is
the shared expert's output plus the weighted sum of its experts' outputs, the
slots added in order 0..top_k-1.

Each expert's rows are computed in one call (so its weights are fetched once)
and every (token, slot) result is kept until the slots are added in order, so
each token sees the same additions in the same order as a slot-by-slot loop.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Callable, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (strict IEEE float64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden_size", ctypes.c_int32), ("n_routed_experts", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("n_shared_experts", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_double)]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        lib.oracle_route.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64, p, p, p, p, p, p, p]
        lib.oracle_route.restype = ctypes.c_int
        lib.oracle_swiglu.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      p, p, p, p, p]
        lib.oracle_swiglu.restype = ctypes.c_int
        lib.oracle_bias_update.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, p, p,
                                           ctypes.c_float, p]
        lib.oracle_bias_update.restype = None
        lib.oracle_e4m3_round.argtypes = [ctypes.c_double]
        lib.oracle_e4m3_round.restype = ctypes.c_double
        lib.oracle_mx_scale_code.argtypes = [ctypes.c_double]
        lib.oracle_mx_scale_code.restype = ctypes.c_int
        lib.oracle_mx_quantize.argtypes = [ctypes.c_int64, ctypes.c_int64, p, p, p, p]
        lib.oracle_mx_quantize.restype = None
        lib.oracle_e4m3_round_n.argtypes = [ctypes.c_int64, p, p]
        lib.oracle_e4m3_round_n.restype = None
        lib.oracle_e4m3_bits_n.argtypes = [ctypes.c_int64, p, p]
        lib.oracle_e4m3_bits_n.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bits as uint16, got {a.dtype}")
    return a


def _cfg(shape) -> _Cfg:
    return _Cfg(shape.hidden_size, shape.n_routed_experts, shape.num_experts_per_tok,
                shape.n_group, shape.topk_group, shape.moe_intermediate_size,
                shape.n_shared_experts, int(bool(shape.norm_topk_prob)),
                float(shape.routed_scaling_factor))


def route(shape, x_bits, router_w, e_bias, want_scores: bool = False):
    """Router for every row of ``x_bits`` [n, H] (bf16 bits).

    Returns (idx int32 [n,k], w float64 [n,k], margin float64 [n]) and, when
    asked, the unbiased sigmoid scores float64 [n,E].
    """
    lib = _load()
    x_bits = _u16(x_bits)
    n = x_bits.shape[0]
    k, E = shape.num_experts_per_tok, shape.n_routed_experts
    rw = np.ascontiguousarray(router_w, dtype=np.float32)
    eb = np.ascontiguousarray(e_bias, dtype=np.float32)
    idx = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float64)
    margin = np.zeros((n,), np.float64)
    scores = np.zeros((n, E), np.float64) if want_scores else None
    rc = lib.oracle_route(ctypes.byref(_cfg(shape)), n, _ptr(x_bits), _ptr(rw), _ptr(eb),
                          _ptr(idx), _ptr(w), _ptr(margin),
                          _ptr(scores) if want_scores else None)
    if rc != 0:
        raise ValueError(f"oracle_route rejected the configuration {shape}")
    return (idx, w, margin, scores) if want_scores else (idx, w, margin)


def swiglu(x_bits, w_gate, w_up, w_down) -> np.ndarray:
    """down(silu(gate x) * up x) in float64 for rows x_bits [n,H]; weights (out, in)."""
    lib = _load()
    x_bits, w_gate, w_up, w_down = (_u16(a) for a in (x_bits, w_gate, w_up, w_down))
    n, H = x_bits.shape
    I = w_gate.shape[0]
    assert w_gate.shape == (I, H) and w_up.shape == (I, H) and w_down.shape == (H, I)
    out = np.zeros((n, H), np.float64)
    if n == 0 or I == 0:
        return out
    rc = lib.oracle_swiglu(n, H, I, _ptr(x_bits), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                           _ptr(out))
    if rc != 0:
        raise MemoryError("oracle_swiglu failed to allocate")
    return out


ExpertFetch = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def _run_serial(fn, jobs):
    return (fn(*job) for job in jobs)


def moe_layer(shape, x_bits, router_w, e_bias, expert: ExpertFetch,
              shared: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]],
              routing: Optional[Tuple[np.ndarray, np.ndarray]] = None, run_experts=None):
    """The layer's forward for the rows of ``x_bits`` (any subset of tokens).

    ``expert(e)`` returns (w_gate[e], w_up[e], w_down[e]) as bf16 bits; it is
    called once per expert that some row uses.  ``shared`` is the concatenated
    shared expert (ws_gate [S*I,H], ws_up [S*I,H], ws_down [H,S*I]) or None.
    ``routing`` optionally supplies (idx, w) instead of the oracle's own router
    (used to score an alternative, equally correct near-tie selection).
    ``run_experts(fn, jobs)`` optionally evaluates ``fn(*job)`` for each expert's
    job, in order (``oracle.pool.ExpertRunner`` spreads them over processes);
    by default they run here, one after the other.

    Returns (y float64 [n,H], idx, w, margin or None).
    """
    x_bits = _u16(x_bits)
    n, H = x_bits.shape
    k = shape.num_experts_per_tok
    margin = None
    if routing is None:
        idx, w, margin = route(shape, x_bits, router_w, e_bias)
    else:
        idx, w = routing
        idx = np.asarray(idx, np.int32)
        w = np.asarray(w, np.float64)

    # shared_expert(x): runs unconditionally for every row.
    if shared is not None and shape.n_shared_experts > 0:
        shared_out = swiglu(x_bits, *shared)
    else:
        shared_out = np.zeros((n, H), np.float64)

    # routed: contribution of (row, slot) = w[row, slot] * expert_e(x[row]).
    contrib = np.zeros((n, k, H), np.float64)
    experts = [int(e) for e in np.unique(idx)]
    jobs = ((x_bits[np.nonzero(idx == e)[0]], *expert(e)) for e in experts)
    for e, out in zip(experts, (run_experts or _run_serial)(swiglu, jobs)):
        rows, slots = np.nonzero(idx == e)
        contrib[rows, slots] = w[rows, slots][:, None] * out
    output = np.zeros((n, H), np.float64)
    for j in range(k):
        output += contrib[:, j]
    return shared_out + output, idx, w, margin


def in_memory_experts(w_gate, w_up, w_down) -> ExpertFetch:
    """Expert fetcher over host arrays [E,I,H], [E,I,H], [E,H,I] of bf16 bits."""
    return lambda e: (w_gate[e], w_up[e], w_down[e])



# ----------------------------------------------------------------------------
# MXFP8 variant of the expert FFNs ("DeepSeek-V3 notes" (knlb.dev), § fp8:
# fine-grained block-wise E4M3 quantisation with scales taken online from each
# block's maximum; gating kept in high precision).  Quantised operands: the token
# rows entering the experts (blocks of 32 along H), the gate/up weights (blocks of
# 32 along H, the contraction axis), the SwiGLU output h (blocks of 32 along I)
# and the down weights (blocks of 32 along I).  Everything else — routing, the
# products and their sums, SwiGLU itself, the weighted combine — stays float64.
# ----------------------------------------------------------------------------

def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value of each element (ties to even), float64."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(v)
    lib.oracle_e4m3_round_n(v.size, _ptr(v), _ptr(out))
    return out


def e4m3_bits(q) -> np.ndarray:
    """E4M3 bit patterns (uint8) of values already on the E4M3 grid."""
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    out = np.empty(q.shape, np.uint8)
    lib.oracle_e4m3_bits_n(q.size, _ptr(q), _ptr(out))
    return out


def mx_scale_code(amax: float) -> int:
    return int(_load().oracle_mx_scale_code(float(amax)))


def mx_quantize(a):
    """Blocks of 32 along the last axis of a [rows, K] array (float64 or bf16 bits).

    Returns (q, codes, deq): E4M3 element values (float64, unscaled), uint8 scale
    codes [rows, K/32] and the dequantised values q * 2^(code - 127)."""
    lib = _load()
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = widen_bf16(a)
    a = np.ascontiguousarray(a, dtype=np.float64)
    rows, K = a.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q = np.empty_like(a)
    deq = np.empty_like(a)
    codes = np.empty((rows, K // 32), np.uint8)
    lib.oracle_mx_quantize(rows, K, _ptr(a), _ptr(q), _ptr(codes), _ptr(deq))
    return q, codes, deq


def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def swiglu_mx(x_deq, w_gate, w_up, w_down, h_out=None) -> np.ndarray:
    """One expert with MXFP8 operands, float64 arithmetic: rows x_deq [n,H] are the
    already-quantised tokens; the weights (bf16 bits, (out, in) layout) are
    quantised here; h = silu(gate x) * up x is quantised before the down
    projection.  Returns [n,H]; ``h_out`` (optional list) receives the float64 h."""
    wg = mx_quantize(w_gate)[2]
    wu = mx_quantize(w_up)[2]
    wd = mx_quantize(w_down)[2]
    g = x_deq @ wg.T
    u = x_deq @ wu.T
    h = g / (1.0 + np.exp(-g)) * u
    if h_out is not None:
        h_out.append(h)
    return mx_quantize(h)[2] @ wd.T


def moe_layer_mx(shape, x_bits, router_w, e_bias, expert: ExpertFetch,
                 shared: Optional[Tuple[np.ndarray, np.ndarray, np.ndarray]],
                 routing: Optional[Tuple[np.ndarray, np.ndarray]] = None, run_experts=None):
    """The layer's forward with MXFP8 expert FFNs, for the rows of ``x_bits``.

    Same structure as ``moe_layer`` (shared expert on every row; routed outputs
    weighted and summed in slot order); the router is the float64 one on the
    unquantised bf16 rows.  Returns (y float64 [n,H], idx, w, margin or None)."""
    x_bits = _u16(x_bits)
    n, H = x_bits.shape
    k = shape.num_experts_per_tok
    margin = None
    if routing is None:
        idx, w, margin = route(shape, x_bits, router_w, e_bias)
    else:
        idx = np.asarray(routing[0], np.int32)
        w = np.asarray(routing[1], np.float64)
    xq = mx_quantize(x_bits)[2]
    if shared is not None and shape.n_shared_experts > 0:
        shared_out = swiglu_mx(xq, *shared)
    else:
        shared_out = np.zeros((n, H), np.float64)
    contrib = np.zeros((n, k, H), np.float64)
    experts = [int(e) for e in np.unique(idx)]
    jobs = ((xq[np.nonzero(idx == e)[0]], *expert(e)) for e in experts)
    for e, out in zip(experts, (run_experts or _run_serial)(swiglu_mx, jobs)):
        rows, slots = np.nonzero(idx == e)
        contrib[rows, slots] = w[rows, slots][:, None] * out
    output = np.zeros((n, H), np.float64)
    for j in range(k):
        output += contrib[:, j]
    return shared_out + output, idx, w, margin


def bias_update(idx, n_experts: int, bias, gamma: float):
    """Aux-loss-free bias step: returns (new bias fp32 [E], load int64 [E])."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    b = np.array(bias, dtype=np.float32, copy=True)
    load = np.zeros(n_experts, np.int64)
    lib.oracle_bias_update(T, k, n_experts, _ptr(idx), _ptr(b), ctypes.c_float(gamma), _ptr(load))
    return b, load
