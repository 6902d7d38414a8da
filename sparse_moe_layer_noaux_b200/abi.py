"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every entry point keeps the C name and order of arguments; tensors are torch
CUDA tensors (PyTorch provides device memory and the stream), turned into
device pointers here.  There is no fallback: if libmoe.so is missing or a call
returns an error status, a MoEError is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT,
 MOE_ERR_STATIC_LIMIT, MOE_ERR_DEVICE_CHECK) = range(8)
MOE_DTYPE_F32, MOE_DTYPE_BF16 = 0, 1


def out_dtype_code(t: torch.Tensor) -> int:
    """moe_dtype of an output tensor (fp32 or bf16)."""
    if t.dtype == torch.float32:
        return MOE_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    raise TypeError(f"layer output must be float32 or bfloat16, got {t.dtype}")


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")


class MoEConfig(ctypes.Structure):
    """Mirror of `moe_config` (DeepSeek-V3 config field names)."""

    _fields_ = [("hidden_size", ctypes.c_int32), ("n_routed_experts", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("n_shared_experts", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float)]

    @classmethod
    def from_shape(cls, s) -> "MoEConfig":
        return cls(s.hidden_size, s.n_routed_experts, s.num_experts_per_tok, s.n_group,
                   s.topk_group, s.moe_intermediate_size, s.n_shared_experts,
                   int(bool(s.norm_topk_prob)), float(s.routed_scaling_factor))


_lib = None
_P = ctypes.c_void_p


class MXMatrix(ctypes.Structure):
    """Mirror of `moe_mx_matrix`: E4M3 bytes and their scale atoms (device pointers)."""

    _fields_ = [("q", ctypes.c_void_p), ("sf", ctypes.c_void_p)]


class MXWeights(ctypes.Structure):
    """Mirror of `moe_mx_weights`."""

    _fields_ = [("gate", MXMatrix), ("up", MXMatrix), ("down", MXMatrix), ("shared_gate", MXMatrix),
                ("shared_up", MXMatrix), ("shared_down", MXMatrix)]


def lib():
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not found at {LIB_PATH}; build it with "
                               "`python -m sparse_moe_layer_noaux_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        cfgp = ctypes.POINTER(MoEConfig)
        i64, sz = ctypes.c_int64, ctypes.c_size_t
        L.moe_workspace_size.argtypes = [cfgp, i64, ctypes.POINTER(sz)]
        L.moe_route.argtypes = [cfgp, i64, _P, _P, _P, _P, _P, _P, sz, _P]
        L.moe_dispatch.argtypes = [cfgp, i64, _P, _P, _P, _P, _P, _P, _P, sz, _P]
        L.moe_experts.argtypes = [cfgp, i64] + [_P] * 16
        L.moe_dispatch_noalloc.argtypes = [cfgp, i64, _P, _P, _P, _P, _P, _P, _P]
        L.moe_experts_gate_up.argtypes = [cfgp, i64] + [_P] * 10
        L.moe_experts_down.argtypes = [cfgp, i64] + [_P] * 10
        L.moe_combine.argtypes = [cfgp, i64, _P, _P, _P, _P, ctypes.c_int32, _P]
        L.moe_forward.argtypes = [cfgp, i64] + [_P] * 10 + [ctypes.c_int32, _P, _P, _P, sz, _P]
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_int32)]
        L.moe_launch_count.argtypes = []
        L.moe_launch_count.restype = ctypes.c_uint64
        L.moe_selftest_wait_timeout.argtypes = [ctypes.c_uint64, _P]
        L.moe_bias_update.argtypes = [cfgp, i64, _P, _P, ctypes.c_float, _P, _P]
        L.moe_mx_scale_bytes.argtypes = [i64, i64]
        L.moe_mx_scale_bytes.restype = ctypes.c_int64
        L.moe_mx_quantize.argtypes = [i64, i64, _P, _P, _P, _P]
        L.moe_workspace_size_mx.argtypes = [cfgp, i64, ctypes.POINTER(sz)]
        L.moe_mx_routed_rows.argtypes = [cfgp, i64, ctypes.POINTER(i64)]
        L.moe_dispatch_mx.argtypes = [cfgp, i64] + [_P] * 11 + [sz, _P]
        L.moe_forward_mx.argtypes = [cfgp, i64, _P, _P, _P, ctypes.POINTER(MXWeights), _P, ctypes.c_int32,
                                     _P, _P, _P, sz, _P]
        wp = ctypes.POINTER(MXWeights)
        L.moe_experts_gate_up_mx.argtypes = [cfgp, i64] + [_P] * 6 + [wp] + [_P] * 5
        L.moe_experts_down_mx.argtypes = [cfgp, i64] + [_P] * 8 + [wp] + [_P] * 3
        L.moe_combine_mx.argtypes = [cfgp, i64, _P, _P, _P, _P, ctypes.c_int32, _P]
        L.moe_workspace_size_bwd.argtypes = [cfgp, i64, ctypes.POINTER(sz)]
        L.moe_workspace_size_host.argtypes = [cfgp, i64, i64, ctypes.c_int32, ctypes.POINTER(sz)]
        L.moe_forward_train.argtypes = [cfgp, i64] + [_P] * 10 + [ctypes.c_int32, _P, sz, _P]
        L.moe_backward_train.argtypes = [cfgp, i64] + [_P] * 18 + [sz, _P]
        L.moe_forward_host.argtypes = [cfgp, i64] + [_P] * 10 + [ctypes.c_int32, i64, _P, sz, _P]
        L.moe_backward.argtypes = [cfgp, i64] + [_P] * 19 + [sz, _P]
        i32 = ctypes.c_int32
        L.moe_ep_row_bytes.argtypes = [cfgp, ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.moe_ep_workspace_size.argtypes = [cfgp, i32, i32, i64, i64, ctypes.POINTER(sz)]
        L.moe_ep_place.argtypes = [i32, i32, _P, i32, i32, _P]
        L.moe_ep_local_experts.argtypes = [i32, i32, i32, _P, i32, _P, ctypes.POINTER(i32)]
        L.moe_ep_send.argtypes = [cfgp, i32, i64, _P, _P, _P, _P, i32] + [_P] * 4 + [sz, _P]
        L.moe_ep_experts.argtypes = [cfgp, i32, i32, _P, i32, i64, _P, i64] + [_P] * 11 + [sz, _P]
        L.moe_ep_combine.argtypes = [cfgp, i32, i64, i64] + [_P] * 5 + [i32, _P]
        for fn in ("moe_workspace_size", "moe_route", "moe_dispatch", "moe_dispatch_noalloc", "moe_experts",
                   "moe_experts_gate_up", "moe_experts_down",
                   "moe_combine", "moe_forward", "moe_device_status", "moe_selftest_wait_timeout",
                   "moe_bias_update", "moe_mx_quantize", "moe_workspace_size_mx", "moe_mx_routed_rows",
                   "moe_dispatch_mx", "moe_forward_mx", "moe_experts_gate_up_mx", "moe_experts_down_mx",
                   "moe_combine_mx", "moe_workspace_size_bwd", "moe_backward", "moe_workspace_size_host",
                   "moe_forward_host", "moe_forward_train", "moe_backward_train", "moe_ep_row_bytes",
                   "moe_ep_workspace_size", "moe_ep_place", "moe_ep_local_experts", "moe_ep_send",
                   "moe_ep_experts", "moe_ep_combine"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoEError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _cfg(cfg):
    return cfg if isinstance(cfg, MoEConfig) else MoEConfig.from_shape(cfg)


# ---------------------------------------------------------------- argument checks
# The C ABI takes raw pointers and cannot see buffer sizes, so every wrapper checks
# each tensor before its address is passed on: element type, dense (contiguous)
# layout, the current CUDA device (pinned host memory for the host-buffer entry
# point) and at least as many elements as the call reads or writes.  A violation
# raises TypeError / ValueError before anything is launched.

_BF16, _F16, _F32, _I32, _U8 = torch.bfloat16, torch.float16, torch.float32, torch.int32, torch.uint8
_OUT = (torch.float32, torch.bfloat16)


class _Dims:
    def __init__(self, cfg, T: int):
        c = _cfg(cfg)
        self.T, self.H, self.E = int(T), int(c.hidden_size), int(c.n_routed_experts)
        self.k, self.I, self.S = int(c.num_experts_per_tok), int(c.moe_intermediate_size), int(c.n_shared_experts)
        self.SI = self.S * self.I
        self.scale_cols = y_perm_scale_cols(self.H)


def _on_current_cuda_device(t: torch.Tensor) -> bool:
    return t.device.type == "cuda" and t.device.index == torch.cuda.current_device()


def _req(name: str, t, dtype, numel: int, where: str = "cuda", optional: bool = False):
    """Check one tensor argument (see above); `numel` is the minimum element count."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name}: a tensor is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    allowed = dtype if isinstance(dtype, tuple) else (dtype,)
    if t.dtype not in allowed:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in allowed)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if where == "cuda":
        if not _on_current_cuda_device(t):
            raise ValueError(f"{name}: must be on the current CUDA device, is on {t.device}")
    elif t.device.type != "cpu":
        raise ValueError(f"{name}: must be a host (CPU) tensor, is on {t.device}")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, the call needs at least {numel}")


def _rows_2d(name: str, x, H: int) -> int:
    """Rows T of a [T, H] argument."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2 or x.shape[1] != H:
        shape = tuple(x.shape) if isinstance(x, torch.Tensor) else type(x).__name__
        raise ValueError(f"{name}: expected shape [T, {H}], got {shape}")
    return int(x.shape[0])


def _req_weights(d: _Dims, w_gate=None, w_up=None, w_down=None, ws_gate=None, ws_up=None, ws_down=None,
                 prefix: str = "", need=("gate", "up", "down")):
    """Routed expert weights [E, I, H] / [E, H, I] and, when S > 0, the shared ones."""
    EIH, SIH = d.E * d.I * d.H, d.SI * d.H
    if "gate" in need:
        _req(prefix + "w_gate", w_gate, _BF16, EIH)
        _req(prefix + "ws_gate", ws_gate, _BF16, SIH, optional=d.S == 0)
    if "up" in need:
        _req(prefix + "w_up", w_up, _BF16, EIH)
        _req(prefix + "ws_up", ws_up, _BF16, SIH, optional=d.S == 0)
    if "down" in need:
        _req(prefix + "w_down", w_down, _BF16, EIH)
        _req(prefix + "ws_down", ws_down, _BF16, SIH, optional=d.S == 0)


def _n(d: _Dims, count: int) -> int:
    """A minimum size that only applies to a non-empty batch (T = 0 is a no-op)."""
    return count if d.T > 0 else 0


def workspace_size(cfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(_cfg(cfg)), T, ctypes.byref(n)))
    return n.value


def moe_route(cfg, x, router_w, e_bias, topk_idx, topk_w, workspace, stream=None):
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _req("x", x, _BF16, 0)
    _req("router_w", router_w, _F32, d.E * d.H)
    _req("e_bias", e_bias, _F32, d.E)
    _req("topk_idx", topk_idx, _I32, d.T * d.k)
    _req("topk_w", topk_w, _F32, d.T * d.k)
    _req("workspace", workspace, _U8, 0)
    _check("moe_route", lib().moe_route(ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w),
                                        _ptr(e_bias), _ptr(topk_idx), _ptr(topk_w), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream)))


def _req_dispatch(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of) -> _Dims:
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _req("x", x, _BF16, 0)
    _req("topk_idx", topk_idx, _I32, d.T * d.k)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req("x_perm", x_perm, _BF16, d.T * d.k * d.H)
    _req("perm_src", perm_src, _I32, d.T * d.k)
    _req("row_of", row_of, _I32, d.T * d.k)
    return d


def moe_dispatch(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of, workspace, stream=None):
    _req_dispatch(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of)
    _req("workspace", workspace, _U8, 0)
    _check("moe_dispatch", lib().moe_dispatch(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(topk_idx), _ptr(expert_offsets),
        _ptr(x_perm), _ptr(perm_src), _ptr(row_of), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_dispatch_noalloc(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of, stream=None):
    """moe_dispatch without a workspace: its scratch is a fixed 1 MiB array inside
    the library (see include/moe.h for the size limit and the sharing rules)."""
    _req_dispatch(cfg, x, topk_idx, expert_offsets, x_perm, perm_src, row_of)
    _check("moe_dispatch_noalloc", lib().moe_dispatch_noalloc(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(topk_idx), _ptr(expert_offsets),
        _ptr(x_perm), _ptr(perm_src), _ptr(row_of), _stream(stream)))


def y_perm_scale_cols(H: int) -> int:
    """Row pitch (bytes) of the y_perm block-scale codes: one per 32 columns, padded to 8."""
    return (H // 32 + 7) // 8 * 8


def moe_experts(cfg, T, x, x_perm, expert_offsets, perm_src, topk_w, w_gate, w_up, w_down,
                ws_gate, ws_up, ws_down, h_routed, h_shared, y_perm, y_perm_scale, stream=None):
    d = _Dims(cfg, T)
    _req_gate_up(d, x, x_perm, expert_offsets, w_gate, w_up, ws_gate, ws_up, h_routed, h_shared)
    _req_down(d, h_routed, h_shared, expert_offsets, perm_src, topk_w, w_down, ws_down, y_perm, y_perm_scale)
    _check("moe_experts", lib().moe_experts(
        ctypes.byref(_cfg(cfg)), T, _ptr(x), _ptr(x_perm), _ptr(expert_offsets), _ptr(perm_src),
        _ptr(topk_w), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up),
        _ptr(ws_down), _ptr(h_routed), _ptr(h_shared), _ptr(y_perm), _ptr(y_perm_scale),
        _stream(stream)))


def _req_gate_up(d, x, x_perm, expert_offsets, w_gate, w_up, ws_gate, ws_up, h_routed, h_shared):
    shared = d.S > 0
    _req("x", x, _BF16, d.T * d.H if shared else 0, optional=not shared)
    _req("x_perm", x_perm, _BF16, d.T * d.k * d.H)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req_weights(d, w_gate=w_gate, w_up=w_up, ws_gate=ws_gate, ws_up=ws_up, need=("gate", "up"))
    _req("h_routed", h_routed, _BF16, d.T * d.k * d.I)
    _req("h_shared", h_shared, _BF16, d.T * d.SI, optional=not shared)


def _req_down(d, h_routed, h_shared, expert_offsets, perm_src, topk_w, w_down, ws_down, y_perm, y_perm_scale):
    shared = d.S > 0
    rows = d.T * d.k + (d.T if shared else 0)
    _req("h_routed", h_routed, _BF16, d.T * d.k * d.I)
    _req("h_shared", h_shared, _BF16, d.T * d.SI, optional=not shared)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req("perm_src", perm_src, _I32, d.T * d.k)
    _req("topk_w", topk_w, _F32, d.T * d.k)
    _req_weights(d, w_down=w_down, ws_down=ws_down, need=("down",))
    _req("y_perm", y_perm, _F16, rows * d.H)
    _req("y_perm_scale", y_perm_scale, _U8, rows * d.scale_cols)


def moe_experts_gate_up(cfg, T, x, x_perm, expert_offsets, w_gate, w_up, ws_gate, ws_up, h_routed,
                        h_shared, stream=None):
    _req_gate_up(_Dims(cfg, T), x, x_perm, expert_offsets, w_gate, w_up, ws_gate, ws_up, h_routed, h_shared)
    _check("moe_experts_gate_up", lib().moe_experts_gate_up(
        ctypes.byref(_cfg(cfg)), T, _ptr(x), _ptr(x_perm), _ptr(expert_offsets), _ptr(w_gate),
        _ptr(w_up), _ptr(ws_gate), _ptr(ws_up), _ptr(h_routed), _ptr(h_shared), _stream(stream)))


def moe_experts_down(cfg, T, h_routed, h_shared, expert_offsets, perm_src, topk_w, w_down, ws_down,
                     y_perm, y_perm_scale, stream=None):
    _req_down(_Dims(cfg, T), h_routed, h_shared, expert_offsets, perm_src, topk_w, w_down, ws_down, y_perm,
              y_perm_scale)
    _check("moe_experts_down", lib().moe_experts_down(
        ctypes.byref(_cfg(cfg)), T, _ptr(h_routed), _ptr(h_shared), _ptr(expert_offsets),
        _ptr(perm_src), _ptr(topk_w), _ptr(w_down), _ptr(ws_down), _ptr(y_perm), _ptr(y_perm_scale),
        _stream(stream)))


def _req_combine(d, routed_rows, y_perm, y_perm_scale, row_of, y):
    rows = routed_rows + (d.T if d.S > 0 else 0)
    _req("y_perm", y_perm, _F16, rows * d.H)
    _req("y_perm_scale", y_perm_scale, _U8, rows * d.scale_cols)
    _req("row_of", row_of, _I32, d.T * d.k)
    _req("y", y, _OUT, d.T * d.H)


def moe_combine(cfg, T, y_perm, y_perm_scale, row_of, y, stream=None):
    d = _Dims(cfg, T)
    _req_combine(d, d.T * d.k, y_perm, y_perm_scale, row_of, y)
    _check("moe_combine", lib().moe_combine(ctypes.byref(_cfg(cfg)), T, _ptr(y_perm), _ptr(y_perm_scale),
                                            _ptr(row_of), _ptr(y), out_dtype_code(y), _stream(stream)))


def _req_layer(cfg, x, router_w, e_bias, y, topk_idx_out, topk_w_out, x_where="cuda") -> _Dims:
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _req("x", x, _BF16, 0, where=x_where)
    _req("router_w", router_w, _F32, d.E * d.H)
    _req("e_bias", e_bias, _F32, d.E)
    _req("y", y, _OUT, d.T * d.H, where=x_where)
    _req("topk_idx_out", topk_idx_out, _I32, d.T * d.k, optional=True)
    _req("topk_w_out", topk_w_out, _F32, d.T * d.k, optional=True)
    return d


def moe_forward(cfg, x, router_w, e_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y,
                topk_idx_out=None, topk_w_out=None, workspace=None, stream=None):
    d = _req_layer(cfg, x, router_w, e_bias, y, topk_idx_out, topk_w_out)
    _req_weights(d, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    _req("workspace", workspace, _U8, 0, optional=True)
    _check("moe_forward", lib().moe_forward(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w), _ptr(e_bias), _ptr(w_gate),
        _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y),
        out_dtype_code(y), _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))


def device_status(stream=None) -> int:
    """Synchronise the stream and return (then clear) the device error word:
    0, a bounded-wait code, or a 0x4xx code of a skipped out-of-range index."""
    word = ctypes.c_int32(0)
    rc = lib().moe_device_status(_stream(stream), ctypes.byref(word))
    if rc not in (MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK):
        raise MoEError("moe_device_status", rc)
    return word.value


def launch_count() -> int:
    return int(lib().moe_launch_count())


def selftest_wait_timeout(limit_ns: int, stream=None):
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def moe_bias_update(cfg, topk_idx, e_bias, gamma: float, expert_load=None, stream=None):
    """Aux-loss-free balancing step: e_bias -= gamma where the expert was overloaded,
    += gamma where underloaded (in place); expert_load [E] int32 optionally receives the loads."""
    c = _cfg(cfg)
    if not isinstance(topk_idx, torch.Tensor) or topk_idx.dim() != 2 or topk_idx.shape[1] != c.num_experts_per_tok:
        raise ValueError(f"topk_idx: expected shape [T, {c.num_experts_per_tok}]")
    _req("topk_idx", topk_idx, _I32, 0)
    _req("e_bias", e_bias, _F32, c.n_routed_experts)
    _req("expert_load", expert_load, _I32, c.n_routed_experts, optional=True)
    _check("moe_bias_update", lib().moe_bias_update(ctypes.byref(_cfg(cfg)), topk_idx.shape[0],
                                                    _ptr(topk_idx), _ptr(e_bias), float(gamma),
                                                    _ptr(expert_load), _stream(stream)))


# ---------------------------------------------------------------- MXFP8 path

def mx_scale_bytes(rows: int, K: int) -> int:
    n = int(lib().moe_mx_scale_bytes(rows, K))
    if n < 0:
        raise MoEError("moe_mx_scale_bytes", MOE_ERR_UNSUPPORTED)
    return n


def moe_mx_quantize(src: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, stream=None):
    """E4M3 bytes q [rows, K] and scale atoms sf of the bf16 matrix src [rows, K]."""
    if not isinstance(src, torch.Tensor) or src.dim() != 2:
        raise ValueError("src: expected a 2-D [rows, K] tensor")
    rows, K = src.shape
    _req("src", src, _BF16, 0)
    _req("q", q, _U8, rows * K)
    _req("sf", sf, _U8, mx_scale_bytes(rows, K) if K % 128 == 0 and rows > 0 else 0)
    _check("moe_mx_quantize", lib().moe_mx_quantize(rows, K, _ptr(src), _ptr(q), _ptr(sf), _stream(stream)))


def mx_quantize(src: torch.Tensor, stream=None):
    """Allocate and fill (q uint8 [rows, K], sf uint8 [moe_mx_scale_bytes]) for a 2-D bf16 tensor."""
    src = src.reshape(-1, src.shape[-1])
    q = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    sf = torch.empty(mx_scale_bytes(*src.shape), dtype=torch.uint8, device=src.device)
    moe_mx_quantize(src, q, sf, stream)
    return q, sf


def workspace_size_mx(cfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size_mx", lib().moe_workspace_size_mx(ctypes.byref(_cfg(cfg)), T, ctypes.byref(n)))
    return n.value


def mx_routed_rows(cfg, T: int) -> int:
    n = ctypes.c_int64(0)
    _check("moe_mx_routed_rows", lib().moe_mx_routed_rows(ctypes.byref(_cfg(cfg)), T, ctypes.byref(n)))
    return n.value


def _mx_rows(d: _Dims, cfg):
    """(Rp, Tp): padded routed rows and the shared rows rounded up to 128 (0, 0 if T = 0)."""
    if d.T == 0:
        return 0, 0
    return mx_routed_rows(cfg, d.T), (d.T + 127) // 128 * 128


def moe_dispatch_mx(cfg, x, topk_idx, expert_offsets, expert_counts, xq_perm, xq_perm_sf, xq_shared,
                    xq_shared_sf, perm_src, row_of, workspace, stream=None):
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    Rp, Tp = _mx_rows(d, cfg)
    shared = d.S > 0
    _req("x", x, _BF16, 0)
    _req("topk_idx", topk_idx, _I32, d.T * d.k)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req("expert_counts", expert_counts, _I32, _n(d, d.E))
    _req("xq_perm", xq_perm, _U8, Rp * d.H)
    _req("xq_perm_sf", xq_perm_sf, _U8, mx_scale_bytes(Rp, d.H) if Rp else 0)
    _req("xq_shared", xq_shared, _U8, Tp * d.H if shared else 0, optional=not shared)
    _req("xq_shared_sf", xq_shared_sf, _U8, mx_scale_bytes(Tp, d.H) if shared and Tp else 0, optional=not shared)
    _req("perm_src", perm_src, _I32, Rp)
    _req("row_of", row_of, _I32, d.T * d.k)
    _req("workspace", workspace, _U8, 0)
    _check("moe_dispatch_mx", lib().moe_dispatch_mx(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(topk_idx), _ptr(expert_offsets),
        _ptr(expert_counts), _ptr(xq_perm), _ptr(xq_perm_sf), _ptr(xq_shared), _ptr(xq_shared_sf),
        _ptr(perm_src), _ptr(row_of), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def mx_weights(gate, up, down, shared_gate=None, shared_up=None, shared_down=None) -> MXWeights:
    """MXWeights from (q, sf) tensor pairs (the shared ones may be None)."""
    def m(pair):
        if pair is None:
            return MXMatrix(None, None)
        _req("MXFP8 weight bytes", pair[0], _U8, 0)
        _req("MXFP8 weight scales", pair[1], _U8, 0)
        return MXMatrix(pair[0].data_ptr(), pair[1].data_ptr())
    return MXWeights(m(gate), m(up), m(down), m(shared_gate), m(shared_up), m(shared_down))


def moe_forward_mx(cfg, x, router_w, e_bias, weights: MXWeights, y, topk_idx_out=None, topk_w_out=None,
                   workspace=None, stream=None):
    _req_layer(cfg, x, router_w, e_bias, y, topk_idx_out, topk_w_out)
    _req("workspace", workspace, _U8, 0, optional=True)
    _check("moe_forward_mx", lib().moe_forward_mx(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w), _ptr(e_bias), ctypes.byref(weights),
        _ptr(y), out_dtype_code(y), _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_experts_gate_up_mx(cfg, T, xq_perm, xq_perm_sf, xq_shared, xq_shared_sf, expert_offsets, expert_counts,
                           weights: MXWeights, hq_routed, hq_routed_sf, hq_shared, hq_shared_sf, stream=None):
    d = _Dims(cfg, T)
    Rp, Tp = _mx_rows(d, cfg)
    shared = d.S > 0
    _req("xq_perm", xq_perm, _U8, Rp * d.H)
    _req("xq_perm_sf", xq_perm_sf, _U8, mx_scale_bytes(Rp, d.H) if Rp else 0)
    _req("xq_shared", xq_shared, _U8, Tp * d.H if shared else 0, optional=not shared)
    _req("xq_shared_sf", xq_shared_sf, _U8, mx_scale_bytes(Tp, d.H) if shared and Tp else 0, optional=not shared)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req("expert_counts", expert_counts, _I32, _n(d, d.E))
    _req("hq_routed", hq_routed, _U8, Rp * d.I)
    _req("hq_routed_sf", hq_routed_sf, _U8, mx_scale_bytes(Rp, d.I) if Rp else 0)
    _req("hq_shared", hq_shared, _U8, Tp * d.SI if shared else 0, optional=not shared)
    _req("hq_shared_sf", hq_shared_sf, _U8, mx_scale_bytes(Tp, d.SI) if shared and Tp else 0, optional=not shared)
    _check("moe_experts_gate_up_mx", lib().moe_experts_gate_up_mx(
        ctypes.byref(_cfg(cfg)), T, _ptr(xq_perm), _ptr(xq_perm_sf), _ptr(xq_shared), _ptr(xq_shared_sf),
        _ptr(expert_offsets), _ptr(expert_counts), ctypes.byref(weights), _ptr(hq_routed), _ptr(hq_routed_sf),
        _ptr(hq_shared), _ptr(hq_shared_sf), _stream(stream)))


def moe_experts_down_mx(cfg, T, hq_routed, hq_routed_sf, hq_shared, hq_shared_sf, expert_offsets, expert_counts,
                        perm_src, topk_w, weights: MXWeights, y_perm, y_perm_scale, stream=None):
    d = _Dims(cfg, T)
    Rp, Tp = _mx_rows(d, cfg)
    shared = d.S > 0
    rows = Rp + (d.T if shared else 0)
    _req("hq_routed", hq_routed, _U8, Rp * d.I)
    _req("hq_routed_sf", hq_routed_sf, _U8, mx_scale_bytes(Rp, d.I) if Rp else 0)
    _req("hq_shared", hq_shared, _U8, Tp * d.SI if shared else 0, optional=not shared)
    _req("hq_shared_sf", hq_shared_sf, _U8, mx_scale_bytes(Tp, d.SI) if shared and Tp else 0, optional=not shared)
    _req("expert_offsets", expert_offsets, _I32, _n(d, d.E + 1))
    _req("expert_counts", expert_counts, _I32, _n(d, d.E))
    _req("perm_src", perm_src, _I32, Rp)
    _req("topk_w", topk_w, _F32, d.T * d.k)
    _req("y_perm", y_perm, _F16, rows * d.H)
    _req("y_perm_scale", y_perm_scale, _U8, rows * d.scale_cols)
    _check("moe_experts_down_mx", lib().moe_experts_down_mx(
        ctypes.byref(_cfg(cfg)), T, _ptr(hq_routed), _ptr(hq_routed_sf), _ptr(hq_shared), _ptr(hq_shared_sf),
        _ptr(expert_offsets), _ptr(expert_counts), _ptr(perm_src), _ptr(topk_w), ctypes.byref(weights),
        _ptr(y_perm), _ptr(y_perm_scale), _stream(stream)))


def moe_combine_mx(cfg, T, y_perm, y_perm_scale, row_of, y, stream=None):
    d = _Dims(cfg, T)
    _req_combine(d, _mx_rows(d, cfg)[0], y_perm, y_perm_scale, row_of, y)
    _check("moe_combine_mx", lib().moe_combine_mx(ctypes.byref(_cfg(cfg)), T, _ptr(y_perm), _ptr(y_perm_scale),
                                                  _ptr(row_of), _ptr(y), out_dtype_code(y), _stream(stream)))


# ---------------------------------------------------------------- backward pass

def workspace_size_bwd(cfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size_bwd", lib().moe_workspace_size_bwd(ctypes.byref(_cfg(cfg)), T, ctypes.byref(n)))
    return n.value


def _req_grads(d, dy, dx, d_router_w, d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down):
    _req("dy", dy, _BF16, d.T * d.H)
    _req("dx", dx, _F32, d.T * d.H)
    _req("d_router_w", d_router_w, _F32, d.E * d.H)
    _req_weights(d, d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down, prefix="d_")


def moe_backward(cfg, x, router_w, e_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, dy, dx, d_router_w,
                 d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down, workspace, stream=None):
    """Gradients of sum(y * dy): dx fp32 [T,H], d_router_w fp32 [E,H], expert and shared
    weight gradients bf16 in the weights' layouts (include/moe.h)."""
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _req("x", x, _BF16, 0)
    _req("router_w", router_w, _F32, d.E * d.H)
    _req("e_bias", e_bias, _F32, d.E)
    _req_weights(d, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    _req_grads(d, dy, dx, d_router_w, d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down)
    _req("workspace", workspace, _U8, 0)
    _check("moe_backward", lib().moe_backward(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w), _ptr(e_bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(dy), _ptr(dx), _ptr(d_router_w),
        _ptr(d_w_gate), _ptr(d_w_up), _ptr(d_w_down), _ptr(d_ws_gate), _ptr(d_ws_up), _ptr(d_ws_down),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


# ---------------------------------------------------------------- host buffers

def workspace_size_host(cfg, T: int, chunk_tokens: int, y_dtype: int = MOE_DTYPE_F32) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size_host", lib().moe_workspace_size_host(ctypes.byref(_cfg(cfg)), T, chunk_tokens,
                                                                    y_dtype, ctypes.byref(n)))
    return n.value


def moe_forward_host(cfg, x_host, router_w, e_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y_host,
                     chunk_tokens, workspace, stream=None):
    """The forward from pinned host x [T,H] bf16 to host y [T,H] (fp32 or bf16), copies
    overlapped with the layer chunk by chunk (include/moe.h)."""
    d = _req_layer(cfg, x_host, router_w, e_bias, y_host, None, None, x_where="host")
    _req_weights(d, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    _req("workspace", workspace, _U8, 0)
    _check("moe_forward_host", lib().moe_forward_host(
        ctypes.byref(_cfg(cfg)), x_host.shape[0], _ptr(x_host), _ptr(router_w), _ptr(e_bias), _ptr(w_gate),
        _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y_host), out_dtype_code(y_host),
        int(chunk_tokens), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_forward_train(cfg, x, router_w, e_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y, context,
                      stream=None):
    """The forward, keeping in `context` (workspace_size_bwd bytes) what moe_backward_train needs."""
    d = _req_layer(cfg, x, router_w, e_bias, y, None, None)
    _req_weights(d, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    _req("context", context, _U8, 0)
    _check("moe_forward_train", lib().moe_forward_train(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w), _ptr(e_bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y), out_dtype_code(y), _ptr(context),
        context.numel() * context.element_size(), _stream(stream)))


def moe_backward_train(cfg, x, router_w, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, dy, dx, d_router_w,
                       d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down, context, stream=None):
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _req("x", x, _BF16, 0)
    _req("router_w", router_w, _F32, d.E * d.H)
    _req_weights(d, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
    _req_grads(d, dy, dx, d_router_w, d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down)
    _req("context", context, _U8, 0)
    _check("moe_backward_train", lib().moe_backward_train(
        ctypes.byref(_cfg(cfg)), x.shape[0], _ptr(x), _ptr(router_w), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(dy), _ptr(dx), _ptr(d_router_w), _ptr(d_w_gate),
        _ptr(d_w_up), _ptr(d_w_down), _ptr(d_ws_gate), _ptr(d_ws_up), _ptr(d_ws_down), _ptr(context),
        context.numel() * context.element_size(), _stream(stream)))


# ---------------------------------------------------------------- expert parallelism

def ep_row_bytes(cfg) -> Tuple[int, int]:
    """(send row bytes, return row bytes) of the expert-parallel wire rows (include/moe.h)."""
    a, b = ctypes.c_int64(0), ctypes.c_int64(0)
    _check("moe_ep_row_bytes", lib().moe_ep_row_bytes(ctypes.byref(_cfg(cfg)), ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def ep_send_rows_max(cfg, T: int, world: int) -> int:
    """Send rows of T tokens at most: one per (token, destination rank)."""
    return T * min(int(_cfg(cfg).num_experts_per_tok), world)


def ep_workspace_size(cfg, world: int, T: int, R: int, n_local: Optional[int] = None) -> int:
    """Workspace bytes for moe_ep_send on T tokens and moe_ep_experts on R received rows
    with n_local local experts (default E/world)."""
    c = _cfg(cfg)
    if n_local is None:
        n_local = c.n_routed_experts // max(int(world), 1)
    n = ctypes.c_size_t(0)
    _check("moe_ep_workspace_size", lib().moe_ep_workspace_size(ctypes.byref(c), int(world), int(n_local), T, R,
                                                                ctypes.byref(n)))
    return n.value


def _host_i32(name, t, count):
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or t.dtype != torch.int32 or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous int32 CPU tensor")
    if t.numel() < count:
        raise ValueError(f"{name}: needs {count} elements, has {t.numel()}")


def ep_place(E: int, world: int, load, n_redundant: int, max_rep: int) -> torch.Tensor:
    """Placement table int32 [E, max_rep] (host) with n_redundant extra copies of the
    most loaded experts, from per-expert loads [E] (include/moe.h, moe_ep_place)."""
    ld = torch.as_tensor(load, dtype=torch.int64).cpu().contiguous()
    if ld.numel() != E:
        raise ValueError(f"load: needs {E} entries, has {ld.numel()}")
    out = torch.empty((E, max_rep), dtype=torch.int32)
    _check("moe_ep_place", lib().moe_ep_place(int(E), int(world), _ptr(ld), int(n_redundant), int(max_rep),
                                              _ptr(out)))
    return out


def ep_local_experts(E: int, world: int, rank: int, expert_ranks: torch.Tensor) -> Tuple[torch.Tensor, int]:
    """(local_of int32 [E], n_local) of rank `rank` under a placement table (host)."""
    if expert_ranks.dim() != 2 or expert_ranks.shape[0] != E:
        raise ValueError(f"expert_ranks: expected shape [{E}, max_rep]")
    _host_i32("expert_ranks", expert_ranks, 0)
    local_of = torch.empty(E, dtype=torch.int32)
    n = ctypes.c_int32(0)
    _check("moe_ep_local_experts", lib().moe_ep_local_experts(int(E), int(world), int(rank), _ptr(expert_ranks),
                                                              int(expert_ranks.shape[1]), _ptr(local_of),
                                                              ctypes.byref(n)))
    return local_of, n.value


def _ep_world(d, world: int, rank: int = 0) -> int:
    if world < 1 or d.E % world:
        raise ValueError(f"world {world} must divide n_routed_experts {d.E}")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    return d.E // world


def _wire_rows(name, t, row_bytes) -> int:
    if not isinstance(t, torch.Tensor) or t.dim() != 2 or t.shape[1] != row_bytes:
        raise ValueError(f"{name}: expected a uint8 tensor of shape [rows, {row_bytes}]")
    _req(name, t, _U8, 0)
    return int(t.shape[0])


def moe_ep_send(cfg, world: int, x, topk_idx, topk_w, send_counts, send_rows, send_row_of, workspace,
                expert_ranks=None, stream=None):
    """The source side's send rows, one per (token, destination rank), sorted by rank
    (include/moe.h); expert_ranks: the placement table [E, max_rep] on the device, or
    None for E/world-expert blocks."""
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    _ep_world(d, world)
    Wb, _ = ep_row_bytes(cfg)
    _req("x", x, _BF16, 0)
    _req("topk_idx", topk_idx, _I32, d.T * d.k)
    _req("topk_w", topk_w, _F32, d.T * d.k)
    max_rep = 1
    if expert_ranks is not None:
        if expert_ranks.dim() != 2 or expert_ranks.shape[0] != d.E:
            raise ValueError(f"expert_ranks: expected shape [{d.E}, max_rep]")
        _req("expert_ranks", expert_ranks, _I32, 0)
        max_rep = int(expert_ranks.shape[1])
    _req("send_counts", send_counts, _I32, world)
    if _wire_rows("send_rows", send_rows, Wb) < ep_send_rows_max(cfg, d.T, world):
        raise ValueError(f"send_rows: needs {ep_send_rows_max(cfg, d.T, world)} rows")
    _req("send_row_of", send_row_of, _I32, d.T * d.k)
    _req("workspace", workspace, _U8, 0)
    _check("moe_ep_send", lib().moe_ep_send(
        ctypes.byref(_cfg(cfg)), int(world), d.T, _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(expert_ranks),
        max_rep, _ptr(send_counts), _ptr(send_rows), _ptr(send_row_of), _ptr(workspace), workspace.numel(),
        _stream(stream)))


def moe_ep_experts(cfg, world: int, rank: int, x, recv_rows, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                   return_rows, y_shared, y_shared_scale, workspace, local_of=None, n_local=None, stream=None):
    """Rank `rank`'s experts over the received send rows -> return rows, and the shared
    experts over its own tokens x (include/moe.h).  Weights are the rank's experts: its
    E/world block, or with local_of (device int32 [E], from ep_local_experts) its
    n_local experts in ascending id order."""
    d = _Dims(cfg, _rows_2d("x", x, _cfg(cfg).hidden_size))
    El = _ep_world(d, world, rank)
    if local_of is not None:
        if n_local is None or not 1 <= int(n_local) <= d.E:
            raise ValueError(f"n_local must be in [1, {d.E}] with local_of")
        _req("local_of", local_of, _I32, d.E)
        El = int(n_local)
    Wb, Wr = ep_row_bytes(cfg)
    R = _wire_rows("recv_rows", recv_rows, Wb)
    if _wire_rows("return_rows", return_rows, Wr) < R:
        raise ValueError(f"return_rows: needs {R} rows")
    shared = d.S > 0 and d.T > 0
    _req("x", x, _BF16, 0)
    _req("w_gate", w_gate, _BF16, El * d.I * d.H)
    _req("w_up", w_up, _BF16, El * d.I * d.H)
    _req("w_down", w_down, _BF16, El * d.I * d.H)
    for name, t in (("ws_gate", ws_gate), ("ws_up", ws_up), ("ws_down", ws_down)):
        _req(name, t, _BF16, d.SI * d.H, optional=not shared)
    _req("y_shared", y_shared, _F16, d.T * d.H, optional=not shared)
    _req("y_shared_scale", y_shared_scale, _U8, d.T * d.scale_cols, optional=not shared)
    _req("workspace", workspace, _U8, 0)
    _check("moe_ep_experts", lib().moe_ep_experts(
        ctypes.byref(_cfg(cfg)), int(world), int(rank), _ptr(local_of), El, d.T, _ptr(x), R, _ptr(recv_rows),
        _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(return_rows), _ptr(y_shared),
        _ptr(y_shared_scale), _ptr(workspace), workspace.numel(), _stream(stream)))


def moe_ep_combine(cfg, world: int, back_rows, send_row_of, y_shared, y_shared_scale, y, stream=None):
    """y [T, H] = the shared rows + the returned rows of each token (include/moe.h);
    back_rows holds exactly the rows that came back (sum of the send counts)."""
    d = _Dims(cfg, _rows_2d("y", y, _cfg(cfg).hidden_size))
    _ep_world(d, world)
    _, Wr = ep_row_bytes(cfg)
    n = _wire_rows("back_rows", back_rows, Wr)
    if n > ep_send_rows_max(cfg, d.T, world):
        raise ValueError(f"back_rows: more than {ep_send_rows_max(cfg, d.T, world)} rows")
    _req("send_row_of", send_row_of, _I32, d.T * d.k)
    _req("y_shared", y_shared, _F16, d.T * d.H, optional=d.S == 0)
    _req("y_shared_scale", y_shared_scale, _U8, d.T * d.scale_cols, optional=d.S == 0)
    _req("y", y, _OUT, d.T * d.H)
    _check("moe_ep_combine", lib().moe_ep_combine(
        ctypes.byref(_cfg(cfg)), int(world), d.T, n, _ptr(back_rows), _ptr(send_row_of), _ptr(y_shared),
        _ptr(y_shared_scale), _ptr(y), out_dtype_code(y), _stream(stream)))
