"""The C ABI library on the host (no GPU needed): it builds, loads, exports every
symbol include/moe.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from sparse_moe_layer_noaux_b200 import abi, build
from sparse_moe_layer_noaux_b200.workloads import MID, TINY, V3_PREFILL

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def test_header_symbols_exported(lib):
    names = declared_functions()
    assert {"moe_route", "moe_dispatch", "moe_forward", "moe_workspace_size",
            "moe_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(8):
        assert abi.status_string(code) != "unknown status", code
    assert abi.status_string(99) == "unknown status"


def fwd(lib, c, T, ptrs, ws, nbytes, y_dtype=0):
    """moe_forward with the 12 pointer arguments x .. topk_w_out given as a list."""
    return lib.moe_forward(ctypes.byref(c), T, *ptrs[:10], y_dtype, ptrs[10], ptrs[11], ws, nbytes, None)


def _cfg(**kw):
    c = abi.MoEConfig.from_shape(TINY)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,code", [
    (dict(n_group=3), abi.MOE_ERR_INVALID_ARG),               # E % G != 0
    (dict(topk_group=5), abi.MOE_ERR_INVALID_ARG),            # TG > G
    (dict(num_experts_per_tok=0), abi.MOE_ERR_INVALID_ARG),
    (dict(num_experts_per_tok=9), abi.MOE_ERR_INVALID_ARG),   # k > TG * E / G = 8
    (dict(norm_topk_prob=2), abi.MOE_ERR_INVALID_ARG),
    (dict(hidden_size=0), abi.MOE_ERR_INVALID_ARG),
    (dict(n_shared_experts=-1), abi.MOE_ERR_INVALID_ARG),
    (dict(hidden_size=200), abi.MOE_ERR_UNSUPPORTED),          # not a multiple of 64
    (dict(moe_intermediate_size=96), abi.MOE_ERR_UNSUPPORTED),
    (dict(n_routed_experts=512, n_group=8), abi.MOE_ERR_UNSUPPORTED),
])
def test_bad_config_rejected(lib, kw, code):
    c = _cfg(**kw)
    n = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(c), 64, ctypes.byref(n)) == code
    p = ctypes.c_void_p(1 << 20)
    assert lib.moe_route(ctypes.byref(c), 64, p, p, p, p, p, p, 1 << 30, None) == code
    assert fwd(lib, c, 64, [p] * 12, p, 1 << 30) == code


def test_negative_tokens_and_nulls(lib):
    c = _cfg()
    p = ctypes.c_void_p(1 << 20)
    n = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(c), -1, ctypes.byref(n)) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_workspace_size(None, 4, ctypes.byref(n)) == abi.MOE_ERR_INVALID_ARG
    assert lib.moe_route(ctypes.byref(c), 4, None, p, p, p, p, p, 1 << 30, None) == abi.MOE_ERR_INVALID_ARG
    args = [p] * 12
    args[9] = None  # y
    assert fwd(lib, c, 4, args, p, 1 << 30) == abi.MOE_ERR_INVALID_ARG
    assert fwd(lib, c, 4, [p] * 12, p, 1 << 30, y_dtype=7) == abi.MOE_ERR_INVALID_ARG


def test_misaligned_pointer_rejected(lib):
    c = _cfg()
    p = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 2)
    assert lib.moe_route(ctypes.byref(c), 4, bad, p, p, p, p, p, 1 << 30, None) == abi.MOE_ERR_UNSUPPORTED
    args = [p] * 12
    args[3] = bad  # w_gate
    assert fwd(lib, c, 4, args, p, 1 << 30) == abi.MOE_ERR_UNSUPPORTED


def test_workspace_too_small_rejected(lib):
    c = _cfg()
    need = abi.workspace_size(c, 64)
    p = ctypes.c_void_p(1 << 20)
    assert fwd(lib, c, 64, [p] * 12, p, need - 1) == abi.MOE_ERR_WORKSPACE
    assert fwd(lib, c, 64, [p] * 12, None, need) == abi.MOE_ERR_WORKSPACE
    assert lib.moe_route(ctypes.byref(c), 64, p, p, p, p, p, None, need, None) == abi.MOE_ERR_WORKSPACE


def test_zero_tokens_needs_nothing(lib):
    c = _cfg()
    # T = 0 returns before any pointer or workspace is looked at.
    assert fwd(lib, c, 0, [None] * 12, None, 0) == abi.MOE_OK
    assert lib.moe_route(ctypes.byref(c), 0, None, None, None, None, None, None, 0, None) == abi.MOE_OK


def test_workspace_size_scales(lib):
    small = abi.workspace_size(MID.with_(T=16), 16)
    big = abi.workspace_size(MID, MID.T)
    assert 0 < small < big
    # The prefill workspace holds x_perm, h, y_perm: a few GB, well inside 180 GB.
    ws = abi.workspace_size(V3_PREFILL, V3_PREFILL.T)
    assert 4.5e9 < ws < 5.5e9  # x_perm 1.9 GB + h 0.6 GB + block-scaled fp16 y_perm 2.2 GB


def test_workspace_size_of_an_empty_batch(lib):
    # Sizing a workspace for T = 0 is a valid query (no router tiles at all).
    assert 0 < abi.workspace_size(TINY, 0) < abi.workspace_size(TINY, 64)
    assert 0 < abi.workspace_size_mx(TINY, 0) < abi.workspace_size_mx(TINY, 64)


def test_mx_host_queries(lib):
    # Scale atoms: 512 bytes per 128 rows x 128 K, rows rounded up to 128.
    assert abi.mx_scale_bytes(1, 128) == 512
    assert abi.mx_scale_bytes(129, 256) == 2 * 2 * 512
    assert lib.moe_mx_scale_bytes(128, 100) == -1
    # Padded routed rows: T*k + 127*E rounded up to 128.
    assert abi.mx_routed_rows(V3_PREFILL, V3_PREFILL.T) == (16384 * 8 + 127 * 256 + 127) // 128 * 128
    # Shapes the MXFP8 GEMMs do not take.
    with pytest.raises(abi.MoEError) as ei:
        abi.workspace_size_mx(TINY.with_(hidden_size=320), 4)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    with pytest.raises(abi.MoEError):
        abi.workspace_size_mx(TINY.with_(moe_intermediate_size=192), 4)
    # The MXFP8 prefill workspace: E4M3 x_perm 1.17 GB + h 0.34 GB + y_perm 2.6 GB.
    ws = abi.workspace_size_mx(V3_PREFILL, V3_PREFILL.T)
    assert 4.0e9 < ws < 4.8e9
    # Quantising nothing is a no-op; a K that is not a multiple of 128 is refused.
    assert lib.moe_mx_quantize(0, 256, None, None, None, None) == abi.MOE_OK
    assert lib.moe_mx_quantize(4, 96, None, None, None, None) == abi.MOE_ERR_UNSUPPORTED


def test_row_space_beyond_int32_rejected(lib):
    # Row indices are int32: the routed rows, their per-expert padding to 128
    # and the shared rows must all fit.  A batch whose unpadded rows fit but
    # whose padded ones do not is refused before any size is computed.
    c = abi.MoEConfig.from_shape(V3_PREFILL)
    n = ctypes.c_size_t(0)
    k, E = V3_PREFILL.k, V3_PREFILL.E
    limit = (1 << 31) - 256
    T_pad_overflow = (limit - 128 * E) // (k + 1) + 1
    assert T_pad_overflow * (k + 1) < limit
    assert lib.moe_workspace_size(ctypes.byref(c), T_pad_overflow, ctypes.byref(n)) == abi.MOE_ERR_UNSUPPORTED
    T_fits = (limit - 128 * E) // (k + 1) - 1
    assert lib.moe_workspace_size(ctypes.byref(c), T_fits, ctypes.byref(n)) == abi.MOE_OK


def test_host_forward_workspace_holds_two_slots_and_one_chunk(lib):
    # Two staging slots each for x (bf16) and y (fp32 or bf16), plus the device
    # forward's workspace for the largest chunk (a full chunk or the last one).
    s = V3_PREFILL
    H, T = s.H, s.T
    whole = abi.workspace_size_host(s, T, 0, abi.MOE_DTYPE_F32)
    assert whole >= abi.workspace_size(s, T) + 2 * T * H * 2 + 2 * T * H * 4
    chunk = 6000                                   # 3 chunks: 6000, 6000, 4384 rows
    per = abi.workspace_size_host(s, T, chunk, abi.MOE_DTYPE_F32)
    fwd = max(abi.workspace_size(s, chunk), abi.workspace_size(s, T - 2 * chunk))
    assert per >= fwd + 2 * chunk * H * 2 + 2 * chunk * H * 4
    assert per < whole
    assert abi.workspace_size_host(s, T, chunk, abi.MOE_DTYPE_BF16) < per
    # chunk_tokens >= T is one chunk, like 0.
    assert abi.workspace_size_host(s, T, T + 5, abi.MOE_DTYPE_F32) == whole
    with pytest.raises(abi.MoEError):
        abi.workspace_size_host(s, T, chunk, 7)     # not a moe_dtype
