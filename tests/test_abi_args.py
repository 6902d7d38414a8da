"""Argument checks of the Python binding, on the CPU.

The C ABI takes raw pointers, so the binding checks every tensor (element type,
contiguity, device, minimum size) before passing its address.  Here the library's
compute entry points are replaced by a recorder (nothing is launched; the host-only
size queries still go to the real library) and device placement is relaxed to the
CPU, so the checks themselves run: every wrapper accepts buffers allocated exactly
as the GPU tests allocate them, with and without a shared expert and for T = 0, and
rejects a wrong dtype, a short buffer, a strided view or a wrong row width before
the library is called."""
import pytest
import torch

from sparse_moe_layer_noaux_b200 import abi
from sparse_moe_layer_noaux_b200.workloads import TINY, MoEShape

NOSHARED = MoEShape("noshared", T=50, hidden_size=256, n_routed_experts=16, n_group=1, topk_group=1,
                    num_experts_per_tok=3, moe_intermediate_size=128, n_shared_experts=0,
                    routed_scaling_factor=1.0, norm_topk_prob=True, seed=9)
HOST_QUERIES = ("moe_workspace_size", "moe_workspace_size_mx", "moe_workspace_size_bwd",
                "moe_workspace_size_host", "moe_mx_routed_rows", "moe_mx_scale_bytes", "moe_status_string",
                "moe_ep_row_bytes", "moe_ep_workspace_size", "moe_ep_place", "moe_ep_local_experts")


class _Recorder:
    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in HOST_QUERIES:
            return getattr(self.real, name)

        def call(*args):
            self.calls.append(name)
            return abi.MOE_OK
        return call


@pytest.fixture()
def rec(monkeypatch):
    r = _Recorder(abi.lib())
    monkeypatch.setattr(abi, "lib", lambda: r)
    monkeypatch.setattr(abi, "_on_current_cuda_device", lambda t: t.device.type == "cpu")
    monkeypatch.setattr(abi, "_stream", lambda s: None)
    return r


def e(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def layer_tensors(s):
    T, H, E, I, S, k = s.T, s.H, s.E, s.I, s.S, s.k
    return dict(x=e(T, H), router_w=e(E, H, dtype=torch.float32), e_bias=e(E, dtype=torch.float32),
                w_gate=e(E, I, H), w_up=e(E, I, H), w_down=e(E, H, I),
                ws_gate=e(S * I, H), ws_up=e(S * I, H), ws_down=e(H, S * I))


def run_all(s):
    """Every wrapper once with buffers shaped as the GPU tests make them."""
    T, H, E, I, S, k = s.T, s.H, s.E, s.I, s.S, s.k
    cfg = abi.MoEConfig.from_shape(s)
    L = layer_tensors(s)
    W = (L["w_gate"], L["w_up"], L["w_down"], L["ws_gate"], L["ws_up"], L["ws_down"])
    i32, f32, u8, f16 = torch.int32, torch.float32, torch.uint8, torch.float16
    ws = e(256, dtype=u8)
    idx, w = e(T, k, dtype=i32), e(T, k, dtype=f32)
    offsets, perm_src, row_of = e(E + 1, dtype=i32), e(T * k, dtype=i32), e(T, k, dtype=i32)
    x_perm = e(T * k, H)
    abi.moe_route(cfg, L["x"], L["router_w"], L["e_bias"], idx, w, ws)
    abi.moe_dispatch(cfg, L["x"], idx, offsets, x_perm, perm_src, row_of, ws)
    abi.moe_dispatch_noalloc(cfg, L["x"], idx, offsets, x_perm, perm_src, row_of)
    h_r, h_s = e(T * k, I), e(T, S * I)
    y_perm, y_sc = e(T * k + T, H, dtype=f16), e(T * k + T, abi.y_perm_scale_cols(H), dtype=u8)
    abi.moe_experts(cfg, T, L["x"], x_perm, offsets, perm_src, w, *W, h_r, h_s, y_perm, y_sc)
    abi.moe_experts_gate_up(cfg, T, L["x"], x_perm, offsets, L["w_gate"], L["w_up"], L["ws_gate"], L["ws_up"],
                            h_r, h_s)
    abi.moe_experts_down(cfg, T, h_r, h_s, offsets, perm_src, w, L["w_down"], L["ws_down"], y_perm, y_sc)
    for dt in (f32, torch.bfloat16):
        abi.moe_combine(cfg, T, y_perm, y_sc, row_of, e(T, H, dtype=dt))
        abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], *W, e(T, H, dtype=dt), idx, w, ws)
    abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], *W, e(T, H, dtype=f32))
    abi.moe_bias_update(cfg, idx, L["e_bias"].clone(), 1e-3, e(E, dtype=i32))
    # MXFP8
    q = e(T, H, dtype=u8)
    abi.moe_mx_quantize(L["x"], q, e(abi.mx_scale_bytes(max(T, 1), H), dtype=u8))
    Rp = abi.mx_routed_rows(cfg, T) if T else 0
    Tp = (T + 127) // 128 * 128
    sb = lambda r, K: e(abi.mx_scale_bytes(r, K) if r and K else 0, dtype=u8)
    counts, perm_mx = e(E, dtype=i32), e(Rp, dtype=i32)
    xq, xsf, xqs, xssf = e(Rp, H, dtype=u8), sb(Rp, H), e(Tp, H, dtype=u8), sb(Tp, H)
    abi.moe_dispatch_mx(cfg, L["x"], idx, offsets, counts, xq, xsf, xqs, xssf, perm_mx, row_of, ws)
    mxw = abi.mx_weights((e(E * I, H, dtype=u8), e(64, dtype=u8)), (e(E * I, H, dtype=u8), e(64, dtype=u8)),
                         (e(E * H, I, dtype=u8), e(64, dtype=u8)))
    abi.moe_forward_mx(cfg, L["x"], L["router_w"], L["e_bias"], mxw, e(T, H, dtype=f32), idx, w, ws)
    hq, hsf, hqs, hssf = e(Rp, I, dtype=u8), sb(Rp, I), e(Tp, S * I, dtype=u8), sb(Tp, S * I)
    abi.moe_experts_gate_up_mx(cfg, T, xq, xsf, xqs, xssf, offsets, counts, mxw, hq, hsf, hqs, hssf)
    yp_mx = e(Rp + T, H, dtype=f16)
    ysc_mx = e(Rp + T, abi.y_perm_scale_cols(H), dtype=u8)
    abi.moe_experts_down_mx(cfg, T, hq, hsf, hqs, hssf, offsets, counts, perm_mx, w, mxw, yp_mx, ysc_mx)
    abi.moe_combine_mx(cfg, T, yp_mx, ysc_mx, row_of, e(T, H, dtype=f32))
    # backward, training pair, host buffers
    G = (e(E, I, H), e(E, I, H), e(E, H, I), e(S * I, H), e(S * I, H), e(H, S * I))
    dy, dx, drw = e(T, H), e(T, H, dtype=f32), e(E, H, dtype=f32)
    abi.moe_backward(cfg, L["x"], L["router_w"], L["e_bias"], *W, dy, dx, drw, *G, ws)
    abi.moe_forward_train(cfg, L["x"], L["router_w"], L["e_bias"], *W, e(T, H, dtype=f32), ws)
    abi.moe_backward_train(cfg, L["x"], L["router_w"], *W, dy, dx, drw, *G, ws)
    abi.moe_forward_host(cfg, L["x"], L["router_w"], L["e_bias"], *W, e(T, H, dtype=f32), 0, ws)
    # expert parallelism (world 2: this rank holds E/2 experts and receives R rows)
    world, R = 2, 7
    El = E // world
    Wb, Wr = abi.ep_row_bytes(cfg)
    n_send = abi.ep_send_rows_max(cfg, T, world)
    ws_ep = e(abi.ep_workspace_size(cfg, world, T, R), dtype=u8)
    send_row_of = e(T, k, dtype=i32)
    placement = abi.ep_place(E, world, torch.arange(E, dtype=torch.int64), 2, 2)
    local_of, n_local = abi.ep_local_experts(E, world, 1, placement)
    abi.moe_ep_send(cfg, world, L["x"], idx, w, e(world, dtype=i32), e(n_send, Wb, dtype=u8), send_row_of, ws_ep,
                    expert_ranks=placement)
    y_sh, y_sh_sc = e(T, H, dtype=f16), e(T, abi.y_perm_scale_cols(H), dtype=u8)
    abi.moe_ep_experts(cfg, world, 1, L["x"], e(R, Wb, dtype=u8), e(n_local, I, H), e(n_local, I, H),
                       e(n_local, H, I), L["ws_gate"], L["ws_up"], L["ws_down"], e(R, Wr, dtype=u8), y_sh, y_sh_sc,
                       ws_ep, local_of=local_of, n_local=n_local)
    abi.moe_ep_combine(cfg, world, e(n_send, Wr, dtype=u8), send_row_of, y_sh, y_sh_sc, e(T, H, dtype=f32))


@pytest.mark.parametrize("shape", [TINY, NOSHARED, TINY.with_(name="empty", T=0)], ids=lambda s: s.name)
def test_valid_buffers_reach_the_library(rec, shape):
    run_all(shape)
    assert len(rec.calls) == 25 and "moe_backward_train" in rec.calls and "moe_ep_combine" in rec.calls


def test_bad_arguments_are_rejected_before_the_call(rec):
    s = TINY
    T, H, E, I, k = s.T, s.H, s.E, s.I, s.k
    cfg = abi.MoEConfig.from_shape(s)
    L = layer_tensors(s)
    W = (L["w_gate"], L["w_up"], L["w_down"], L["ws_gate"], L["ws_up"], L["ws_down"])
    idx, w = e(T, k, dtype=torch.int32), e(T, k, dtype=torch.float32)
    y = e(T, H, dtype=torch.float32)
    ws = e(256, dtype=torch.uint8)
    Wb, Wr = abi.ep_row_bytes(cfg)
    bad = [
        (TypeError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"].bfloat16(), L["e_bias"], *W, y)),
        (TypeError, lambda: abi.moe_forward(cfg, L["x"].float(), L["router_w"], L["e_bias"], *W, y)),
        (TypeError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], *W, y.half())),
        (ValueError, lambda: abi.moe_forward(cfg, L["x"][:, : H // 2], L["router_w"], L["e_bias"], *W, y)),
        (ValueError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"][: E - 1], L["e_bias"], *W, y)),
        (ValueError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], L["w_gate"][:-1],
                                             *W[1:], y)),
        (ValueError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], *W[:3], None, None,
                                             None, y)),   # S = 1 needs the shared weights
        (ValueError, lambda: abi.moe_forward(cfg, L["x"], L["router_w"], L["e_bias"], *W, y[: T - 1])),
        (ValueError, lambda: abi.moe_route(cfg, L["x"], L["router_w"], L["e_bias"], idx.t(), w, ws)),
        (TypeError, lambda: abi.moe_route(cfg, L["x"], L["router_w"], L["e_bias"], idx.long(), w, ws)),
        (ValueError, lambda: abi.moe_dispatch(cfg, L["x"], idx, e(E + 1, dtype=torch.int32), e(T * k - 1, H),
                                              e(T * k, dtype=torch.int32), idx, ws)),
        (TypeError, lambda: abi.moe_combine(cfg, T, e(T * k + T, H), e(T * k + T, 8, dtype=torch.uint8),
                                            idx, y)),   # y_perm must be fp16
        (TypeError, lambda: abi.moe_forward_host(cfg, L["x"], L["router_w"], L["e_bias"], *W, [0.0], 0, ws)),
        (ValueError, lambda: abi.moe_ep_experts(cfg, 3, 0, L["x"], e(4, Wb, dtype=torch.uint8), *W,
                                                e(4, Wr, dtype=torch.uint8), e(T, H, dtype=torch.float16),
                                                e(T, 8, dtype=torch.uint8), ws)),   # 3 does not divide E
        (ValueError, lambda: abi.moe_ep_experts(cfg, 2, 2, L["x"], e(4, Wb, dtype=torch.uint8), *W,
                                                e(4, Wr, dtype=torch.uint8), e(T, H, dtype=torch.float16),
                                                e(T, 8, dtype=torch.uint8), ws)),   # rank outside [0, 2)
        (ValueError, lambda: abi.moe_ep_experts(cfg, 2, 0, L["x"], e(4, Wb, dtype=torch.uint8), *W,
                                                e(3, Wr, dtype=torch.uint8), e(T, H, dtype=torch.float16),
                                                e(T, 8, dtype=torch.uint8), ws)),   # fewer return rows than received
        (ValueError, lambda: abi.moe_ep_send(cfg, 2, L["x"], idx, w, e(2, dtype=torch.int32),
                                             e(T * 2, Wb - 16, dtype=torch.uint8), idx, ws)),   # row width
        (ValueError, lambda: abi.moe_ep_send(cfg, 2, L["x"], idx, w, e(2, dtype=torch.int32),
                                             e(T * 2 - 1, Wb, dtype=torch.uint8), idx, ws)),   # too few rows
        (TypeError, lambda: abi.moe_ep_combine(cfg, 2, e(T, Wr, dtype=torch.uint8), idx.float(),
                                               e(T, H, dtype=torch.float16), e(T, 8, dtype=torch.uint8), y)),
        (ValueError, lambda: abi.moe_ep_experts(cfg, 2, 0, L["x"], e(4, Wb, dtype=torch.uint8), *W,
                                                e(4, Wr, dtype=torch.uint8), e(T, H, dtype=torch.float16),
                                                e(T, 8, dtype=torch.uint8), ws,
                                                local_of=e(E, dtype=torch.int32))),   # local_of without n_local
        (ValueError, lambda: abi.moe_ep_send(cfg, 2, L["x"], idx, w, e(2, dtype=torch.int32),
                                             e(T * 2, Wb, dtype=torch.uint8), idx, ws,
                                             expert_ranks=e(E - 1, 2, dtype=torch.int32))),   # table rows
        (ValueError, lambda: abi.moe_ep_combine(cfg, 2, e(2 * T + 1, Wr, dtype=torch.uint8), idx,
                                                e(T, H, dtype=torch.float16), e(T, 8, dtype=torch.uint8), y)),
    ]
    for exc, call in bad:
        with pytest.raises(exc):
            call()
    assert rec.calls == []
