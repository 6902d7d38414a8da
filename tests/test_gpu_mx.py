"""MXFP8 expert FFNs on B200 against the MXFP8 oracle ("DeepSeek-V3 notes"
(knlb.dev), § fp8: fine-grained block-wise E4M3 quantisation with scales from
each block's maximum).

Quantisation of bf16 inputs (weights, dispatched token rows) is bit-exact with
the oracle: the same power-of-two scale codes and the same E4M3 bytes.  The
layer output is compared with the oracle's float64 MXFP8 layer on the same
bits, at the bf16 path's tolerances."""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_noaux_b200 import MoELayerMX, abi
from sparse_moe_layer_noaux_b200.workloads import (MID, TINY, V3_DECODE, V3_PREFILL, V3_SKEWED, MoEShape,
                                                   bf16_bits, make_inputs)
from tests import parity
from tests.test_oracle_mx import decode_e4m3

pytestmark = pytest.mark.gpu

E4M3 = np.array([decode_e4m3(b) for b in range(256)])


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import build
    build.build()
    oracle.build()
    yield
    torch.cuda.empty_cache()


def unpack_codes(sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Scale codes [rows, K/32] out of the 512-byte atoms (128 rows x 4 codes per
    K slice of 128; row r, block j at 16*(r%32) + 4*(r//32) + j)."""
    r = np.arange(rows)[:, None]
    b = np.arange(K // 32)[None, :]
    off = ((r // 128) * (K // 128) + b // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + b % 4
    return sf[off]


def check_rows_quantised(q_bytes, codes, x_bits_rows):
    """GPU bytes and codes of some rows == the oracle's quantisation of the bf16 rows."""
    oq, oc, _ = oracle.mx_quantize(x_bits_rows)
    np.testing.assert_array_equal(codes, oc)
    np.testing.assert_array_equal(q_bytes, oracle.e4m3_bits(oq))


@pytest.mark.parametrize("rows,K", [(200, 256), (128, 7168), (3, 384)])
def test_quantize_is_bit_exact(rows, K):
    g = torch.Generator(device="cuda").manual_seed(rows + K)
    mag = torch.exp2(torch.randint(-12, 12, (rows, K // 32, 1), device="cuda", generator=g).float())
    src = (torch.randn((rows, K // 32, 32), device="cuda", generator=g) * mag).view(rows, K).bfloat16()
    src[0, :32] = 0                               # an all-zero block
    src[-1, 32:64] = 448.0                        # exactly at the E4M3 maximum
    src[-1, 64:96] = torch.tensor(2.0 ** -120)    # far below 1
    q, sf = abi.mx_quantize(src)
    torch.cuda.synchronize()
    check_rows_quantised(q.cpu().numpy(), unpack_codes(sf.cpu().numpy(), rows, K), bf16_bits(src))


def test_quantize_v3_expert_weights_bit_exact():
    shape = V3_PREFILL
    g = torch.Generator(device="cuda").manual_seed(11)
    w = (torch.randn((shape.I, shape.H), device="cuda", generator=g) * 0.02).bfloat16()
    q, sf = abi.mx_quantize(w)
    torch.cuda.synchronize()
    check_rows_quantised(q.cpu().numpy(), unpack_codes(sf.cpu().numpy(), shape.I, shape.H), bf16_bits(w))


def routed(shape, inp):
    cfg = abi.MoEConfig.from_shape(shape)
    T, k = shape.T, shape.k
    # one buffer serves moe_route (bf16 workspace size) and moe_dispatch_mx (MXFP8 size)
    ws = torch.empty(max(abi.workspace_size_mx(cfg, T), abi.workspace_size(cfg, T)), dtype=torch.uint8,
                     device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    return cfg, ws, idx, w


SMALL_MX = [
    TINY,
    TINY.with_(name="tiny_T1", T=1, seed=21),
    TINY.with_(name="tiny_T3", T=3, seed=22),
    MoEShape("ragged", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
             num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
             routed_scaling_factor=2.5, norm_topk_prob=True, seed=7),
    # ~1100 rows per expert (9 row tiles, the last ragged), I = 3 x 128, two shared experts;
    # T >= 2048 puts the router logits on the tensor cores.
    MoEShape("mx_tiles", T=2200, hidden_size=512, n_routed_experts=8, n_group=2, topk_group=1,
             num_experts_per_tok=4, moe_intermediate_size=384, n_shared_experts=2,
             routed_scaling_factor=1.3, norm_topk_prob=False, seed=8),
    MoEShape("noshared", T=500, hidden_size=256, n_routed_experts=16, n_group=1, topk_group=1,
             num_experts_per_tok=3, moe_intermediate_size=128, n_shared_experts=0,
             routed_scaling_factor=1.0, norm_topk_prob=True, seed=9),
    # DeepSeek-V2's expert counts (160 routed in groups of 20, top-6, 2 shared).
    MoEShape("v2_groups", T=700, hidden_size=256, n_routed_experts=160, n_group=8, topk_group=3,
             num_experts_per_tok=6, moe_intermediate_size=128, n_shared_experts=2,
             routed_scaling_factor=16.0, norm_topk_prob=False, seed=11),
]


@pytest.mark.parametrize("shape", [SMALL_MX[0], SMALL_MX[2], SMALL_MX[3], SMALL_MX[5]], ids=lambda s: s.name)
def test_dispatch_mx_bit_exact(shape):
    inp = make_inputs(shape, "cuda")
    cfg, ws, idx, _ = routed(shape, inp)
    T, k, E, H = shape.T, shape.k, shape.E, shape.H
    Rp = abi.mx_routed_rows(cfg, T)
    Tp = (T + 127) // 128 * 128
    dev = "cuda"
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    xq = torch.empty((Rp, H), dtype=torch.uint8, device=dev)
    xsf = torch.empty(abi.mx_scale_bytes(Rp, H), dtype=torch.uint8, device=dev)
    xqs = torch.empty((Tp, H), dtype=torch.uint8, device=dev)
    xssf = torch.empty(abi.mx_scale_bytes(Tp, H), dtype=torch.uint8, device=dev)
    perm_src = torch.full((Rp,), -1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    abi.moe_dispatch_mx(cfg, inp["x"], idx, offsets, counts, xq, xsf, xqs, xssf, perm_src, row_of, ws)
    torch.cuda.synchronize()
    flat = idx.cpu().numpy().reshape(-1)
    cnt = np.bincount(flat, minlength=E)
    np.testing.assert_array_equal(counts.cpu().numpy(), cnt)
    pad = (cnt + 127) // 128 * 128
    np.testing.assert_array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(pad)]))
    assert offsets[-1].item() <= Rp
    # Stable order inside each segment: the slots of expert e in ascending (t, j).
    ro = row_of.cpu().numpy().reshape(-1)
    off = offsets.cpu().numpy()
    order = np.argsort(flat, kind="stable")
    want = np.empty_like(ro)
    for e in range(E):
        sl = order[flat[order] == e]
        want[sl] = off[e] + np.arange(len(sl))
    np.testing.assert_array_equal(ro, want)
    ps = perm_src.cpu().numpy()
    np.testing.assert_array_equal(ps[ro], np.arange(T * k))
    # Quantised rows: row_of[t, j] holds x[t]'s MXFP8 bytes and codes; shared rows in token order.
    x_bits = bf16_bits(inp["x"])
    codes = unpack_codes(xsf.cpu().numpy(), Rp, H)
    xq_np = xq.cpu().numpy()
    tok = np.arange(T * k) // k
    check_rows_quantised(xq_np[ro], codes[ro], x_bits[tok])
    if shape.S > 0:
        check_rows_quantised(xqs.cpu().numpy()[:T], unpack_codes(xssf.cpu().numpy(), Tp, H)[:T], x_bits)


def run_forward_mx(shape, inp, out_dtype=torch.float32):
    layer = MoELayerMX.from_inputs(shape, inp)
    T, k = shape.T, shape.k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    y = layer(inp["x"], topk_idx=idx, topk_w=w, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    return y, idx, w, layer


def check_layer(shape, inp, y, idx, w, rows, parallel=False):
    x_bits = bf16_bits(inp["x"])
    rw, bias = inp["router_w"].cpu().numpy(), inp["e_bias"].cpu().numpy()
    ref_idx, ref_w, margin, scores = parity.oracle_route_all(shape, x_bits, rw, bias)
    rep = parity.compare_routing(shape, idx.cpu().numpy(), w.cpu().numpy(), ref_idx, ref_w, margin, scores, bias)
    assert not rep.mismatched_tokens, rep
    y_ref = parity.oracle_layer_rows(shape, inp, rows, idx.cpu().numpy(), scores, ref_idx, ref_w, margin,
                                     layer=oracle.moe_layer_mx, parallel=parallel)
    got = y.float().cpu().numpy()[rows]
    err = parity.output_errors(got, y_ref)
    print(f"{shape.name} mxfp8: {len(rows)} rows, max|err|/RMS {err['max_abs_over_rms']:.2e}, "
          f"rel L1 {err['rel_l1']:.2e}, near ties {rep.near_ties}")
    parity.assert_output_close(got, y_ref, shape.name)
    return err


@pytest.mark.parametrize("shape", SMALL_MX, ids=lambda s: s.name)
def test_small_layer_mx_every_token(shape):
    inp = make_inputs(shape, "cuda")
    y, idx, w, _ = run_forward_mx(shape, inp)
    check_layer(shape, inp, y, idx, w, np.arange(shape.T))


@pytest.mark.parametrize("shape,n_rows", [(MID, 256), (V3_DECODE, 256), (V3_PREFILL, 256), (V3_SKEWED, 256)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_full_size_layer_mx_sampled(shape, n_rows):
    """A seeded sample aimed at the last partial 128-row tile of 16 experts, the
    smallest segments and the most loaded expert (see parity.targeted_rows)."""
    inp = make_inputs(shape, "cuda")
    y, idx, w, layer = run_forward_mx(shape, inp)
    rows, info = parity.targeted_rows(shape, idx.cpu().numpy(), n_min=n_rows, seed=shape.seed)
    print(f"{shape.name} mxfp8 sample: {info}")
    check_layer(shape, inp, y, idx, w, rows, parallel=True)
    del layer


def test_mx_deterministic_and_bf16_output():
    shape = SMALL_MX[3]
    inp = make_inputs(shape, "cuda")
    y1, *_ = run_forward_mx(shape, inp)
    y2, *_ = run_forward_mx(shape, inp)
    assert torch.equal(y1, y2)
    y16, *_ = run_forward_mx(shape, inp, out_dtype=torch.bfloat16)
    assert torch.equal(y16, y1.bfloat16())


def test_mx_rejects_unsupported_shapes_and_handles_empty_batch():
    bad = TINY.with_(hidden_size=320)
    cfg = abi.MoEConfig.from_shape(bad)
    with pytest.raises(abi.MoEError) as ei:
        abi.workspace_size_mx(cfg, 4)
    assert ei.value.status == abi.MOE_ERR_UNSUPPORTED
    inp = make_inputs(TINY.with_(T=0), "cuda")
    layer = MoELayerMX.from_inputs(TINY.with_(T=0), inp)
    y = layer(inp["x"])
    torch.cuda.synchronize()
    assert y.shape == (0, TINY.H)


def test_mx_stages_compose_to_forward():
    """dispatch_mx -> gate_up_mx -> down_mx -> combine_mx through the C ABI equals
    moe_forward_mx bit for bit, and the quantised h matches the oracle's h
    (computed in float64 from the same E4M3 operands) up to its own rounding."""
    shape = SMALL_MX[4]
    inp = make_inputs(shape, "cuda")
    T, k, E, H, I, S = shape.T, shape.k, shape.E, shape.H, shape.I, shape.S
    cfg, ws, idx, w = routed(shape, inp)
    Rp, Tp = abi.mx_routed_rows(cfg, T), (T + 127) // 128 * 128
    dev = "cuda"
    u8 = lambda *s: torch.empty(s, dtype=torch.uint8, device=dev)
    i32 = lambda *s: torch.empty(s, dtype=torch.int32, device=dev)
    offsets, counts, perm_src, row_of = i32(E + 1), i32(E), i32(Rp), i32(T, k)
    xq, xsf = u8(Rp, H), u8(abi.mx_scale_bytes(Rp, H))
    xqs, xssf = u8(Tp, H), u8(abi.mx_scale_bytes(Tp, H))
    abi.moe_dispatch_mx(cfg, inp["x"], idx, offsets, counts, xq, xsf, xqs, xssf, perm_src, row_of, ws)
    layer = MoELayerMX.from_inputs(shape, inp)
    hq, hsf = u8(Rp, I), u8(abi.mx_scale_bytes(Rp, I))
    hqs, hssf = u8(Tp, S * I), u8(abi.mx_scale_bytes(Tp, S * I))
    abi.moe_experts_gate_up_mx(cfg, T, xq, xsf, xqs, xssf, offsets, counts, layer.weights, hq, hsf, hqs, hssf)
    y_perm = torch.empty((Rp + T, H), dtype=torch.float16, device=dev)
    y_sc = u8(Rp + T, abi.y_perm_scale_cols(H))
    abi.moe_experts_down_mx(cfg, T, hq, hsf, hqs, hssf, offsets, counts, perm_src, w, layer.weights, y_perm, y_sc)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    abi.moe_combine_mx(cfg, T, y_perm, y_sc, row_of, y)
    y_fwd = layer(inp["x"])
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    assert torch.equal(y, y_fwd)

    # h of one routed expert: GPU bytes and codes against the oracle's quantisation
    # of silu(xq Wg^T) * (xq Wu^T) computed in float64 from the GPU's own operands.
    e = int(torch.argmax(counts).item())
    a, n = int(offsets[e].item()), int(counts[e].item())
    assert n > 0 and a % 128 == 0
    xdeq = E4M3[xq[a:a + n].cpu().numpy()] * np.exp2(
        np.repeat(unpack_codes(xsf.cpu().numpy(), Rp, H)[a:a + n].astype(np.float64), 32, 1) - 127)
    wg = oracle.mx_quantize(bf16_bits(inp["w_gate"][e]))[2]
    wu = oracle.mx_quantize(bf16_bits(inp["w_up"][e]))[2]
    g, u = xdeq @ wg.T, xdeq @ wu.T
    h = g / (1 + np.exp(-g)) * u
    oq, oc, odeq = oracle.mx_quantize(h)
    codes = unpack_codes(hsf.cpu().numpy(), Rp, I)
    got_codes = codes[a:a + n]
    got = E4M3[hq[a:a + n].cpu().numpy()] * np.exp2(np.repeat(got_codes.astype(np.float64), 32, 1) - 127)
    assert (got_codes == oc).mean() > 0.999
    same = got == odeq
    assert same.mean() > 0.999, same.mean()
    # where they differ, by one E4M3 step at most (h near a rounding midpoint in fp32 vs float64)
    diff = np.abs(got - odeq)[~same]
    assert (diff <= 2.0 ** -3 * np.abs(odeq[~same]) + 2.0 ** -9 * np.exp2(np.repeat(oc.astype(np.float64), 32, 1) - 127)[~same]).all()
    # rows past the segment's count, up to the next multiple of 128, are zeros
    pad_end = a + (n + 127) // 128 * 128
    assert int(hq[a + n:pad_end].sum().item()) == 0


def test_mx_forward_replays_from_a_cuda_graph():
    shape = SMALL_MX[3]
    inp = make_inputs(shape, "cuda")
    layer = MoELayerMX.from_inputs(shape, inp)
    y_eager = layer(inp["x"])
    y = torch.empty_like(y_eager)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(inp["x"], y)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    y.zero_()
    with torch.cuda.graph(g):
        layer(inp["x"], y)
    g.replay()
    torch.cuda.synchronize()
    assert abi.device_status() == 0
    assert torch.equal(y, y_eager)
    del g
