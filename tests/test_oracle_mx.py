"""Pins of the MXFP8 oracle ("DeepSeek-V3 notes" (knlb.dev), § fp8: fine-grained
block-wise E4M3 quantisation, scales from each block's maximum).

Each pin checks the oracle against something outside it: the E4M3 format as a
bit-level definition decoded here, torch's float8_e4m3fn conversion (a library
routine), hand-worked scale codes, the rounding error bound of a 3-bit
significand, and a one-expert layer recomputed with torch float64 and torch's
float8 cast."""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_noaux_b200.workloads import TINY, bf16_bits, make_inputs


def decode_e4m3(byte: int) -> float:
    """E4M3 from its fields: sign, 4-bit exponent (bias 7), 3-bit mantissa."""
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m / 8.0 * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


FINITE = [b for b in range(256) if not np.isnan(decode_e4m3(b))]


def test_grid_is_fixed_and_encodes_back():
    vals = np.array([decode_e4m3(b) for b in FINITE])
    assert len(FINITE) == 254 and vals.max() == 448.0 and np.min(vals[vals > 0]) == 2.0 ** -9
    np.testing.assert_array_equal(oracle.e4m3_round(vals), vals)
    bits = oracle.e4m3_bits(vals)
    # +0 and -0 both encode; every other value has a unique pattern
    for b, v, got in zip(FINITE, vals, bits):
        assert decode_e4m3(int(got)) == v and (v == 0 or got == b)


def test_midpoints_round_to_even_significand():
    pos = sorted({decode_e4m3(b) for b in FINITE if decode_e4m3(b) >= 0})
    by_value = {decode_e4m3(b): b for b in FINITE if not (b & 0x80)}
    mids = np.array([(a + b) / 2 for a, b in zip(pos[:-1], pos[1:])])
    got = oracle.e4m3_round(mids)
    for lo, hi, g in zip(pos[:-1], pos[1:], got):
        want = lo if (by_value[lo] & 1) == 0 else hi
        assert g == want, (lo, hi, g)
    # just off the midpoint goes to the nearer neighbour
    np.testing.assert_array_equal(oracle.e4m3_round(np.nextafter(mids, 0)), np.array(pos[:-1]))
    np.testing.assert_array_equal(oracle.e4m3_round(np.nextafter(mids, 1e9)), np.array(pos[1:]))


def test_rounding_matches_torch_float8_cast():
    # torch's float32 -> float8_e4m3fn conversion is the library reference; inputs are
    # float32 values so that no double rounding enters on either side.
    g = np.random.default_rng(7)
    mag = np.exp2(g.uniform(-12, np.log2(448.0), 200_000)).astype(np.float32)
    v = (mag * g.choice([-1, 1], mag.size)).astype(np.float32)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(v.astype(np.float64)), want)


@pytest.mark.parametrize("amax,code", [
    (448.0, 127), (np.nextafter(448.0, 1e9), 128), (449.0, 128), (1.0, 119), (448.0 * 2.0 ** -10, 117),
    (448.0 * 2.0 ** -10 * 1.0001, 118), (0.0, 0), (3.0, 120), (224.0, 126), (224.5, 127)])
def test_scale_code_hand_worked(amax, code):
    # code = 127 + e, e the smallest integer with amax <= 448 * 2^e
    assert oracle.mx_scale_code(amax) == code


def test_scale_is_the_smallest_power_of_two_that_fits():
    g = np.random.default_rng(3)
    a = g.standard_normal((500, 32)) * np.exp2(g.uniform(-20, 20, (500, 1)))
    q, codes, deq = oracle.mx_quantize(a)
    amax = np.abs(a).max(axis=1)
    scale = np.exp2(codes[:, 0].astype(np.float64) - 127)
    assert (amax / scale <= 448.0).all() and (amax / (scale / 2) > 448.0).all()
    np.testing.assert_array_equal(deq, q * scale[:, None])
    assert np.abs(q).max() <= 448.0


def test_quantisation_error_bound():
    # RNE with a 3-bit significand: |x - deq| <= 2^-4 |x| in the normal range,
    # and <= half the subnormal spacing 2^-10 (times the scale) below it.
    g = np.random.default_rng(5)
    a = g.standard_normal((64, 256)) * np.exp2(g.uniform(-3, 3, (64, 256)))
    q, codes, deq = oracle.mx_quantize(a)
    scale = np.repeat(np.exp2(codes.astype(np.float64) - 127), 32, axis=1)
    err = np.abs(a - deq)
    normal = np.abs(a) / scale >= 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(a[normal])).all()
    assert (err[~normal] <= 2.0 ** -10 * scale[~normal]).all()
    assert normal.mean() > 0.9


def test_bf16_bits_are_widened_exactly():
    g = np.random.default_rng(1)
    x = torch.from_numpy(g.standard_normal((4, 64)).astype(np.float32)).bfloat16()
    bits = bf16_bits(x)
    np.testing.assert_array_equal(oracle.widen_bf16(bits), x.double().numpy())
    np.testing.assert_array_equal(oracle.mx_quantize(bits)[2], oracle.mx_quantize(x.double().numpy())[2])


def _torch_mx(a: torch.Tensor) -> torch.Tensor:
    """Block-32 MX quantise-dequantise with torch ops: amax per block, the power-of-two
    scale from torch.frexp, the element rounding by torch's float8_e4m3fn cast."""
    r, K = a.shape
    b = a.reshape(r, K // 32, 32)
    amax = b.abs().amax(dim=2, keepdim=True)
    m, p = torch.frexp(amax)
    e = torch.where(m <= 0.875, p - 9, p - 8)
    scale = torch.where(amax > 0, torch.exp2(e.double()), torch.full_like(amax, 2.0 ** -127))
    q = (b / scale).float().to(torch.float8_e4m3fn).double()
    return (q * scale).reshape(r, K)


def test_one_expert_layer_closed_form():
    # E = 1, one group, top-1, no shared expert, normalised: the layer is
    # scale * down(Q(silu(gate Q(x)) * up Q(x))) with every Q the block-32 MX
    # quantisation — recomputed here with torch float64 and torch's float8 cast.
    shape = TINY.with_(n_routed_experts=1, n_group=1, topk_group=1, num_experts_per_tok=1,
                       n_shared_experts=0, T=9)
    inp = make_inputs(shape, "cpu", weight_std=0.05)
    xb = bf16_bits(inp["x"])
    wg, wu, wd = (bf16_bits(inp[n][0]) for n in ("w_gate", "w_up", "w_down"))
    y, idx, w, _ = oracle.moe_layer_mx(shape, xb, inp["router_w"].numpy(), inp["e_bias"].numpy(),
                                       lambda e: (wg, wu, wd), None)
    assert (idx == 0).all() and np.allclose(w, shape.routed_scaling_factor)
    X = _torch_mx(inp["x"].double())
    G = X @ _torch_mx(inp["w_gate"][0].double()).T
    U = X @ _torch_mx(inp["w_up"][0].double()).T
    h = _torch_mx(torch.nn.functional.silu(G) * U)
    ref = shape.routed_scaling_factor * (h @ _torch_mx(inp["w_down"][0].double()).T)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12 * float(ref.abs().max()))


def test_mx_layer_close_to_unquantised_layer():
    # Quantisation moves the output by about the E4M3 relative precision, not more:
    # a wrong scale (off by a power of two) or a missing dequantisation would not.
    shape = TINY
    inp = make_inputs(shape, "cpu")
    xb = bf16_bits(inp["x"])
    fetch = oracle.in_memory_experts(bf16_bits(inp["w_gate"]), bf16_bits(inp["w_up"]), bf16_bits(inp["w_down"]))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    args = (shape, xb, inp["router_w"].numpy(), inp["e_bias"].numpy(), fetch, shared)
    y, *_ = oracle.moe_layer(*args)
    yq, *_ = oracle.moe_layer_mx(*args)
    rel = np.abs(yq - y).sum() / np.abs(y).sum()
    assert 0.005 < rel < 0.08, rel
