"""Auxiliary-loss-free bias update ("The Evolving Transformer · 07", § 06: the
per-expert bias is nudged down when overloaded and up when underloaded).

CPU: the oracle step pinned by a hand-worked case, by numpy float32 arithmetic
for the fp32 state, and by the method's purpose (repeated steps even out the
load).  GPU: moe_bias_update matches the oracle bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_noaux_b200.workloads import MID, TINY, V3_SKEWED, MoEShape, bf16_bits, make_inputs


def test_hand_worked_step():
    # 4 tokens x 2 slots over 4 experts: loads (5, 1, 2, 0), mean 8 / 4 = 2.
    # Expert 0 is overloaded (down), 1 and 3 underloaded (up), 2 exactly at the mean.
    idx = np.array([[0, 1], [0, 2], [0, 0], [2, 0]])
    bias, load = oracle.bias_update(idx, 4, np.array([0.5, -0.25, 0.125, 0.0], np.float32), 0.25)
    assert load.tolist() == [5, 1, 2, 0]
    assert bias.tolist() == [0.25, 0.0, 0.125, 0.25]


def test_fp32_state_matches_numpy_float32():
    rng = np.random.default_rng(0)
    E, T, k = 16, 50, 3
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    b0 = (rng.standard_normal(E) * 10).astype(np.float32)
    gamma = np.float32(1e-3)
    bias, load = oracle.bias_update(idx, E, b0, float(gamma))
    counts = np.bincount(idx.reshape(-1), minlength=E)
    sign = np.sign(T * k - counts * E).astype(np.float32)  # +1 under, -1 over, 0 at the mean
    np.testing.assert_array_equal(load, counts)
    np.testing.assert_array_equal(bias, b0 + sign * gamma)  # float32 adds
    # A step far below half an ulp leaves the bias unchanged (fp32 rounding).
    same, _ = oracle.bias_update(idx, E, np.full(E, 1.0, np.float32), 1e-9)
    assert (same == 1.0).all()


def test_repeated_steps_even_out_the_load():
    # Skewed start (Zipf bias: max / mean load ~7); router weights wide enough that
    # tokens disagree on their experts; routing by the oracle.  60 steps of size
    # 0.02 must bring the max / mean load down by more than half — the purpose of
    # the update.  A wrong sign would make it worse.
    shape = V3_SKEWED.with_(T=256, hidden_size=64, n_routed_experts=32, n_group=4, topk_group=2,
                            num_experts_per_tok=4, moe_intermediate_size=64)
    inp = make_inputs(shape, "cpu", weight_std=0.3)
    x, rw = bf16_bits(inp["x"]), inp["router_w"].numpy()
    bias = inp["e_bias"].numpy().copy()
    imbalance = []
    for _ in range(60):
        idx, _, _ = oracle.route(shape, x, rw, bias)
        bias, load = oracle.bias_update(idx, shape.E, bias, 0.02)
        imbalance.append(load.max() / load.mean())
    assert imbalance[0] > 5 and imbalance[-1] < 0.5 * imbalance[0], imbalance


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [TINY, MID, V3_SKEWED.with_(T=2048)], ids=lambda s: s.name)
def test_gpu_bias_update_matches_oracle(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sparse_moe_layer_noaux_b200 import abi
    inp = make_inputs(shape, "cuda")
    cfg = abi.MoEConfig.from_shape(shape)
    ws = torch.empty(abi.workspace_size(cfg, shape.T), dtype=torch.uint8, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    abi.moe_route(cfg, inp["x"], inp["router_w"], inp["e_bias"], idx, w, ws)
    bias = inp["e_bias"].clone()
    load = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    abi.moe_bias_update(cfg, idx, bias, 1e-3, load)
    torch.cuda.synchronize()
    ref_bias, ref_load = oracle.bias_update(idx.cpu().numpy(), shape.E, inp["e_bias"].cpu().numpy(), 1e-3)
    np.testing.assert_array_equal(load.cpu().numpy(), ref_load)
    np.testing.assert_array_equal(bias.cpu().numpy().view(np.uint32), ref_bias.view(np.uint32))


@pytest.mark.gpu
def test_gpu_balancing_loop_evens_out_the_skewed_v3_load():
    """The V3 skewed routing (Zipf bias: one expert takes every token, max / mean 32)
    through repeated moe_route + moe_bias_update on the GPU: the load evens out —
    the purpose of the update (the CPU oracle loop shows the same at a small shape)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bench
    shape = V3_SKEWED.with_(T=4096)
    inp = make_inputs(shape, "cuda")
    res = bench.bias_balancing(shape, inp, steps=60, gamma=0.05)
    tr = res["max_over_mean_every_10_steps"]
    print(f"v3_skewed T=4096 max/mean load every 10 steps (gamma 0.05): {tr}")
    assert tr[0] > 20 and tr[-1] < 0.25 * tr[0], tr
