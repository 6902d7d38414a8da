"""The expert-parallel layer's exchange on CPU ranks (gloo): MoELayerEP.forward with
its all-to-alls over a real process group, the library calls replaced by the
oracle-backed stand-in of tests/ep_cpu_kernels.py.  Each rank holds E/world of
the routed experts and its own tokens; every rank's output must equal the float64
oracle's single-device layer on its tokens, and the rows a rank receives must be
exactly the other ranks' rows for its experts."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_layer_noaux_b200.workloads import MoEShape, bf16_bits, make_inputs

SHAPE = MoEShape("ep", T=24, hidden_size=256, n_routed_experts=16, n_group=4, topk_group=2,
                 num_experts_per_tok=4, moe_intermediate_size=128, n_shared_experts=1,
                 routed_scaling_factor=2.5, norm_topk_prob=True, seed=41)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_tokens(shape, rank):
    T = shape.T + 5 * rank  # ranks bring different batch sizes (one may be empty)
    if rank == 3:
        T = 0
    g = torch.Generator().manual_seed(1000 + rank)
    return torch.randn((T, shape.H), generator=g).to(torch.bfloat16)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from sparse_moe_layer_noaux_b200.ep import MoELayerEP, expert_block
    from tests import ep_cpu_kernels
    import oracle
    shape = SHAPE
    inp = make_inputs(shape, "cpu")            # same seed: the same weights on every rank
    layer = MoELayerEP(shape, world, rank, inp["router_w"], inp["e_bias"],
                       expert_block(inp["w_gate"], world, rank), expert_block(inp["w_up"], world, rank),
                       expert_block(inp["w_down"], world, rank), inp["ws_gate"], inp["ws_up"], inp["ws_down"],
                       _kernels=ep_cpu_kernels)
    x = _rank_tokens(shape, rank)
    y = layer(x)
    # The same batch through the exchange phases by hand, to look at what arrived.
    st = layer.route_and_pack(x)
    recv = torch.empty_like(st.counts)
    dist.all_to_all_single(recv, st.counts)
    layer.plan(st, recv)
    # The oracle's single-device layer on this rank's tokens (all experts).
    fetch = oracle.in_memory_experts(bf16_bits(inp["w_gate"]), bf16_bits(inp["w_up"]), bf16_bits(inp["w_down"]))
    shared = tuple(bf16_bits(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    y_ref, idx_ref, _, _ = oracle.moe_layer(shape, bf16_bits(x), inp["router_w"].numpy(), inp["e_bias"].numpy(),
                                            fetch, shared)
    out[rank] = {"y": y.numpy(), "y_ref": y_ref, "idx": st.idx.numpy(), "idx_ref": idx_ref,
                 "recv_counts": recv.numpy(), "send_splits": st.send_splits, "recv_splits": st.recv_splits,
                 "recv_offsets": st.recv_offsets.numpy()}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_matches_the_single_device_layer(world, oracle_lib):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    El = SHAPE.E // world
    gsz = SHAPE.E // SHAPE.n_group
    for r in range(world):
        d = res[r]
        assert (d["idx"] == d["idx_ref"]).all()
        if d["y"].size:
            rms = np.sqrt(np.mean(d["y_ref"] ** 2))
            err = np.abs(d["y"] - d["y_ref"]).max() / rms
            assert err <= 2e-2, (r, err)   # fp16 storage of the expert outputs
        # Rows sent to rank d are this rank's rows for d's experts; rank d receives
        # exactly what every source sent it, counted per (source, local expert).
        for dst in range(world):
            sent_counts = np.bincount(d["idx"].reshape(-1), minlength=SHAPE.E)[dst * El:(dst + 1) * El]
            assert d["send_splits"][dst] == sent_counts.sum()
            np.testing.assert_array_equal(res[dst]["recv_counts"].reshape(world, El)[r], sent_counts)
            assert res[dst]["recv_splits"][r] == sent_counts.sum()
        np.testing.assert_array_equal(d["recv_offsets"], np.concatenate([[0], np.cumsum(d["recv_counts"])]))
        # Groups do not straddle ranks here, so a token's rows reach at most topk_group ranks.
        if El % gsz == 0 and d["idx"].size:
            ranks_per_token = [len({int(e) // El for e in row}) for row in d["idx"]]
            assert max(ranks_per_token) <= SHAPE.topk_group
