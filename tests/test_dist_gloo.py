"""The multi-rank host logic of bench.py on CPU with the gloo backend (world size 2):
weights are replicated, tokens differ per rank, the step time is the max over
ranks and the throughput counts every rank's tokens."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_layer_noaux_b200.workloads import TINY


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    inp = bench.rank_inputs(TINY, rank, "cpu")
    sums = torch.tensor([inp["w_gate"].float().sum().item(), inp["router_w"].sum().item(),
                         inp["x"].float().sum().item()], dtype=torch.float64)
    gathered = [torch.zeros_like(sums) for _ in range(world)]
    dist.all_gather(gathered, sums)
    ms = bench.max_over_ranks(10.0 + rank, world)
    out[rank] = (gathered[0].tolist(), gathered[1].tolist(), ms,
                 bench.job_throughput(TINY.T, world, ms))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_replicas():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded process
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    g0, g1, ms, thr = res[0]
    assert g0[0] == g1[0] and g0[1] == g1[1]      # same weights on both ranks
    assert g0[2] != g1[2]                          # different tokens
    assert ms == 11.0 and res[1][2] == 11.0        # max over ranks, seen by all
    assert abs(thr - 2 * TINY.T / 11e-3) < 1e-6    # all ranks' tokens / slowest time


def test_reference_arm_under_torchrun_prints_once_from_rank0():
    """`bench.py --impl reference` under torchrun: rank 0 alone times the oracle and
    prints one JSON line; the other rank exits 0 at once (no process group, so no
    barrier that could time out while rank 0 works)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
