"""Spread oracle work over spawned processes (test infrastructure only):
  * the single-threaded router on disjoint row blocks (rows are independent, so
    the result is exactly that of one call over all rows);
  * the per-expert SwiGLU calls of ``moe_layer`` / ``moe_layer_mx``, one job
    per expert, results returned in job order (each expert's rows are computed
    by the same function on the same operands as in a serial run).
The arithmetic is untouched: only where each call runs changes.  (The MXFP8
layer's float64 matrix products go through numpy's BLAS, whose summation order
may depend on its thread count; workers use one BLAS thread.)"""
from __future__ import annotations

import collections
import concurrent.futures as cf
import multiprocessing as mp
import os
import types

import numpy as np

from . import build, route

_FIELDS = ("hidden_size", "n_routed_experts", "num_experts_per_tok", "n_group", "topk_group",
           "moe_intermediate_size", "n_shared_experts", "norm_topk_prob", "routed_scaling_factor")


def _plain(shape):
    return types.SimpleNamespace(**{f: getattr(shape, f) for f in _FIELDS})


def _route_block(args):
    shape, x_bits, rw, bias = args
    return route(shape, x_bits, rw, bias, want_scores=True)


def route_rows(shape, x_bits, rw, bias, workers: int = 0, min_work: float = 2e9):
    """(idx, w, margin, scores) for every row of x_bits, as oracle.route gives."""
    n = x_bits.shape[0]
    if workers <= 0:
        workers = min(32, os.cpu_count() or 1)
    shape = _plain(shape)
    if workers == 1 or n * shape.n_routed_experts * shape.hidden_size < min_work:
        return route(shape, x_bits, rw, bias, want_scores=True)
    build()
    bounds = np.linspace(0, n, workers + 1).astype(int)
    blocks = [(shape, x_bits[a:b], rw, bias) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    with cf.ProcessPoolExecutor(len(blocks), mp_context=mp.get_context("spawn")) as ex:
        parts = list(ex.map(_route_block, blocks))
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(4))


def _one_blas_thread():
    try:
        import threadpoolctl
        threadpoolctl.threadpool_limits(1)
    except Exception:  # the limit only avoids oversubscription
        pass


class ExpertRunner:
    """``run_experts`` for ``oracle.moe_layer``: evaluates fn(*job) for each job in
    a pool of spawned processes, yielding results in job order with at most
    2 x workers jobs queued (so only that many experts' weights are in memory)."""

    def __init__(self, workers: int = 0):
        self.workers = workers if workers > 0 else max(1, min(16, os.cpu_count() or 1))

    def __call__(self, fn, jobs):
        build()
        with cf.ProcessPoolExecutor(self.workers, mp_context=mp.get_context("spawn"),
                                    initializer=_one_blas_thread) as ex:
            pending = collections.deque()
            for job in jobs:
                pending.append(ex.submit(fn, *job))
                if len(pending) >= 2 * self.workers:
                    yield pending.popleft().result()
            while pending:
                yield pending.popleft().result()
