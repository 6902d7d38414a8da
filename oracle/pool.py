"""Run the single-threaded oracle router on disjoint row blocks in spawned
processes (test infrastructure only).  Rows are independent, so the result is
exactly that of one call over all rows; the arithmetic is untouched."""
from __future__ import annotations

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
