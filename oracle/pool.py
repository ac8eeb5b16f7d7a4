"""The float64 oracle over a whole named workload, spread over the host's cores.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests and the CPU-baseline leg
of ``bench.py`` use it; the library never does.

The oracle walks every node's path one token at a time, so a full workload of thousands of
nodes x 32 heads takes minutes on one core.  Here it runs in a pool of worker processes
(started with ``spawn``, never forked from a process that has touched the GPU), each
limited to one BLAS thread, over (sequence, head) items.  Workers rebuild the workload from
its seed instead of receiving it, and return plain arrays; nothing here does any arithmetic
of the method beyond calling ``oracle.oracle``.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

_CACHE = {}


def _init():
    from threadpoolctl import threadpool_limits
    _CACHE["limit"] = threadpool_limits(limits=1)


def _workload(spec):
    if spec not in _CACHE:
        from linear_attention_tree_b200 import workloads as W
        kind, idx, seed = spec
        assert kind == "config"
        _CACHE[spec] = W.config(idx, seed)
    return _CACHE[spec]


def _work(job):
    from oracle import oracle as O
    spec, items = job
    w = _workload(spec)
    out = []
    for s, h in items:
        lo, hi = int(w.node_offsets[s]), int(w.node_offsets[s + 1])
        o = np.empty((hi - lo, w.dv))
        u = np.empty((hi - lo, w.dv))
        for n in range(hi - lo):
            o[n], u[n] = O.verify_node(w, s, n, h)
        S = O.commit_sequence(w, s, h, w.accepted_path[s])
        out.append((s, h, o, u, S))
    return out


def workers() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_config(idx: int, seed: int = 0, n_workers: int | None = None, pool=None):
    """(w, o, U, S_new) of named workload ``idx`` in float64: every node, head and state.
    ``pool``: a started `start_pool` to reuse (its start-up is then not paid again)."""
    from linear_attention_tree_b200 import workloads as W
    w = W.config(idx, seed)
    spec = ("config", idx, seed)
    items = [(s, h) for s in range(w.B) for h in range(w.H)]
    n_workers = n_workers or workers()
    chunk = max(1, len(items) // (4 * n_workers))
    jobs = [(spec, items[i:i + chunk]) for i in range(0, len(items), chunk)]
    o = np.full((w.T, w.H, w.dv), np.nan)
    U = np.full((w.T, w.H, w.dv), np.nan)
    S_new = np.full((w.B, w.H, w.dv, w.dk), np.nan)
    own = pool is None
    if own:
        pool = start_pool(n_workers)
    try:
        for res in pool.imap_unordered(_work, jobs):
            for s, h, oo, uu, S in res:
                lo, hi = int(w.node_offsets[s]), int(w.node_offsets[s + 1])
                o[lo:hi, h] = oo
                U[lo:hi, h] = uu
                S_new[s, h] = S
    finally:
        if own:
            pool.close()
            pool.join()
    return w, o, U, S_new


def start_pool(n_workers: int | None = None):
    """A spawn pool of one-BLAS-thread workers, warmed up (imports done)."""
    pool = mp.get_context("spawn").Pool(n_workers or workers(), initializer=_init)
    pool.map(_ping, range(4 * (n_workers or workers())))
    return pool


def _ping(_):
    import oracle.oracle  # noqa: F401  (import cost paid before anything is timed)
    return 0


def _rows_work(job):
    from oracle import oracle as O
    spec, rows = job
    w = _workload(spec)
    done = 0
    for row in rows:
        s = int(np.searchsorted(w.node_offsets, row, side="right") - 1)
        n = int(row - w.node_offsets[s])
        for h in range(w.H):
            O.verify_node(w, s, n, h)
        if row == int(w.node_offsets[s + 1]) - 1:
            for h in range(w.H):
                O.commit_sequence(w, s, h, w.accepted_path[s])
        done += 1
    return done


def oracle_rows(idx: int, seed: int, rows, pool) -> int:
    """The oracle on global node rows of named workload ``idx`` (every head of each row,
    plus the commit of every sequence whose last node is among them), spread over ``pool``.
    Returns the number of rows done; the results are discarded (a timing sample)."""
    rows = [int(r) for r in rows]
    n = len(pool._pool) if hasattr(pool, "_pool") else workers()
    chunk = max(1, len(rows) // (2 * n))
    jobs = [(("config", idx, seed), rows[i:i + chunk]) for i in range(0, len(rows), chunk)]
    return sum(pool.map(_rows_work, jobs))
