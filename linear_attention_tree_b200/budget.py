"""Batch-wide verification budget: how many draft nodes each sequence sends to verification.

The Twig abstract names "batch-wide verification budgeting" as a runtime optimisation, and the
Bole abstract and its machine summary (section 批级验证预算校准) describe one verification
budget for the whole batch, calibrated against the cost of the hybrid forward pass.  The pages
give no algorithm.  This module implements the plain reading, for the verify kernel alone.

* Each draft node arrives with a conditional acceptance estimate p(n): the drafter's
  probability that the target accepts the token once its parent is accepted.  Node n is
  accepted with probability P(n), the product of p over its root path.  Every accepted
  draft token lies on the accepted path, so a verified subtree is worth
  sum_{n in subtree} P(n) accepted tokens in expectation, plus the bonus token every
  sequence gets.
* A node budget is spent greedily on the largest P(n) in the batch (`select_nodes`).
  P cannot grow along a path, and ties go to the shallower node, so every prefix of that
  order is ancestor-closed in every tree.  Each tree's marginal gains therefore fall as it
  grows, and the greedy prefix is the best subtree family of its size.  With a per-tree cap,
  nodes past a tree's cap are skipped; the rest of the order is unchanged.
* A time budget uses `CostModel`, a linear model of the verify kernel's time fitted on the GPU
  (`calibrate`).  `allocate_time` takes the largest greedy prefix whose predicted time fits.
  It does this once with every tree capped at the tensor-core kernel's 64 nodes and once
  uncapped, and keeps the prefix with more expected tokens.
* `choose_budget` picks the budget itself.  It maximises expected tokens per unit of step
  time, where step time is a fixed cost the caller gives for the rest of the step plus
  ``layers`` times the predicted verify time.
* `cap_largest` is the simpler rule: shrink the largest trees one node at a time until the
  batch fits.

`prune` and `pack` turn kept node sets into the arrays `tree_verify` takes: topological local
parents, node offsets, and the global row of every kept node.
"""
from __future__ import annotations

import dataclasses
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "path_probability", "select_nodes", "cap_largest", "prune", "pack", "CostModel",
    "allocate_time", "choose_budget", "expected_tokens", "calibrate", "measure_us",
    "calibration_workload", "B200_DEFAULT",
]

TC_MAX_NODES = 64          # trees up to this size take the ≤64-node tensor-core kernel


def _depths(parent: np.ndarray) -> np.ndarray:
    d = np.zeros(len(parent), dtype=np.int64)
    for i, p in enumerate(parent):
        d[i] = 1 if p < 0 else d[p] + 1
    return d


def path_probability(parent: Sequence[int], p_accept: Sequence[float]) -> np.ndarray:
    """P(n) = product of ``p_accept`` over the root->n path of one topological tree."""
    parent = np.asarray(parent, dtype=np.int64)
    p = np.asarray(p_accept, dtype=np.float64)
    if parent.shape != p.shape:
        raise ValueError("parent and p_accept differ in length")
    if np.any((p < 0) | (p > 1)):
        raise ValueError("acceptance estimates must lie in [0, 1]")
    out = np.empty_like(p)
    for i, par in enumerate(parent):
        if par >= i or par < -1:
            raise ValueError(f"parent[{i}] = {par} is not topological")
        out[i] = p[i] if par < 0 else out[par] * p[i]
    return out


def _order(trees) -> Tuple[np.ndarray, np.ndarray, np.ndarray, List[np.ndarray]]:
    """Global greedy order over all nodes of all trees: (sequence, node, P) per position,
    plus each tree's P.  Key: P descending, then depth, sequence, node ascending."""
    probs, seqs, nodes, deps, per_tree = [], [], [], [], []
    for s, (parent, p) in enumerate(trees):
        P = path_probability(parent, p)
        per_tree.append(P)
        probs.append(P)
        deps.append(_depths(np.asarray(parent)))
        seqs.append(np.full(len(P), s, dtype=np.int64))
        nodes.append(np.arange(len(P), dtype=np.int64))
    if not probs:
        z = np.zeros(0, dtype=np.int64)
        return z, z, np.zeros(0), per_tree
    P, S, N, D = (np.concatenate(x) for x in (probs, seqs, nodes, deps))
    idx = np.lexsort((N, S, D, -P))
    return S[idx], N[idx], P[idx], per_tree


def _capped(S: np.ndarray, cap: Optional[int]) -> np.ndarray:
    """Mask of order positions whose node ranks below ``cap`` inside its own sequence."""
    if cap is None or len(S) == 0:
        return np.ones(len(S), dtype=bool)
    rank = np.empty(len(S), dtype=np.int64)
    seen: dict = {}
    for i, s in enumerate(S):
        r = seen.get(int(s), 0)
        rank[i] = r
        seen[int(s)] = r + 1
    return rank < cap


def _reserve(S: np.ndarray, n_seq: int, min_nodes: int) -> np.ndarray:
    """Mask of order positions that are among the first ``min_nodes`` of their sequence."""
    return _capped(S, min_nodes) if min_nodes > 0 else np.zeros(len(S), dtype=bool)


def _greedy_positions(S: np.ndarray, n_seq: int, budget: int, cap: Optional[int],
                      min_nodes: int) -> np.ndarray:
    """Order positions chosen: the reserved ones first, then the best others up to budget."""
    ok = _capped(S, cap)
    if cap is not None:
        min_nodes = min(min_nodes, cap)
    res = _reserve(S, n_seq, min_nodes) & ok
    n_res = int(res.sum())
    if budget < n_res:
        raise ValueError(f"budget {budget} is below the {n_res} nodes min_nodes reserves")
    rest = np.flatnonzero(ok & ~res)[:budget - n_res]
    return np.sort(np.concatenate([np.flatnonzero(res), rest]))


def _split(S, N, pos, n_seq) -> List[np.ndarray]:
    keeps: List[List[int]] = [[] for _ in range(n_seq)]
    for i in pos:
        keeps[int(S[i])].append(int(N[i]))
    return [np.sort(np.asarray(k, dtype=np.int64)) for k in keeps]


def select_nodes(trees: Sequence[Tuple[Sequence[int], Sequence[float]]], budget: int, *,
                 cap: Optional[int] = None, min_nodes: int = 0) -> List[np.ndarray]:
    """Kept node ids (ascending, ancestor-closed) of every tree under a batch node budget.

    ``trees``: one (parent, p_accept) pair per sequence, parents local and topological.
    ``cap`` bounds the nodes kept in one tree; ``min_nodes`` nodes of every tree (its best
    ones) are kept before the rest of the budget is spent.
    """
    if budget < 0:
        raise ValueError("budget must be non-negative")
    S, N, _, _ = _order(trees)
    pos = _greedy_positions(S, len(trees), budget, cap, min_nodes)
    return _split(S, N, pos, len(trees))


def expected_tokens(trees, keeps: Sequence[np.ndarray]) -> float:
    """Expected accepted tokens of one verification: per sequence 1 (the bonus token)
    plus the sum of P(n) over its kept nodes."""
    total = 0.0
    for (parent, p), keep in zip(trees, keeps):
        P = path_probability(parent, p)
        total += 1.0 + float(P[np.asarray(keep, dtype=np.int64)].sum())
    return total


def cap_largest(sizes: Sequence[int], budget: int) -> np.ndarray:
    """Shrink the largest tree (the lowest index among equals) by one node until the sizes
    sum to at most ``budget``; closed form of that loop (a water level)."""
    n = np.asarray(sizes, dtype=np.int64)
    if budget < 0 or np.any(n < 0):
        raise ValueError("sizes and budget must be non-negative")
    excess = int(n.sum()) - budget
    if excess <= 0:
        return n.copy()
    # Highest level L with sum(min(n, L)) <= budget: every tree above L ends at L or L + 1.
    lo, hi = 0, int(n.max())
    while lo < hi:
        mid = (lo + hi) // 2
        if int(np.minimum(n, mid).sum()) <= budget:
            lo = mid + 1
        else:
            hi = mid
    L = lo - 1                                   # sum(min(n, L)) <= budget < sum(min(n, L+1))
    out = np.minimum(n, L + 1)
    drop = int(out.sum()) - budget               # trees at L + 1 that still lose a node
    at_top = np.flatnonzero(out == L + 1)
    out[at_top[:drop]] = L
    return out


def prune(parent: Sequence[int], keep: Sequence[int]) -> np.ndarray:
    """Local parent array of the subtree made of ``keep`` (kept ids in ascending order keep
    the order topological).  Raises if a kept node's parent is not kept."""
    parent = np.asarray(parent, dtype=np.int64)
    keep = np.asarray(keep, dtype=np.int64)
    if len(keep) and (np.any(np.diff(keep) <= 0) or keep[0] < 0 or keep[-1] >= len(parent)):
        raise ValueError("keep must be distinct node ids in ascending order")
    pos = np.full(len(parent), -1, dtype=np.int64)
    pos[keep] = np.arange(len(keep))
    out = np.empty(len(keep), dtype=np.int32)
    for i, n in enumerate(keep):
        p = parent[n]
        if p >= 0 and pos[p] < 0:
            raise ValueError(f"node {n} is kept but its parent {p} is not")
        out[i] = -1 if p < 0 else pos[p]
    return out


def pack(parents: Sequence[Sequence[int]], keeps: Sequence[Sequence[int]]
         ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(parent, node_offsets, rows) of the pruned batch: the local parents of every kept
    subtree concatenated, their offsets, and for every kept node its row in the unpruned
    batch (the index that gathers q, k, v, log_a and b)."""
    if len(parents) != len(keeps):
        raise ValueError("one keep list per tree")
    par, rows, offs = [], [], [0]
    base = 0
    for parent, keep in zip(parents, keeps):
        keep = np.asarray(keep, dtype=np.int64)
        par.append(prune(parent, keep))
        rows.append(base + keep)
        offs.append(offs[-1] + len(keep))
        base += len(parent)
    cat = lambda xs, dt: np.concatenate(xs).astype(dt) if xs else np.zeros(0, dt)
    return cat(par, np.int32), np.asarray(offs, dtype=np.int32), cat(rows, np.int64)


@dataclasses.dataclass(frozen=True)
class CostModel:
    """Predicted verify time in µs for one batch of trees with H heads.

    Kernel class by the batch's largest tree: up to 64 nodes the ≤64-node tensor-core kernel
    (one CTA per (sequence, head), two per SM), otherwise the wide-tree kernel (64-node
    tiles, one CTA per SM).  Features: a constant, items = B·H, node-heads = T·H, and for
    the wide class tile-heads = H·Σ ceil(n_b / 64).  Coefficients are non-negative, so
    predictions grow with every node added inside a class.  Trees deeper than 8 (≤64-node
    kernel) or 16 (wide kernel) take slower paths the model does not see.
    """
    tc: Tuple[float, float, float]                 # c0, per item, per node-head
    wide: Tuple[float, float, float, float]        # c0, per item, per node-head, per tile-head

    @staticmethod
    def features(sizes: Sequence[int], H: int) -> Tuple[str, np.ndarray]:
        n = np.asarray(sizes, dtype=np.int64)
        items, nodes = len(n) * H, int(n.sum()) * H
        if len(n) == 0 or int(n.max()) <= TC_MAX_NODES:
            return "tc", np.array([1.0, items, nodes])
        tiles = int(((n + TC_MAX_NODES - 1) // TC_MAX_NODES).sum()) * H
        return "wide", np.array([1.0, items, nodes, tiles])

    def predict_us(self, sizes: Sequence[int], H: int) -> float:
        cls, x = self.features(sizes, H)
        return float(np.dot(x, self.tc if cls == "tc" else self.wide))

    @classmethod
    def fit(cls, samples: Iterable[Tuple[Sequence[int], int, float]]) -> "CostModel":
        """Non-negative least squares per kernel class over (sizes, H, µs) samples,
        weighted by 1/µs so that the relative error is what gets minimised."""
        from scipy.optimize import nnls
        rows: dict = {"tc": ([], []), "wide": ([], [])}
        for sizes, H, us in samples:
            c, x = cls.features(sizes, H)
            rows[c][0].append(x / us)
            rows[c][1].append(1.0)
        coef = {}
        for c, width in (("tc", 3), ("wide", 4)):
            X, y = rows[c]
            if len(X) < width:
                raise ValueError(f"need at least {width} samples of the {c} class, got {len(X)}")
            X = np.asarray(X)
            scale = X.max(axis=0)
            scale[scale == 0] = 1.0
            sol, _ = nnls(X / scale, np.asarray(y))
            coef[c] = tuple(float(v) for v in sol / scale)
        return cls(tc=coef["tc"], wide=coef["wide"])


# Fitted on a B200 (SM clock 1965 MHz) by `calibrate()` with H = 32, dk = dv = 128, bf16
# inputs, fp32 o and U, cold L2 before every launch: 14 batches, largest relative error of
# the fit 7%; the three bench workloads, which it did not see, were predicted within 8%.
B200_DEFAULT = CostModel(tc=(9.584, 0.03315, 0.0001474), wide=(32.77, 0.002634, 0.001159, 0.008996))


def _prefix_curve(trees, H: int, model: CostModel, cap: Optional[int], min_nodes: int,
                  layers: int, fixed_us: float):
    """For every greedy prefix (reserved nodes first): (positions, sizes, value, µs)."""
    S, N, P, _ = _order(trees)
    n_seq = len(trees)
    ok = _capped(S, cap)
    if cap is not None:
        min_nodes = min(min_nodes, cap)
    res = _reserve(S, n_seq, min_nodes) & ok
    seq_order = np.concatenate([np.flatnonzero(res), np.flatnonzero(ok & ~res)])
    sizes = np.zeros(n_seq, dtype=np.int64)
    for i in np.flatnonzero(res):
        sizes[S[i]] += 1
    value = n_seq + float(P[res].sum())
    n_res = int(res.sum())
    out = [(n_res, sizes.copy(), value, fixed_us + layers * model.predict_us(sizes, H))]
    for j in seq_order[n_res:]:
        sizes[S[j]] += 1
        value += float(P[j])
        out.append((len(out) + n_res, sizes.copy(), value,
                    fixed_us + layers * model.predict_us(sizes, H)))
    return S, N, seq_order, out


def allocate_time(trees, H: int, budget_us: float, model: CostModel = B200_DEFAULT, *,
                  min_nodes: int = 1) -> Tuple[List[np.ndarray], float, float]:
    """Kept nodes of every tree whose predicted verify time fits ``budget_us``.

    Returns (keeps, predicted µs, expected tokens).  The ``min_nodes`` reserve must fit.
    """
    best = None
    for cap in (TC_MAX_NODES, None):
        S, N, order, curve = _prefix_curve(trees, H, model, cap, min_nodes, 1, 0.0)
        for count, sizes, value, us in curve:
            if us <= budget_us and (best is None or value > best[2]):
                best = (_split(S, N, order[:count], len(trees)), us, value)
    if best is None:
        raise ValueError(f"not even the min_nodes reserve fits {budget_us} µs")
    return best


def choose_budget(trees, H: int, model: CostModel = B200_DEFAULT, *, fixed_us: float = 0.0,
                  layers: int = 1, min_nodes: int = 1) -> dict:
    """The node budget that maximises expected tokens per µs of the step.

    Step time = ``fixed_us`` (the rest of the step) + ``layers`` × predicted verify time.
    Every greedy prefix, with trees capped at 64 nodes and uncapped, is a candidate.
    Returns {"keeps", "budget", "us", "tokens", "tokens_per_us"}.
    """
    best = None
    for cap in (TC_MAX_NODES, None):
        S, N, order, curve = _prefix_curve(trees, H, model, cap, min_nodes, layers, fixed_us)
        for count, sizes, value, us in curve:
            rate = value / us if us > 0 else float("inf")
            if best is None or rate > best[0]:
                best = (rate, S, N, order[:count], count, us, value)
    rate, S, N, pos, count, us, value = best
    return {"keeps": _split(S, N, pos, len(trees)), "budget": int(count), "us": us,
            "tokens": value, "tokens_per_us": rate}


def measure_us(w, *, launches: int = 12, flush=None, kernel: str = "auto") -> float:
    """Median device time in µs of `tree_verify` on workload ``w`` (bf16 or fp32 inputs),
    timed with CUDA events around each launch on the current stream, after reading a
    256 MB buffer so that every launch starts from a cold L2."""
    import torch
    from . import binding as Lb
    from .tensors import to_device

    d = to_device(w, "cuda")
    if flush is None:
        flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    out = torch.empty((w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    U = torch.empty_like(out)
    ws = Lb.new_workspace(Lb.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes,
                                          qk_heads=w.qk_heads))
    times = []
    for it in range(launches + 2):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        Lb.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                       d["node_offsets"], d["S_root"], max_nodes=w.max_nodes, out=out, U=U,
                       workspace=ws, mode=w.mode, kernel=kernel)
        e1.record()
        if it >= 2:
            times.append((e0, e1))
    torch.cuda.synchronize()
    if Lb.get_status(ws) != 0:
        raise RuntimeError(f"device status {Lb.get_status(ws)} after timing {w.name}")
    return 1e3 * float(np.median([a.elapsed_time(b) for a, b in times]))


# (B, smallest tree, largest tree, deepest path, most children of a node)
CALIBRATION_BATCHES = (
    (16, 8, 32, 8, 4), (32, 1, 8, 8, 4), (32, 33, 64, 8, 2), (64, 8, 48, 7, 4),
    (128, 8, 48, 7, 4), (64, 48, 64, 8, 8), (192, 4, 24, 6, 4), (8, 64, 64, 8, 4),
    (2, 65, 128, 10, 4), (4, 128, 256, 10, 8), (8, 200, 256, 10, 8), (12, 65, 256, 8, 3),
    (8, 8, 130, 10, 4), (8, 256, 256, 12, 4),
)


def calibration_workload(B: int, lo: int, hi: int, max_depth: int = 8, fmax: int = 4, *,
                         H: int = 32, seed: int = 0):
    """Synthetic batch of B frontier trees (paths up to ``max_depth`` deep, up to ``fmax``
    children per node) whose sizes are uniform in [lo, hi]; bf16 q / k / v, dk = dv = 128."""
    from .workloads import frontier_tree, synthetic
    rng = np.random.Generator(np.random.PCG64([seed, B, lo, hi, max_depth, fmax]))
    sizes = [int(x) for x in rng.integers(lo, hi + 1, size=B)]
    parents = [frontier_tree(int(rng.integers(1 << 30)), n, max_depth, fmax)[0] for n in sizes]
    return synthetic(parents, H, 128, 128, seed=int(rng.integers(1 << 30)),
                     name=f"calib-B{B}-n{lo}..{hi}")


def calibrate(H: int = 32, *, seed: int = 0, launches: int = 12,
              batches: Sequence[Tuple[int, int, int, int, int]] = CALIBRATION_BATCHES
              ) -> Tuple[CostModel, List[Tuple[List[int], int, float]]]:
    """Fit a `CostModel` on this GPU from `measure_us` of `calibration_workload` batches,
    given as (B, smallest tree, largest tree, deepest path, most children).  Returns the
    model and its (sizes, H, µs) samples."""
    import torch
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    samples = []
    for B, lo, hi, depth, fmax in batches:
        w = calibration_workload(B, lo, hi, depth, fmax, H=H, seed=seed)
        us = measure_us(w, launches=launches, flush=flush)
        samples.append(([int(x) for x in np.diff(w.node_offsets)], H, us))
    return CostModel.fit(samples), samples
