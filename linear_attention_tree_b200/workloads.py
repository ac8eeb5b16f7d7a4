"""Seeded synthetic inputs for draft-tree verification through a linear-attention layer.

This module only draws random numbers and builds tree shapes; it performs none of the
method's arithmetic (no recurrence, no decay products, no solve).  Both the CUDA path
(through the bench and the GPU tests) and the CPU oracle (through the tests) consume the
`Workload` objects it returns, so it imports nothing from either side.

The five named workloads mirror the shapes of the pages' setting:

* ``config(1)``: the worked example of the Bole machine summary ("具体技术细节示例"):
  one sequence, one head, a 6-node tree with branches A (a1->a2), B (b1) and
  C (c1->c2->c3), scalar decay lambda = 0.9, fp32, d = 16; the accepted branch is C.
* ``config(2)``: gated delta rule, B=1, H=16, 16-node random tree of depth <= 6.
* ``config(3)``: gated delta rule, B=32, H=32, 64-node trees of depth <= 8, branching 1..4.
* ``config(4)``: gated delta rule, B=128, H=32, ragged trees of 8..48 nodes under a shared
  batch-wide budget of 3072 nodes (the per-batch cap on verified nodes that the Twig/Bole
  abstracts describe), depth <= 7.
* ``config(5)``: gated delta rule, B=8, H=32, 256-node trees of depth <= 10, branching 1..8,
  near-1 decay.

Outputs default to fp32 (``out_dtype``): rounding o to bf16 alone moves the largest
outputs by up to 2^-9 of their size, which exceeds 2e-2 of the output RMS.

Conventions: node indices inside a sequence are local (0..n_b-1) and topological
(``parent[i] < i``); ``-1`` is the root state S_root.  The depth of a first-level draft node
is 1.  Values destined for bf16 storage are rounded to nearest-even here, so the fp32 arrays
carried by a `Workload` are exactly the stored values.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

__all__ = [
    "Workload", "config", "synthetic", "bf16_round", "bf16_bits", "frontier_tree",
    "uniform_parent_tree", "depths_of", "acceptance_estimates", "CONFIG_NAMES",
]

CONFIG_NAMES = {
    1: "scalar-decay fp32, B=1 H=1 d=16, 6-node worked-example tree",
    2: "gdn bf16, B=1 H=16 dk=dv=128, 16-node tree depth<=6",
    3: "gdn bf16, B=32 H=32 dk=dv=128, 64-node trees depth<=8",
    4: "gdn bf16, B=128 H=32 dk=dv=128, ragged 8..48-node trees, budget 3072",
    5: "gdn bf16, B=8 H=32 dk=dv=128, 256-node trees depth<=10",
}


def _rng(seed) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of fp32 values rounded to nearest-even bf16 (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 array holding the nearest-even bf16 value of each element."""
    bits = bf16_bits(x).astype(np.uint32) << 16
    return bits.view(np.float32).reshape(np.shape(x))


def depths_of(parent: Sequence[int]) -> np.ndarray:
    """Depth of every node of one topologically ordered tree (first-level node = 1)."""
    d = np.zeros(len(parent), dtype=np.int32)
    for i, p in enumerate(parent):
        d[i] = 1 if p < 0 else d[p] + 1
    return d


def uniform_parent_tree(rng: np.random.Generator, n: int, max_depth: int) -> List[int]:
    """parent[i] uniform over {root, 0..i-1}; a draw that would exceed max_depth is redrawn."""
    parent: List[int] = []
    depth: List[int] = []
    for i in range(n):
        while True:
            p = int(rng.integers(0, i + 1)) - 1
            dp = 1 if p < 0 else depth[p] + 1
            if dp <= max_depth:
                break
        parent.append(p)
        depth.append(dp)
    return parent


def frontier_tree(seed: int, n: int, max_depth: int, fmax: int):
    """Random-frontier topological growth of an n-node tree.

    The root is expanded first; afterwards a uniformly random not-yet-expanded node of depth
    < max_depth is expanded with f ~ U{1..fmax} children (fewer if the node budget runs out).
    New nodes get the next free index, so the order is topological but not depth-sorted.
    If the frontier empties before n nodes exist, the tree is redrawn from the seed pair
    (seed, attempt).  Returns (parent list, generator positioned after the tree draws).
    """
    attempt = 0
    while True:
        rng = _rng(seed if attempt == 0 else [seed, attempt])
        parent: List[int] = []
        depth: List[int] = []
        frontier: List[int] = []          # unexpanded real nodes, in creation order
        expand = -1                       # the virtual root first
        ok = True
        while len(parent) < n:
            if expand is None:
                cand = [x for x in frontier if depth[x] < max_depth]
                if not cand:
                    ok = False
                    break
                expand = cand[int(rng.integers(0, len(cand)))]
            f = int(rng.integers(1, fmax + 1))
            dchild = 1 if expand < 0 else depth[expand] + 1
            for _ in range(min(f, n - len(parent))):
                parent.append(expand)
                depth.append(dchild)
                frontier.append(len(parent) - 1)
            if expand >= 0:
                frontier.remove(expand)
            expand = None
        if ok:
            return parent, rng
        attempt += 1


def acceptance_estimates(parent: Sequence[int], seed: int) -> np.ndarray:
    """Synthetic per-node acceptance estimates for a draft tree (float64 in (0, 1)).

    Node n of sibling rank r (0 for its parent's first child, in index order) gets
    Beta(4, 2) * 0.6**r: the first child is the drafter's top guess and its siblings are
    successively less likely, as in a top-k expansion.
    """
    rng = _rng(seed)
    seen: dict = {}
    rank = np.empty(len(parent), dtype=np.int64)
    for i, p in enumerate(parent):
        rank[i] = seen.get(int(p), 0)
        seen[int(p)] = rank[i] + 1
    return rng.beta(4.0, 2.0, size=len(parent)) * 0.6 ** rank


@dataclasses.dataclass
class Workload:
    """One batch of draft trees with all per-node, per-head inputs (host numpy arrays).

    Layouts (row-major, contiguous): q, k ``[T][Hk][dk]`` (Hk = ``qk_heads``, H unless
    several value heads share one q / k head: head h reads q / k head h // (H // Hk));
    v ``[T][H][dv]``; log_a, b ``[T][H]``; parent ``[T]`` (local index, -1 = root);
    node_offsets ``[B+1]``; S_root ``[B][H][dv][dk]`` (row v, column k);
    accepted_path ``[B][max_path]`` (root-first local indices, -1 padded).
    """
    name: str
    mode: str                      # "gdn" or "scalar"
    B: int
    H: int
    dk: int
    dv: int
    in_dtype: str                  # "f32" or "bf16"
    out_dtype: str
    parent: np.ndarray
    node_offsets: np.ndarray
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_a: np.ndarray
    b: Optional[np.ndarray]
    S_root: np.ndarray
    accepted_path: np.ndarray
    max_nodes: int
    max_path: int
    Hk: Optional[int] = None       # q / k heads; None = H

    @property
    def T(self) -> int:
        return int(self.node_offsets[-1])

    @property
    def qk_heads(self) -> int:
        return self.H if self.Hk is None else self.Hk

    def seq_parent(self, s: int) -> np.ndarray:
        return self.parent[self.node_offsets[s]:self.node_offsets[s + 1]]

    def subset(self, parent: np.ndarray, node_offsets: np.ndarray, rows: np.ndarray,
               paths: Optional[List[List[int]]] = None) -> "Workload":
        """The same sequences with only some nodes: ``rows`` are the kept nodes' rows in this
        batch, ``parent`` / ``node_offsets`` the kept trees (local, topological).  The
        per-node inputs are gathered row by row; S_root is shared.  ``paths`` (root-first,
        local to the kept trees) default to the root->last-node path of every sequence."""
        rows = np.asarray(rows, dtype=np.int64)
        B = len(node_offsets) - 1
        if B != self.B or int(node_offsets[-1]) != len(rows) or len(parent) != len(rows):
            raise ValueError("subset does not describe this batch")
        parents = [list(parent[node_offsets[s]:node_offsets[s + 1]]) for s in range(B)]
        if paths is None:
            paths = [(_path_to(p, len(p) - 1) if len(p) else []) for p in parents]
        ap = _pad_paths(paths)
        counts = np.diff(node_offsets)
        return dataclasses.replace(
            self, name=self.name + "-subset", parent=np.asarray(parent, dtype=np.int32),
            node_offsets=np.asarray(node_offsets, dtype=np.int32), q=self.q[rows],
            k=self.k[rows], v=self.v[rows], log_a=self.log_a[rows],
            b=None if self.b is None else self.b[rows], accepted_path=ap,
            max_nodes=max([1] + [int(c) for c in counts]), max_path=ap.shape[1])

    def depth_histogram(self) -> dict:
        hist: dict = {}
        for s in range(self.B):
            for d in depths_of(self.seq_parent(s)):
                hist[int(d)] = hist.get(int(d), 0) + 1
        return dict(sorted(hist.items()))


def _unit_rows(x: np.ndarray) -> np.ndarray:
    """Scale each trailing-axis vector to unit L2 norm (data preparation of q and k)."""
    x64 = x.astype(np.float64)
    return (x64 / np.linalg.norm(x64, axis=-1, keepdims=True)).astype(np.float32)


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _pad_paths(paths: List[List[int]], min_len: int = 1) -> np.ndarray:
    width = max([min_len] + [len(p) for p in paths])
    out = np.full((len(paths), width), -1, dtype=np.int32)
    for i, p in enumerate(paths):
        out[i, :len(p)] = p
    return out


def _path_to(parent: Sequence[int], n: int) -> List[int]:
    out = []
    while n >= 0:
        out.append(n)
        n = parent[n]
    return out[::-1]


def synthetic(parents: List[List[int]], H: int, dk: int, dv: int, *, seed: int,
              mode: str = "gdn", in_dtype: str = "bf16", out_dtype: Optional[str] = None,
              paths: Optional[List[List[int]]] = None, log_a_mean: float = -4.0,
              s_std: float = 0.02, name: str = "synthetic",
              max_nodes: Optional[int] = None, qk_heads: Optional[int] = None) -> Workload:
    """Workload for explicit per-sequence parent arrays with config-2 style distributions.

    q, k ~ N(0,1) normalised per (node, q / k head), ``qk_heads`` of them (default H);
    v ~ N(0,1); b = sigmoid(N(0,1));
    log_a = -softplus(N(log_a_mean, 0.5)); S_root ~ N(0, s_std).  In scalar mode the decay
    is one lambda per head (log_a = -softplus(N(log_a_mean, 0.5)) drawn per head) and b is
    absent.  ``paths`` defaults to the root->last-node path of every sequence.
    """
    rng = _rng(seed)
    B = len(parents)
    counts = [len(p) for p in parents]
    offsets = np.zeros(B + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    T = int(offsets[-1])
    Hk = H if qk_heads is None else qk_heads
    S_root = (rng.standard_normal((B, H, dv, dk)) * s_std).astype(np.float32)
    q = _unit_rows(rng.standard_normal((T, Hk, dk)).astype(np.float32))
    k = _unit_rows(rng.standard_normal((T, Hk, dk)).astype(np.float32))
    v = rng.standard_normal((T, H, dv)).astype(np.float32)
    if mode == "gdn":
        b = _sigmoid(rng.standard_normal((T, H))).astype(np.float32)
        log_a = (-_softplus(rng.normal(log_a_mean, 0.5, (T, H)))).astype(np.float32)
    else:
        b = None
        lam = (-_softplus(rng.normal(log_a_mean, 0.5, (1, H)))).astype(np.float32)
        log_a = np.repeat(lam, T, axis=0)
    if in_dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    parent = np.concatenate([np.asarray(p, dtype=np.int32) for p in parents]) if T else \
        np.zeros(0, dtype=np.int32)
    if paths is None:
        paths = [(_path_to(p, len(p) - 1) if len(p) else []) for p in parents]
    ap = _pad_paths(paths)
    return Workload(name=name, mode=mode, B=B, H=H, dk=dk, dv=dv, in_dtype=in_dtype,
                    out_dtype=out_dtype or "f32", parent=parent, node_offsets=offsets,
                    q=q, k=k, v=v, log_a=log_a, b=b, S_root=S_root, accepted_path=ap,
                    max_nodes=max([1] + counts), max_path=ap.shape[1],
                    Hk=None if qk_heads is None else qk_heads)


def _gdn_values(rng, T, H, dk, dv, B, log_a_mean):
    S_root = (rng.standard_normal((B, H, dv, dk)) * 0.02).astype(np.float32)
    q = bf16_round(_unit_rows(rng.standard_normal((T, H, dk)).astype(np.float32)))
    k = bf16_round(_unit_rows(rng.standard_normal((T, H, dk)).astype(np.float32)))
    v = bf16_round(rng.standard_normal((T, H, dv)).astype(np.float32))
    b = _sigmoid(rng.standard_normal((T, H))).astype(np.float32)
    log_a = (-_softplus(rng.normal(log_a_mean, 0.5, (T, H)))).astype(np.float32)
    return S_root, q, k, v, b, log_a


def config(idx: int, seed: int = 0) -> Workload:
    """The named workload ``idx`` (1..5) drawn with data seed ``1000*idx + seed``.

    Tree shapes use their own generators seeded with ``data_seed*10007 + sequence``.
    """
    data_seed = 1000 * idx + seed
    rng = _rng(data_seed)
    if idx == 1:
        d = 16
        parent = np.array([-1, 0, -1, -1, 3, 4], dtype=np.int32)   # a1 a2 b1 c1 c2 c3
        S_root = (rng.standard_normal((1, 1, d, d)) / 4.0).astype(np.float32)
        q = rng.standard_normal((6, 1, d)).astype(np.float32)
        k = rng.standard_normal((6, 1, d)).astype(np.float32)
        v = rng.standard_normal((6, 1, d)).astype(np.float32)
        log_a = np.full((6, 1), np.log(0.9), dtype=np.float32)
        return Workload(name="config1", mode="scalar", B=1, H=1, dk=d, dv=d, in_dtype="f32",
                        out_dtype="f32", parent=parent,
                        node_offsets=np.array([0, 6], dtype=np.int32), q=q, k=k, v=v,
                        log_a=log_a, b=None, S_root=S_root,
                        accepted_path=np.array([[3, 4, 5]], dtype=np.int32),
                        max_nodes=6, max_path=3)

    H, dk, dv = (16 if idx == 2 else 32), 128, 128
    parents: List[List[int]] = []
    paths: List[List[int]] = []
    if idx == 2:
        B = 1
        for s in range(B):
            trng = _rng(data_seed * 10007 + s)
            par = uniform_parent_tree(trng, 16, 6)
            dep = depths_of(par)
            has_child = set(p for p in par if p >= 0)
            leaves = [i for i in range(16) if i not in has_child]
            leaf = leaves[int(trng.integers(0, len(leaves)))]
            parents.append(par)
            paths.append(_path_to(par, leaf))
            assert dep.max() <= 6
    else:
        if idx == 3:
            B, counts, maxd, fmax, lmax = 32, [64] * 32, 8, 4, 8
        elif idx == 4:
            B, maxd, fmax, lmax = 128, 7, 4, 7
            counts = [int(c) for c in rng.integers(8, 49, size=B)]
            while sum(counts) > 3072:
                j = int(np.argmax(counts))          # lowest index among the largest
                counts[j] -= 1
        elif idx == 5:
            B, counts, maxd, fmax, lmax = 8, [256] * 8, 10, 8, None
        else:
            raise ValueError(f"unknown workload {idx}")
        for s in range(B):
            par, trng = frontier_tree(data_seed * 10007 + s, counts[s], maxd, fmax)
            dep = depths_of(par)
            if lmax is None:
                end = int(np.flatnonzero(dep == dep.max())[0])
            else:
                L = min(int(trng.integers(1, lmax + 1)), int(dep.max()))
                at = np.flatnonzero(dep == L)
                end = int(at[int(trng.integers(0, len(at)))])
            parents.append(par)
            paths.append(_path_to(par, end))
    counts = [len(p) for p in parents]
    offsets = np.zeros(B + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    T = int(offsets[-1])
    S_root, q, k, v, b, log_a = _gdn_values(rng, T, H, dk, dv, B, -6.0 if idx == 5 else -4.0)
    parent = np.concatenate([np.asarray(p, dtype=np.int32) for p in parents])
    ap = _pad_paths(paths)
    return Workload(name=f"config{idx}", mode="gdn", B=B, H=H, dk=dk, dv=dv, in_dtype="bf16",
                    out_dtype="f32", parent=parent, node_offsets=offsets, q=q, k=k, v=v,
                    log_a=log_a, b=b, S_root=S_root, accepted_path=ap,
                    max_nodes=max(counts), max_path=ap.shape[1])
