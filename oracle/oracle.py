"""Plain float64 CPU oracle for draft-tree verification through a linear-attention layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or runs this module;
only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.
It shares no code with the CUDA path: the only thing both sides consume is the seeded
`Workload` from ``linear_attention_tree_b200.workloads``, which holds no method arithmetic.

What it computes, and where the pages state it:

* The recurrence.  Scalar decay ``S_t = lambda S_{t-1} + k_t v_t^T`` with output read from
  the state (Bole machine summary, "核心公式", first formula); the gated delta rule
  ``S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T`` of Gated DeltaNet (named by the
  TreeWY abstract, which prints no formula; this is the textbook form of that rule, with
  a_t = exp(log_a_t) and write strength b_t).  This module stores the state as
  ``[dv][dk]`` (the transpose of the summary's ``k v^T`` orientation), so the output read is
  ``o = S q`` and the scalar update is ``S <- lambda S + v k^T``; the outputs are identical
  to the summary's ``o = S^T q`` with ``S <- lambda S + k v^T``.
* Tree semantics.  A draft node's state is the state the sequential recurrence reaches
  after consuming the tokens on its root-to-node path (Twig/Bole abstracts: recurrent layers
  carry parent-dependent states; worked example "具体技术细节示例": ``S_a2``, ``S_c3``).
  Every node is computed here by walking that path from ``S_root`` step by step: there is
  no closed form, no factorisation and no triangular solve in this file.
* The output of node n is read from the post-update state, ``o_n = S_n q_n``.
* Pseudo-values.  The TreeWY abstract replaces per-node snapshots by a pseudo-value
  matrix without printing its formula.  Reading taken: ``u_n`` is the rank-1 factor by
  which node n's own step changes its parent's decayed state,
  ``S_n = a_n S_parent + u_n k_n^T``, i.e. ``u_n = b_n (v_n - a_n S_parent k_n)`` for the
  gated delta rule and ``u_n = v_n`` for scalar decay.
* Commit.  The accepted state is the state at the end of the accepted root-first path
  (worked example: only ``S_c3`` is rebuilt; the Twig abstract rebuilds one state after
  sampling), again by walking the recurrence from ``S_root``.

Each function below is pinned by tests in ``tests/test_oracle_pins.py`` against facts the
pages or the mathematics fix (the printed worked example, the page's closed form, sequential
decoding on chains, b = 0, the delta-rule identity, sibling independence, brute-force
branch-by-branch traversal with snapshots, losslessness of the factorisation).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "path_to", "tree_meta", "step", "walk", "node_states", "verify_node", "tree_verify",
    "tree_commit", "commit_sequence",
]


def path_to(parent: Sequence[int], n: int) -> List[int]:
    """Root-first list of the nodes on the path root -> n (n included).

    Tree semantics of the worked example: branch C is c1 -> c2 -> c3, all under S_root.
    """
    out = []
    while n >= 0:
        out.append(int(n))
        n = int(parent[n])
    out.reverse()
    return out


def tree_meta(parent: Sequence[int], log_a: np.ndarray):
    """Depth, strict-ancestor set and cumulative path log-decay of every node of one tree.

    depth(n) = number of tokens on the root->n path (a first-level node has depth 1, as the
    worked example's lambda^2 on S_root for the depth-2 node a2 implies);
    anc(n) = path minus n; cl[n, h] = sum of log_a over the path (fp64).
    ``log_a`` is ``[n_nodes][H]``.
    """
    n_nodes = len(parent)
    depth = np.zeros(n_nodes, dtype=np.int64)
    anc: List[List[int]] = []
    cl = np.zeros((n_nodes,) + np.shape(log_a)[1:], dtype=np.float64)
    for n in range(n_nodes):
        p = path_to(parent, n)
        depth[n] = len(p)
        anc.append(p[:-1])
        for j in p:
            cl[n] += np.asarray(log_a[j], dtype=np.float64)
    return depth, anc, cl


def step(S: np.ndarray, k: np.ndarray, v: np.ndarray, log_a: float, b, mode: str):
    """One token of the recurrence on a ``[dv][dk]`` fp64 state.

    gdn:    S <- a S (I - b k k^T) + b v k^T        (Gated DeltaNet)
    scalar: S <- lambda S + v k^T                   (summary's first formula, transposed)
    with a = lambda = exp(log_a).
    """
    a = np.exp(np.float64(log_a))
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if mode == "scalar":
        return a * S + np.outer(v, k)
    b = np.float64(b)
    dk = k.shape[0]
    return a * (S @ (np.eye(dk) - b * np.outer(k, k))) + b * np.outer(v, k)


def walk(S_root: np.ndarray, path: Sequence[int], k, v, log_a, b, mode: str):
    """Apply the recurrence along ``path`` (root-first) starting at S_root.

    ``k, v`` are ``[n][d]`` rows of one head, ``log_a, b`` are ``[n]``.  Returns the final
    state and the state before the final token (S_root for a one-token path).
    """
    S = np.asarray(S_root, dtype=np.float64).copy()
    S_prev = S
    for j in path:
        S_prev = S
        S = step(S, k[j], v[j], log_a[j], None if b is None else b[j], mode)
    return S, S_prev


def _head(w, s: int, h: int):
    """Inputs of sequence s, value head h.  When several value heads share one q / k head
    (``w.qk_heads`` < H, as in models whose value heads outnumber their key heads), head h
    reads q / k head h // (H // qk_heads)."""
    lo, hi = int(w.node_offsets[s]), int(w.node_offsets[s + 1])
    f64 = lambda x: np.asarray(x, dtype=np.float64)
    kh = h // (w.H // getattr(w, "qk_heads", w.H))
    return (f64(w.q[lo:hi, kh]), f64(w.k[lo:hi, kh]), f64(w.v[lo:hi, h]),
            f64(w.log_a[lo:hi, h]), None if w.b is None else f64(w.b[lo:hi, h]),
            f64(w.S_root[s, h]), w.parent[lo:hi])


def node_states(w, s: int, h: int) -> np.ndarray:
    """Full post-update state ``S_n`` of every node of sequence s, head h: ``[n][dv][dk]``.

    Used by the tests to check the oracle against the worked example and the closed form.
    """
    q, k, v, la, b, S0, parent = _head(w, s, h)
    return np.stack([walk(S0, path_to(parent, n), k, v, la, b, w.mode)[0]
                     for n in range(len(parent))]) if len(parent) else \
        np.zeros((0, w.dv, w.dk))


def verify_node(w, s: int, n: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """(o_n, u_n) in fp64 for local node n of sequence s, head h, by walking its path."""
    q, k, v, la, b, S0, parent = _head(w, s, h)
    S, S_prev = walk(S0, path_to(parent, n), k, v, la, b, w.mode)
    o = S @ q[n]
    if w.mode == "scalar":
        u = v[n].copy()
    else:
        a = np.exp(la[n])
        u = b[n] * (v[n] - a * (S_prev @ k[n]))
    return o, u


def tree_verify(w, seqs=None, heads=None) -> Tuple[np.ndarray, np.ndarray]:
    """Outputs o ``[T][H][dv]`` and pseudo-values U ``[T][H][dv]`` (fp64) of every node.

    ``seqs`` / ``heads`` restrict the work to a subset (other rows stay NaN).
    """
    o = np.full((w.T, w.H, w.dv), np.nan)
    U = np.full((w.T, w.H, w.dv), np.nan)
    for s in (range(w.B) if seqs is None else seqs):
        lo = int(w.node_offsets[s])
        for h in (range(w.H) if heads is None else heads):
            for n in range(int(w.node_offsets[s + 1]) - lo):
                o[lo + n, h], U[lo + n, h] = verify_node(w, s, n, h)
    return o, U


def commit_sequence(w, s: int, h: int, path: Sequence[int]) -> np.ndarray:
    """Accepted state of sequence s, head h: the recurrence walked along ``path``."""
    q, k, v, la, b, S0, parent = _head(w, s, h)
    path = [int(j) for j in path if j >= 0]
    return walk(S0, path, k, v, la, b, w.mode)[0]


def tree_commit(w, paths=None, seqs=None, heads=None) -> np.ndarray:
    """S_new ``[B][H][dv][dk]`` (fp64) for every sequence's accepted root-first path.

    ``paths`` defaults to ``w.accepted_path``; -1 entries are padding.  An empty path
    returns S_root.
    """
    paths = w.accepted_path if paths is None else paths
    out = np.full((w.B, w.H, w.dv, w.dk), np.nan)
    for s in (range(w.B) if seqs is None else seqs):
        for h in (range(w.H) if heads is None else heads):
            out[s, h] = commit_sequence(w, s, h, paths[s])
    return out
