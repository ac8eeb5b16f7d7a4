"""Pins of the float64 oracle against facts the pages and the mathematics fix.

Every check here compares the oracle's path walk with something that is not the walk
itself: the worked example printed on the Bole summary page, that page's lambda-weighted
closed form (exponents as its example fixes them), plain sequential decoding, special
cases with closed forms (b = 0, the delta-rule identity, one token), a brute-force
branch-by-branch traversal with explicit per-node snapshots, and the losslessness of the
pseudo-value factorisation (TreeWY abstract: a tree-structured WY form whose pseudo-values
come from one triangular solve), solved here with a library triangular solver.  ``test_planted_mistakes``
shows that plausible slips in the oracle (a dropped term, a wrong index, a transposed
operand, the pre-update state) each fail at least one pin.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.linalg

from linear_attention_tree_b200 import workloads as W
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def _parse_golden():
    names, parent_name, states, accepted = [], {}, {}, []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if not line:
                continue
            if line[0] == "node":
                names.append(line[1])
                parent_name[line[1]] = line[2]
            elif line[0] == "state":
                states[line[1]] = [(t.split(":")[0], int(t.split(":")[1])) for t in line[2:]]
            elif line[0] == "accepted":
                accepted = line[1:]
    idx = {n: i for i, n in enumerate(names)}
    parent = [-1 if parent_name[n] == "root" else idx[parent_name[n]] for n in names]
    return names, idx, parent, states, accepted


# ----------------------------------------------------------------------------------- P1
def pin_worked_example():
    """Bole summary, worked example: S_a2 and S_c3 as printed; commit of branch C = S_c3."""
    names, idx, parent, states, accepted = _parse_golden()
    w = W.config(1)
    assert list(w.parent) == parent, "config 1 must be the page's example tree"
    lam = np.exp(np.float64(w.log_a[0, 0]))
    S = O.node_states(w, 0, 0)
    k = w.k[:, 0].astype(np.float64)
    v = w.v[:, 0].astype(np.float64)
    S0 = w.S_root[0, 0].astype(np.float64)
    for name, terms in states.items():
        want = np.zeros_like(S0)
        for term, power in terms:
            want += lam ** power * (S0 if term == "S_root" else np.outer(v[idx[term]], k[idx[term]]))
        got = S[idx[name]]
        assert np.max(np.abs(got - want)) <= 1e-13 * np.max(np.abs(want)), name
    path = [idx[n] for n in accepted]
    assert path == list(w.accepted_path[0])
    S_new = O.tree_commit(w)[0, 0]
    np.testing.assert_allclose(S_new, S[idx[accepted[-1]]], rtol=0, atol=1e-13)


def test_p1_worked_example():
    pin_worked_example()


def test_worked_example_outputs_read_state():
    """o_n = S_n q_n (post-update state) for every node of the worked example."""
    w = W.config(1)
    S = O.node_states(w, 0, 0)
    o, U = O.tree_verify(w)
    for n in range(6):
        np.testing.assert_allclose(o[n, 0], S[n] @ w.q[n, 0].astype(np.float64),
                                   rtol=1e-13, atol=1e-13)
        np.testing.assert_array_equal(U[n, 0], w.v[n, 0].astype(np.float64))


# ----------------------------------------------------------------------------------- P2
def pin_closed_form_scalar(seed=7):
    """Scalar decay: S_n = lambda^d S_root + sum_j lambda^(d-j) v_pj k_pj^T over the path.

    Bole summary, "核心公式" second formula, with the exponent direction and the S_root
    term fixed by its own worked example (lambda^2 S_root for the depth-2 node).
    """
    rng = np.random.default_rng(seed)
    for trial in range(4):
        n = int(rng.integers(1, 12))
        par = W.uniform_parent_tree(rng, n, 5)
        w = W.synthetic([par], H=2, dk=5, dv=4, seed=seed * 100 + trial, mode="scalar",
                        in_dtype="f32")
        for h in range(2):
            lam = np.exp(np.float64(w.log_a[0, h]))
            S = O.node_states(w, 0, h)
            dep = W.depths_of(par)
            for node in range(n):
                chain = [node]
                while par[chain[-1]] >= 0:
                    chain.append(par[chain[-1]])
                chain.reverse()
                d = dep[node]
                want = lam ** d * w.S_root[0, h].astype(np.float64)
                for j, t in enumerate(chain, start=1):
                    want = want + lam ** (d - j) * np.outer(w.v[t, h].astype(np.float64),
                                                            w.k[t, h].astype(np.float64))
                np.testing.assert_allclose(S[node], want, rtol=1e-12, atol=1e-12)


def test_p2_closed_form_scalar():
    pin_closed_form_scalar()


# ----------------------------------------------------------------------------------- P3
def _sequential_decode(S0, q, k, v, log_a, b):
    """Textbook left-to-right gated-delta decoding in its error-correcting form.

    S_t = a_t S_{t-1} + b_t (v_t - a_t S_{t-1} k_t) k_t^T,  o_t = S_t q_t.
    """
    S = S0.copy()
    outs = []
    for t in range(q.shape[0]):
        a = np.exp(log_a[t])
        pred = a * (S @ k[t])
        S = a * S + b[t] * np.outer(v[t] - pred, k[t])
        outs.append(S @ q[t])
    return np.array(outs), S


def pin_chain_is_sequential(seed=3):
    """A chain-shaped tree (parent[i] = i-1) verifies exactly like sequential decoding."""
    n = 9
    w = W.synthetic([[i - 1 for i in range(n)]], H=3, dk=8, dv=6, seed=seed, in_dtype="f32",
                    log_a_mean=-1.0, s_std=0.3)
    o, _ = O.tree_verify(w)
    S_new = O.tree_commit(w)
    for h in range(3):
        f = lambda x: x[:, h].astype(np.float64)
        outs, S = _sequential_decode(w.S_root[0, h].astype(np.float64), f(w.q), f(w.k),
                                     f(w.v), f(w.log_a), f(w.b))
        np.testing.assert_allclose(o[:, h], outs, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S_new[0, h], S, rtol=1e-12, atol=1e-12)


def test_p3_chain_is_sequential():
    pin_chain_is_sequential()


# ----------------------------------------------------------------------------------- P4
def pin_b_zero(seed=11):
    """b = 0: the state only decays, S_n = exp(cl_n) S_root, u_n = 0, o_n = exp(cl_n) S_root q_n."""
    rng = np.random.default_rng(seed)
    par = W.uniform_parent_tree(rng, 10, 4)
    w = W.synthetic([par], H=2, dk=6, dv=5, seed=seed, in_dtype="f32", log_a_mean=-1.0)
    w.b[:] = 0.0
    o, U = O.tree_verify(w)
    S = [O.node_states(w, 0, h) for h in range(2)]
    for h in range(2):
        for n in range(10):
            chain = O.path_to(par, n)
            gamma = np.exp(sum(np.float64(w.log_a[j, h]) for j in chain))
            S0 = w.S_root[0, h].astype(np.float64)
            np.testing.assert_allclose(S[h][n], gamma * S0, rtol=1e-12, atol=1e-15)
            np.testing.assert_array_equal(U[n, h], 0.0)
            np.testing.assert_allclose(o[n, h], gamma * S0 @ w.q[n, h], rtol=1e-12, atol=1e-15)


def test_p4_b_zero():
    pin_b_zero()


# ----------------------------------------------------------------------------------- P5
def pin_delta_rule(seed=5):
    """a = 1, b = 1, unit k: the delta rule stores v under key k, so S_n k_n = v_n,
    and a node whose query equals its key reads back its own value."""
    rng = np.random.default_rng(seed)
    par = W.uniform_parent_tree(rng, 8, 4)
    w = W.synthetic([par], H=1, dk=7, dv=7, seed=seed, in_dtype="f32", s_std=0.5)
    w.log_a[:] = 0.0
    w.b[:] = 1.0
    # keys with an exactly unit norm in binary: four entries of +-1/2
    for n in range(8):
        pos = rng.choice(7, size=4, replace=False)
        w.k[n, 0] = 0.0
        w.k[n, 0, pos] = rng.choice([-0.5, 0.5], size=4)
    w.q[:] = w.k
    S = O.node_states(w, 0, 0)
    o, _ = O.tree_verify(w)
    for n in range(8):
        np.testing.assert_allclose(S[n] @ w.k[n, 0], w.v[n, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o[n, 0], w.v[n, 0], rtol=1e-12, atol=1e-12)


def test_p5_delta_rule():
    pin_delta_rule()


# ----------------------------------------------------------------------------------- P6
def pin_sibling_independence(seed=8):
    """Inputs of nodes off a node's root path never change that node's o or u (bitwise)."""
    rng = np.random.default_rng(seed)
    par = W.uniform_parent_tree(rng, 12, 4)
    w = W.synthetic([par], H=2, dk=6, dv=6, seed=seed, in_dtype="f32")
    o, U = O.tree_verify(w)
    for n in range(12):
        on_path = set(O.path_to(par, n))
        w2 = W.synthetic([par], H=2, dk=6, dv=6, seed=seed, in_dtype="f32")
        for j in range(12):
            if j not in on_path:
                w2.q[j] += 1.0
                w2.k[j] *= -0.5
                w2.v[j] += 3.0
                w2.log_a[j] -= 0.7
                w2.b[j] = 0.1
        o2, U2 = O.tree_verify(w2)
        np.testing.assert_array_equal(o2[n], o[n])
        np.testing.assert_array_equal(U2[n], U[n])


def test_p6_sibling_independence():
    pin_sibling_independence()


# ----------------------------------------------------------------------------------- P7
def _dfs_snapshots(parent, S0, q, k, v, log_a, b):
    """Branch-by-branch traversal with one explicit state snapshot per node.

    The per-node-snapshot baseline of the Twig/Bole abstracts: a depth-first walk keeps the
    parent's full state and derives each child's state from it, one token at a time.
    Returns per node (state, output, rank-one factor of its own step).
    """
    children = {}
    for i, p in enumerate(parent):
        children.setdefault(p, []).append(i)
    res = {}
    stack = [(-1, S0)]
    while stack:
        node, S = stack.pop()
        for c in children.get(node, []):
            a = np.exp(log_a[c])
            decayed = a * S
            # delta rule on the decayed state: replace what key k_c reads by v_c, with rate b_c
            Sc = decayed - b[c] * np.outer(decayed @ k[c] - v[c], k[c])
            kk = float(k[c] @ k[c])
            u = (Sc - decayed) @ k[c] / kk
            res[c] = (Sc, Sc @ q[c], u)
            stack.append((c, Sc))
    return res


def _all_trees(n):
    return itertools.product(*[range(-1, i) for i in range(n)])


def pin_bruteforce(max_n=7, every=1):
    rng = np.random.default_rng(17)
    d = 3
    base = W.synthetic([[-1] * max_n], H=1, dk=d, dv=d, seed=17, in_dtype="f32",
                       log_a_mean=-1.0, s_std=0.5)
    f = lambda x: x[:, 0].astype(np.float64)
    count = 0
    for n in range(1, max_n + 1):
        for t, par in enumerate(_all_trees(n)):
            if t % every:
                continue
            w = W.synthetic([list(par)], H=1, dk=d, dv=d, seed=17, in_dtype="f32",
                            log_a_mean=-1.0, s_std=0.5)
            for name in ("q", "k", "v", "log_a", "b"):
                getattr(w, name)[:] = getattr(base, name)[:n]
            w.S_root[:] = base.S_root
            ref = _dfs_snapshots(list(par), base.S_root[0, 0].astype(np.float64), f(w.q), f(w.k),
                                 f(w.v), f(w.log_a), f(w.b))
            S = O.node_states(w, 0, 0)
            o, U = O.tree_verify(w)
            for i in range(n):
                np.testing.assert_allclose(S[i], ref[i][0], rtol=1e-11, atol=1e-12)
                np.testing.assert_allclose(o[i, 0], ref[i][1], rtol=1e-11, atol=1e-12)
                np.testing.assert_allclose(U[i, 0], ref[i][2], rtol=1e-9, atol=1e-10)
            count += 1
    return count


def test_p7_bruteforce_exhaustive():
    """Every tree with up to 6 nodes (873 trees) and every 7th tree with 7 nodes."""
    assert pin_bruteforce(max_n=6) == 873
    pin_bruteforce_seven()


def pin_bruteforce_seven():
    rng = np.random.default_rng(19)
    d = 3
    trees = list(_all_trees(7))
    base = W.synthetic([[-1] * 7], H=1, dk=d, dv=d, seed=19, in_dtype="f32", log_a_mean=-1.0,
                       s_std=0.5)
    f = lambda x: x[:, 0].astype(np.float64)
    for par in trees[::7]:
        w = W.synthetic([list(par)], H=1, dk=d, dv=d, seed=19, in_dtype="f32",
                        log_a_mean=-1.0, s_std=0.5)
        for name in ("q", "k", "v", "log_a", "b"):
            getattr(w, name)[:] = getattr(base, name)
        w.S_root[:] = base.S_root
        ref = _dfs_snapshots(list(par), base.S_root[0, 0].astype(np.float64), f(w.q), f(w.k),
                             f(w.v), f(w.log_a), f(w.b))
        o, U = O.tree_verify(w)
        for i in range(7):
            np.testing.assert_allclose(o[i, 0], ref[i][1], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(U[i, 0], ref[i][2], rtol=1e-9, atol=1e-10)


# ----------------------------------------------------------------------------------- P8
def pin_lossless_wy(seed=23, mode="gdn"):
    """The pseudo-values losslessly encode every node state (Twig/Bole abstracts), and one
    unit-lower-triangular solve over the tree reproduces them (TreeWY abstract).

    With gamma_n = exp(sum of log_a on the root->n path):
      S_n = gamma_n S_root + sum_{i on path(n)} (gamma_n / gamma_i) u_i k_i^T
    and (I + L) U = R with L[n,i] = b_n (gamma_n/gamma_i) k_n.k_i for strict ancestors i,
    R_n = b_n (v_n - gamma_n S_root k_n); scalar decay has U = V.
    """
    rng = np.random.default_rng(seed)
    par = W.uniform_parent_tree(rng, 20, 6)
    w = W.synthetic([par], H=2, dk=8, dv=6, seed=seed, in_dtype="f32", mode=mode,
                    log_a_mean=-1.0, s_std=0.3)
    o, U = O.tree_verify(w)
    for h in range(2):
        S = O.node_states(w, 0, h)
        la = w.log_a[:, h].astype(np.float64)
        k = w.k[:, h].astype(np.float64)
        v = w.v[:, h].astype(np.float64)
        S0 = w.S_root[0, h].astype(np.float64)
        chains = [O.path_to(par, n) for n in range(20)]
        lg = np.array([sum(la[j] for j in c) for c in chains])
        for n in range(20):
            rec = np.exp(lg[n]) * S0
            for i in chains[n]:
                rec = rec + np.exp(lg[n] - lg[i]) * np.outer(U[i, h], k[i])
            assert np.max(np.abs(rec - S[n])) <= 1e-11 * max(1.0, np.max(np.abs(S[n])))
        if mode == "gdn":
            b = w.b[:, h].astype(np.float64)
            L = np.zeros((20, 20))
            R = np.zeros((20, w.dv))
            for n in range(20):
                for i in chains[n][:-1]:
                    L[n, i] = b[n] * np.exp(lg[n] - lg[i]) * (k[n] @ k[i])
                R[n] = b[n] * (v[n] - np.exp(lg[n]) * (S0 @ k[n]))
            Usolve = scipy.linalg.solve_triangular(np.eye(20) + L, R, lower=True,
                                                   unit_diagonal=True)
            np.testing.assert_allclose(U[:, h], Usolve, rtol=1e-10, atol=1e-12)
        else:
            np.testing.assert_array_equal(U[:, h], v)


def test_p8_lossless_wy():
    pin_lossless_wy(mode="gdn")
    pin_lossless_wy(mode="scalar", seed=29)


# ----------------------------------------------------------------------------------- P9
def pin_relabel(seed=31):
    """A topological relabelling of the tree permutes o and U exactly."""
    rng = np.random.default_rng(seed)
    n = 14
    par = W.uniform_parent_tree(rng, n, 5)
    w = W.synthetic([par], H=2, dk=6, dv=5, seed=seed, in_dtype="f32")
    o, U = O.tree_verify(w)
    # relabel: breadth-first order (still topological, usually different)
    dep = W.depths_of(par)
    order = sorted(range(n), key=lambda i: (dep[i], -i))
    new_of = {old: new for new, old in enumerate(order)}
    par2 = [(-1 if par[old] < 0 else new_of[par[old]]) for old in order]
    assert all(p < i for i, p in enumerate(par2))
    w2 = W.synthetic([par2], H=2, dk=6, dv=5, seed=seed, in_dtype="f32")
    for name in ("q", "k", "v", "log_a", "b"):
        getattr(w2, name)[:] = getattr(w, name)[order]
    w2.S_root[:] = w.S_root
    o2, U2 = O.tree_verify(w2)
    np.testing.assert_array_equal(o2, o[order])
    np.testing.assert_array_equal(U2, U[order])


def test_p9_relabel():
    pin_relabel()


# ---------------------------------------------------------------------------------- P10
def pin_single_token(seed=37):
    """One draft token: S_1 = a S_root (I - b k k^T) + b v k^T, o = S_1 q (one recurrence
    step written with an explicit identity matrix; scalar: lambda S_root + v k^T)."""
    for mode in ("gdn", "scalar"):
        w = W.synthetic([[-1], [-1]], H=2, dk=5, dv=4, seed=seed, in_dtype="f32", mode=mode)
        o, U = O.tree_verify(w)
        S_new = O.tree_commit(w)
        for s in range(2):
            for h in range(2):
                k = w.k[s, h].astype(np.float64)
                v = w.v[s, h].astype(np.float64)
                q = w.q[s, h].astype(np.float64)
                a = np.exp(np.float64(w.log_a[s, h]))
                S0 = w.S_root[s, h].astype(np.float64)
                if mode == "gdn":
                    bb = np.float64(w.b[s, h])
                    S1 = a * S0 @ (np.eye(5) - bb * np.outer(k, k)) + bb * np.outer(v, k)
                else:
                    S1 = a * S0 + np.outer(v, k)
                np.testing.assert_allclose(o[s, h], S1 @ q, rtol=1e-13, atol=1e-14)
                np.testing.assert_allclose(S_new[s, h], S1, rtol=1e-13, atol=1e-14)


def test_p10_single_token():
    pin_single_token()


# ------------------------------------------------------------------------- metadata, commit
def _hadamard16():
    h = np.array([[1.0]])
    for _ in range(4):
        h = np.block([[h, h], [h, -h]])
    return h / 4.0          # orthonormal rows, every entry +-1/4 (exact in fp32)


def pin_orthonormal_keys(seed=43):
    """Gated delta rule with mutually orthonormal keys along every path (general a, b).

    The factors (I - b_i k_i k_i^T) of orthonormal keys commute and each k_i passes through
    the others unchanged, so the recurrence closes to
        S_n = gamma_n S_root (I - sum_i b_i k_i k_i^T) + sum_i exp(cl_n - cl_i) b_i v_i k_i^T,
        u_n = b_n (v_n - gamma_n S_root k_n)        (the tree system's L vanishes: U = R),
    sums over path(n), cl the path sum of log_a and gamma = exp(cl).
    """
    rng = np.random.default_rng(seed)
    for trial in range(4):
        n = int(rng.integers(2, 15))
        par = W.uniform_parent_tree(rng, n, 6)
        w = W.synthetic([par], H=2, dk=16, dv=5, seed=seed * 100 + trial, in_dtype="f32",
                        log_a_mean=-1.0)
        for h in range(2):
            rows = rng.permutation(16)[:n]
            signs = rng.choice([-1.0, 1.0], size=n)
            w.k[:, h, :] = (_hadamard16()[rows] * signs[:, None]).astype(np.float32)
        dk = 16
        for h in range(2):
            S0 = w.S_root[0, h].astype(np.float64)
            k, v = w.k[:, h].astype(np.float64), w.v[:, h].astype(np.float64)
            la, b = w.log_a[:, h].astype(np.float64), w.b[:, h].astype(np.float64)
            S = O.node_states(w, 0, h)
            for node in range(n):
                path = []
                x = node
                while x >= 0:
                    path.append(x)
                    x = par[x]
                path.reverse()
                cl = np.cumsum(la[path])
                proj = np.eye(dk) - sum(b[i] * np.outer(k[i], k[i]) for i in path)
                want = np.exp(cl[-1]) * S0 @ proj
                for j, i in enumerate(path):
                    want = want + np.exp(cl[-1] - cl[j]) * b[i] * np.outer(v[i], k[i])
                np.testing.assert_allclose(S[node], want, rtol=1e-10, atol=1e-12)
                o, u = O.verify_node(w, 0, node, h)
                np.testing.assert_allclose(u, b[node] * (v[node] - np.exp(cl[-1]) * S0 @ k[node]),
                                           rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(o, want @ w.q[node, h].astype(np.float64),
                                           rtol=1e-10, atol=1e-12)


def test_p11_orthonormal_keys():
    pin_orthonormal_keys()


def test_meta_worked_example():
    w = W.config(1)
    depth, anc, cl = O.tree_meta(w.parent, w.log_a)
    assert list(depth) == [1, 2, 1, 1, 2, 3]
    assert anc == [[], [0], [], [], [3], [3, 4]]
    np.testing.assert_allclose(cl[:, 0], np.array(depth) * np.float64(w.log_a[0, 0]), rtol=1e-15)


def pin_meta_varied_decay():
    """Cumulative log-decay with a different log_a on every node.

    (a) Hand-summed values on a 6-node tree (root children 0 and 2, chain 0 -> 1 -> 3,
    2 -> 4, 3 -> 5), one head: cl_n is the sum of log_a over the root -> n path, n
    included (the worked example's depth-2 node carries lambda^2: one factor per path
    token).  (b) With k = 0 in scalar mode the walk only decays, so the walked state is
    exp(cl_n) S_root: the metadata must agree with the recurrence on random trees with
    random per-node, per-head decays.
    """
    parent = [-1, 0, -1, 1, 2, 3]
    log_a = np.array([[-0.5], [-0.25], [-2.0], [-0.125], [-1.0], [-0.0625]])
    depth, anc, cl = O.tree_meta(parent, log_a)
    assert list(depth) == [1, 2, 1, 3, 2, 4]
    assert anc == [[], [0], [], [0, 1], [2], [0, 1, 3]]
    want = np.array([-0.5, -0.75, -2.0, -0.875, -3.0, -0.9375])
    np.testing.assert_array_equal(cl[:, 0], want)       # exact: dyadic values
    rng = np.random.default_rng(43)
    for trial in range(3):
        par = W.uniform_parent_tree(rng, 12, 6)
        w = W.synthetic([par], H=3, dk=4, dv=3, seed=43 + trial, mode="scalar", in_dtype="f32")
        w.log_a = rng.uniform(-1.5, -0.01, size=w.log_a.shape).astype(np.float32)
        w.k[:] = 0.0
        _, _, cl = O.tree_meta(w.seq_parent(0), w.log_a)
        for h in range(w.H):
            S = O.node_states(w, 0, h)
            ratio = S / w.S_root[0, h].astype(np.float64)
            np.testing.assert_allclose(ratio, np.exp(cl[:, h])[:, None, None] *
                                       np.ones_like(ratio), rtol=1e-13)


def test_meta_varied_decay():
    pin_meta_varied_decay()


def _mut_meta_depth_times_own(parent, log_a):
    depth, anc, _ = _orig_tree_meta(parent, log_a)
    return depth, anc, depth[:, None] * np.asarray(log_a, dtype=np.float64)


def _mut_meta_parent_excluded(parent, log_a):
    depth, anc, cl = _orig_tree_meta(parent, log_a)
    return depth, anc, cl - np.asarray(log_a, dtype=np.float64)


def _mut_meta_first_node_decay(parent, log_a):
    depth, anc, _ = _orig_tree_meta(parent, log_a)
    la = np.asarray(log_a, dtype=np.float64)
    return depth, anc, np.array([la[([*a, n])[0]] * d for n, (a, d) in
                                 enumerate(zip(anc, depth))])


_orig_tree_meta = O.tree_meta


@pytest.mark.parametrize("mutant", [_mut_meta_depth_times_own, _mut_meta_parent_excluded,
                                    _mut_meta_first_node_decay],
                         ids=lambda m: m.__name__)
def test_meta_pin_catches_planted_mistakes(monkeypatch, mutant):
    """A per-node mix-up of log_a along the path fails the varied-decay pin."""
    monkeypatch.setattr(O, "tree_meta", mutant)
    with pytest.raises(AssertionError):
        pin_meta_varied_decay()


def test_grouped_qk_heads_equal_repeated_qk():
    """Value heads that share a q / k head give exactly what separate heads holding copies
    of that q / k give (the ungrouped oracle, on an independently expanded workload)."""
    rng = np.random.default_rng(51)
    pars = [W.uniform_parent_tree(rng, 9, 4), W.uniform_parent_tree(rng, 6, 3)]
    w = W.synthetic(pars, H=6, dk=8, dv=5, seed=51, qk_heads=2, in_dtype="f32")
    assert w.q.shape == (w.T, 2, 8) and w.qk_heads == 2
    e = W.synthetic(pars, H=6, dk=8, dv=5, seed=51, in_dtype="f32")
    for name in ("v", "log_a", "b", "S_root", "parent", "node_offsets", "accepted_path"):
        setattr(e, name, getattr(w, name))
    e.q = np.repeat(w.q, 3, axis=1)     # value heads 0-2 share q / k head 0, 3-5 head 1
    e.k = np.repeat(w.k, 3, axis=1)
    o, U = O.tree_verify(w)
    o_e, U_e = O.tree_verify(e)
    np.testing.assert_array_equal(o, o_e)
    np.testing.assert_array_equal(U, U_e)
    np.testing.assert_array_equal(O.tree_commit(w), O.tree_commit(e))


def test_commit_empty_path_is_root_and_matches_node_states():
    rng = np.random.default_rng(41)
    par = W.uniform_parent_tree(rng, 10, 4)
    w = W.synthetic([par, par], H=2, dk=4, dv=3, seed=41, in_dtype="f32")
    paths = np.array([[-1, -1, -1, -1], O.path_to(par, 9) + [-1] * (4 - len(O.path_to(par, 9)))],
                     dtype=np.int32)
    S_new = O.tree_commit(w, paths=paths)
    np.testing.assert_array_equal(S_new[0], w.S_root[0].astype(np.float64))
    for h in range(2):
        np.testing.assert_allclose(S_new[1, h], O.node_states(w, 1, h)[9], rtol=0, atol=0)


# ------------------------------------------------------------------------ planted mistakes
_PINS = [pin_worked_example, pin_closed_form_scalar, pin_chain_is_sequential, pin_b_zero,
         pin_delta_rule, lambda: pin_bruteforce(max_n=4), pin_lossless_wy, pin_single_token,
         pin_orthonormal_keys]

_orig_step = O.step
_orig_verify_node = O.verify_node
_orig_path_to = O.path_to


def _mut_step_transposed(S, k, v, log_a, b, mode):
    a = np.exp(np.float64(log_a))
    if mode == "scalar":
        return a * S + np.outer(k, v)
    return _orig_step(S, v, k, log_a, b, mode)


def _mut_step_no_decay_on_update(S, k, v, log_a, b, mode):
    a = np.exp(np.float64(log_a))
    if mode == "scalar":
        return a * (S + np.outer(v, k))
    bb = np.float64(b)
    return a * (S - bb * np.outer(S @ k, k) + bb * np.outer(v, k))


def _mut_step_drop_b_on_v(S, k, v, log_a, b, mode):
    if mode == "scalar":
        return _orig_step(S, k, v, log_a, b, mode)
    a = np.exp(np.float64(log_a))
    bb = np.float64(b)
    return a * (S @ (np.eye(len(k)) - bb * np.outer(k, k))) + np.outer(v, k)


def _mut_step_scalar_decay_off(S, k, v, log_a, b, mode):
    if mode == "scalar":
        return S + np.outer(v, k)
    return _orig_step(S, k, v, log_a, b, mode)


def _mut_path_reversed(parent, n):
    return _orig_path_to(parent, n)[::-1]


def _mut_path_skips_root_child(parent, n):
    p = _orig_path_to(parent, n)
    return p[1:] if len(p) > 1 else p


def _mut_verify_pre_update(w, s, n, h):
    q, k, v, la, b, S0, parent = O._head(w, s, h)
    S, S_prev = O.walk(S0, O.path_to(parent, n), k, v, la, b, w.mode)
    _, u = _orig_verify_node(w, s, n, h)
    return S_prev @ q[n], u


def _mut_verify_u_without_decay(w, s, n, h):
    q, k, v, la, b, S0, parent = O._head(w, s, h)
    o, u = _orig_verify_node(w, s, n, h)
    if w.mode == "scalar":
        return o, u
    S, S_prev = O.walk(S0, O.path_to(parent, n), k, v, la, b, w.mode)
    return o, b[n] * (v[n] - S_prev @ k[n])


_MUTANTS = [("step", _mut_step_transposed), ("step", _mut_step_no_decay_on_update),
            ("step", _mut_step_drop_b_on_v), ("step", _mut_step_scalar_decay_off),
            ("path_to", _mut_path_reversed), ("path_to", _mut_path_skips_root_child),
            ("verify_node", _mut_verify_pre_update),
            ("verify_node", _mut_verify_u_without_decay)]


@pytest.mark.parametrize("attr,mutant", _MUTANTS, ids=[m.__name__ for _, m in _MUTANTS])
def test_planted_mistakes(monkeypatch, attr, mutant):
    """Each planted slip in the oracle is caught by at least one pin."""
    monkeypatch.setattr(O, attr, mutant)
    caught = 0
    for pin in _PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught >= 1, f"no pin catches {mutant.__name__}"
