"""Parity of the CUDA path with the float64 oracle, element by element.

Bars: max|err| <= 1e-4 * RMS(oracle tensor) for fp32 inputs, <= 2e-2 * RMS for bf16
inputs, separately for o, U and S_new.  Every one of the five named workloads is compared
in full, every node, head and state: 1 and 2 directly, 3-5 against the oracle spread over
the host's cores (``oracle/pool.py``), with both kernels and in the launch
configuration the benchmark times.  Smaller trees of every shape class (ragged, empty,
deep branched, combs, chains) are compared in full as well.
"""
import numpy as np
import pytest

from linear_attention_tree_b200 import workloads as W
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run
from oracle.pool import oracle_config

_FULL = {}


def _oracle_full(idx):
    if idx not in _FULL:
        _FULL[idx] = oracle_config(idx)
    return _FULL[idx]

pytestmark = pytest.mark.gpu


def _full_check(w, kernel="auto", out_dtype=None):
    res, _ = run(w, kernel=kernel, out_dtype=out_dtype)
    o, U = O.tree_verify(w)
    S_new = O.tree_commit(w)
    tol = TOL[w.in_dtype]
    assert_close(res["o"], o, tol, "o")
    if w.mode == "gdn":
        assert_close(res["U"], U, tol, "U")
    else:
        np.testing.assert_array_equal(res["U"], U)     # scalar decay: U = V exactly
    assert_close(res["S_new"], S_new, tol, "S_new")


def _sampled_check(w, kernel="auto", n_nodes=160, n_states=24, seed=0):
    res, _ = run(w, kernel=kernel)
    rng = np.random.default_rng(seed)
    tol = TOL[w.in_dtype]
    seqs = rng.integers(0, w.B, n_nodes)
    got_o, want_o, got_u, want_u = [], [], [], []
    for s in seqs:
        n = int(rng.integers(0, w.node_offsets[s + 1] - w.node_offsets[s]))
        h = int(rng.integers(0, w.H))
        o, u = O.verify_node(w, int(s), n, h)
        row = int(w.node_offsets[s]) + n
        got_o.append(res["o"][row, h]); want_o.append(o)
        got_u.append(res["U"][row, h]); want_u.append(u)
    assert_close(np.array(got_o), np.array(want_o), tol, "o (sampled)")
    assert_close(np.array(got_u), np.array(want_u), tol, "U (sampled)")
    got_s, want_s = [], []
    for _ in range(n_states):
        s, h = int(rng.integers(0, w.B)), int(rng.integers(0, w.H))
        want_s.append(O.commit_sequence(w, s, h, w.accepted_path[s]))
        got_s.append(res["S_new"][s, h])
    assert_close(np.array(got_s), np.array(want_s), tol, "S_new (sampled)")


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_config1_worked_example(kernel):
    _full_check(W.config(1), kernel)


@pytest.mark.parametrize("kernel", ["auto", "simt", "tc"])
def test_config2(kernel):
    _full_check(W.config(2), kernel)


@pytest.mark.parametrize("kernel", ["auto", "simt"])
@pytest.mark.parametrize("idx", [3, 4, 5])
def test_full_size_every_output(idx, kernel):
    """Whole workloads 3-5 against the float64 oracle: every o and U row of every node and
    head, every accepted state."""
    w, o, U, S_new = _oracle_full(idx)
    res, _ = run(w, kernel=kernel)
    tol = TOL[w.in_dtype]
    assert_close(res["o"], o, tol, f"o config {idx} {kernel}")
    assert_close(res["U"], U, tol, f"U config {idx} {kernel}")
    assert_close(res["S_new"], S_new, tol, f"S_new config {idx} {kernel}")


@pytest.mark.parametrize("idx", [3, 4, 5])
def test_full_size_sampled(idx):
    """Default kernel choice, as the benchmark runs it (tensor cores up to 64 nodes)."""
    _sampled_check(W.config(idx))


def test_tc_matches_simt_config3():
    """The two kernels agree at half the oracle bar over the whole workload.

    The tensor-core kernel rounds S_root to bf16 for the state products and rounds the
    operands of its second (tf32) product to nearest; together that moves o by up to about
    0.6% of its RMS, while the CUDA-core kernel stays at fp32 rounding.
    """
    w = W.config(3)
    a, _ = run(w, kernel="tc")
    b, _ = run(w, kernel="simt")
    for key in ("o", "U", "S_new"):
        assert_close(a[key], b[key], 1e-2, key + " tc vs simt")


@pytest.mark.parametrize("idx", [3, 4, 5])
def test_full_size_sampled_simt(idx):
    _sampled_check(W.config(idx), kernel="simt", n_nodes=60, n_states=8, seed=1)


@pytest.mark.parametrize("idx,seed", [(2, 1), (2, 2), (2, 3), (3, 1), (3, 2), (3, 3), (4, 1),
                                      (4, 2), (5, 1)])
def test_extra_seeds(idx, seed):
    _sampled_check(W.config(idx, seed=seed), n_nodes=60, n_states=8, seed=seed)


def _ragged(seed, counts, max_depth=8, fmax=4):
    pars = []
    for i, c in enumerate(counts):
        par, _ = W.frontier_tree(seed * 100 + i, c, max_depth, fmax) if c else ([], None)
        pars.append(par)
    return pars


def test_node_counts_past_the_tensor_core_tile():
    """65 and 255 nodes per tree (the CUDA-core kernel, picked automatically), with a 1-node
    tree beside them, compared in full."""
    w = W.synthetic(_ragged(9, [65, 1, 255], max_depth=10, fmax=6), H=2, dk=128, dv=128,
                    seed=321, name="ragged-wide")
    _full_check(w, "auto")


@pytest.mark.parametrize("kernel", ["tc", "simt"])
@pytest.mark.parametrize("counts", [[64, 37, 9], [1, 63, 64, 2], [5, 0, 17], [64] * 5])
def test_ragged_small_full(kernel, counts):
    """Several sequences, ragged node counts (incl. an empty tree), compared in full."""
    w = W.synthetic(_ragged(len(counts), counts), H=3, dk=128, dv=128,
                    seed=sum(counts), name="ragged")
    _full_check(w, kernel)


@pytest.mark.parametrize("mode", ["gdn", "scalar"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 48), (64, 128)])
def test_dims_f32(mode, dk, dv):
    pars = _ragged(dk + dv, [12, 30])
    w = W.synthetic(pars, H=2, dk=dk, dv=dv, seed=dk * dv, mode=mode, in_dtype="f32",
                    log_a_mean=-2.0, s_std=0.1)
    _full_check(w, "simt")


@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_scalar_bf16(kernel):
    pars = _ragged(5, [40, 64])
    w = W.synthetic(pars, H=2, dk=128, dv=128, seed=5, mode="scalar", log_a_mean=-3.0)
    _full_check(w, kernel)


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_bf16_output(kernel):
    """o stored as bf16: the bar widens by the half-ulp of bf16 at each reference value."""
    pars = _ragged(6, [33, 20, 64])
    w = W.synthetic(pars, H=2, dk=128, dv=128, seed=6, out_dtype="bf16")
    res, _ = run(w, kernel=kernel)
    o, _ = O.tree_verify(w)
    rms = np.sqrt(np.mean(o ** 2))
    bound = TOL["bf16"] * rms + 2.0 ** -9 * np.abs(o)
    assert np.all(np.abs(res["o"] - o) <= bound)


def test_wide_tree_256_nodes():
    pars = _ragged(7, [256], max_depth=10, fmax=8)
    w = W.synthetic(pars, H=1, dk=128, dv=128, seed=7, log_a_mean=-6.0)
    _full_check(w, "auto")


def test_deep_chain_256():
    """A 256-token chain: the tree degenerates to plain sequential decoding."""
    w = W.synthetic([[i - 1 for i in range(256)]], H=1, dk=64, dv=64, seed=8, in_dtype="f32",
                    log_a_mean=-5.0, s_std=0.05)
    _full_check(w, "auto")


def _comb(spine):
    """A spine of ``spine`` nodes with one leaf hanging off every spine node, interleaved in
    topological order: node 2i is spine node i, node 2i+1 its leaf."""
    par = []
    for i in range(spine):
        par.append(2 * (i - 1) if i else -1)
        par.append(2 * i)
    return par


def _deep_branched_trees():
    return {
        # random frontier growth allowed to reach depth 40 with branching <= 2
        "frontier64_d40": [W.frontier_tree(2024, 64, 40, 2)[0]],
        # depth 33 comb: every node has a sparse ancestor set off the spine
        "comb64": [_comb(32)],
        # just past the register-recursion depth, next to shallow and tiny trees
        "mixed_d9": [W.frontier_tree(77, 64, 9, 3)[0], W.frontier_tree(78, 40, 12, 2)[0],
                     [-1], _comb(5)],
        # two long branches that share a stem of 4 nodes
        "fork": [[-1, 0, 1, 2] + [3] + list(range(4, 32)) + [3] + list(range(33, 62))],
    }


@pytest.mark.parametrize("kernel", ["tc", "simt"])
@pytest.mark.parametrize("name", sorted(_deep_branched_trees()))
def test_deep_branched_trees(name, kernel):
    """Branched trees deeper than the tensor-core kernel's register recursion (depth > 8),
    whose nodes have sparse ancestor sets, compared in full with paths to the deepest
    node of each tree."""
    pars = _deep_branched_trees()[name]
    for p in pars:
        assert all(-1 <= x < i for i, x in enumerate(p)) and len(p) <= 64
    assert max(int(W.depths_of(p).max()) for p in pars) > 8
    paths = []
    for p in pars:
        d = W.depths_of(p)
        n = int(np.flatnonzero(d == d.max())[0])
        paths.append(O.path_to(p, n))
    w = W.synthetic(pars, H=4, dk=128, dv=128, seed=len(name) * 7 + len(pars),
                    paths=paths, log_a_mean=-5.0, name=name)
    _full_check(w, kernel)


def _chain_with_depth(n, depth, seed):
    """n nodes: a root chain of `depth` nodes, the rest attached at random above depth - 1,
    so the deepest path has exactly `depth` nodes."""
    rng = np.random.default_rng(seed)
    par = [i - 1 for i in range(depth)]
    dep = list(range(1, depth + 1))
    for i in range(depth, n):
        while True:
            p = int(rng.integers(-1, i))
            d = 1 if p < 0 else dep[p] + 1
            if d <= depth:
                break
        par.append(p)
        dep.append(d)
    return par


@pytest.mark.parametrize("kernel", ["tc", "simt"])
@pytest.mark.parametrize("counts", [[256, 65, 1, 0, 130], [200, 77], [129, 128, 64, 63]])
def test_wide_ragged_full(kernel, counts):
    """Batches whose largest tree is wider than 64 nodes (the wide tensor-core kernel),
    ragged down to empty and one-node trees, compared in full."""
    w = W.synthetic(_ragged(sum(counts) % 97, counts, max_depth=10, fmax=6), H=3, dk=128,
                    dv=128, seed=len(counts) * 31 + sum(counts), name="wide-ragged",
                    log_a_mean=-6.0)
    _full_check(w, kernel)


@pytest.mark.parametrize("depth", [15, 16, 17, 40])
def test_wide_depth_boundary_tc(depth):
    """Paths of up to 16 nodes stay on the wide kernel's tensor-core path; deeper trees take
    the CUDA-core algorithm inside the same launch.  Both sides of the boundary, with a
    shallow wide tree in the same batch."""
    pars = [_chain_with_depth(150, depth, depth), W.frontier_tree(5 + depth, 90, 8, 4)[0]]
    paths = [O.path_to(p, int(np.argmax(W.depths_of(p)))) for p in pars]
    w = W.synthetic(pars, H=2, dk=128, dv=128, seed=depth, paths=paths, log_a_mean=-6.0,
                    name=f"depth{depth}")
    assert int(W.depths_of(pars[0]).max()) == depth
    _full_check(w, "tc")


def test_wide_scalar_and_bf16_output():
    pars = _ragged(11, [180, 90], max_depth=9, fmax=5)
    w = W.synthetic(pars, H=2, dk=128, dv=128, seed=11, mode="scalar", log_a_mean=-3.0)
    _full_check(w, "tc")
    w = W.synthetic(pars, H=2, dk=128, dv=128, seed=12, out_dtype="bf16", log_a_mean=-6.0)
    res, _ = run(w, kernel="tc")
    o, _ = O.tree_verify(w)
    rms = np.sqrt(np.mean(o ** 2))
    assert np.all(np.abs(res["o"] - o) <= TOL["bf16"] * rms + 2.0 ** -9 * np.abs(o))
