"""The seeded generators produce the tree shapes and value distributions they promise."""
import numpy as np
import pytest

from linear_attention_tree_b200 import workloads as W


def _check_common(w):
    assert w.node_offsets[0] == 0 and np.all(np.diff(w.node_offsets) >= 0)
    assert w.q.shape == (w.T, w.H, w.dk) and w.v.shape == (w.T, w.H, w.dv)
    assert w.S_root.shape == (w.B, w.H, w.dv, w.dk)
    for s in range(w.B):
        par = w.seq_parent(s)
        assert all(-1 <= p < i for i, p in enumerate(par)), "topological order"
        path = [int(x) for x in w.accepted_path[s] if x >= 0]
        # padding only at the tail, and the path is a root-first chain of the tree
        assert list(w.accepted_path[s][:len(path)]) == path
        for j, n in enumerate(path):
            assert par[n] == (path[j - 1] if j else -1)
    if w.in_dtype == "bf16":
        for x in (w.q, w.k, w.v):
            np.testing.assert_array_equal(W.bf16_round(x), x)


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_config_shapes(idx):
    w = W.config(idx)
    _check_common(w)
    dep = np.concatenate([W.depths_of(w.seq_parent(s)) for s in range(w.B)])
    expect = {1: (6, 3), 2: (16, 6), 3: (2048, 8), 4: (3072, 7), 5: (2048, 10)}[idx]
    assert w.T == expect[0]
    assert dep.max() <= expect[1]
    if idx == 4:
        n = np.diff(w.node_offsets)
        assert n.min() >= 8 and n.max() <= 48 and n.sum() == 3072
    if idx in (3, 5):
        assert np.all(np.diff(w.node_offsets) == (64 if idx == 3 else 256))
    if idx == 5:
        for s in range(w.B):
            d = W.depths_of(w.seq_parent(s))
            end = [x for x in w.accepted_path[s] if x >= 0][-1]
            assert d[end] == d.max() and end == int(np.flatnonzero(d == d.max())[0])
    if idx >= 2:
        qn = np.linalg.norm(w.q.astype(np.float64), axis=-1)
        assert np.all(np.abs(qn - 1) < 1e-2)
        assert np.all((w.b > 0) & (w.b < 1)) and np.all(w.log_a < 0)


def test_branching_limits():
    for fmax, maxd in ((4, 8), (8, 10)):
        for s in range(20):
            par, _ = W.frontier_tree(1234 + s, 64, maxd, fmax)
            counts = np.bincount(np.array(par) + 1)
            assert counts.max() <= fmax and W.depths_of(par).max() <= maxd


def test_deterministic():
    a, b = W.config(3), W.config(3)
    np.testing.assert_array_equal(a.parent, b.parent)
    np.testing.assert_array_equal(a.S_root, b.S_root)
    np.testing.assert_array_equal(a.accepted_path, b.accepted_path)
    c = W.config(3, seed=1)
    assert not np.array_equal(a.S_root, c.S_root)


def test_bf16_round_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-30], dtype=np.float32)
    r = W.bf16_round(x)
    np.testing.assert_array_equal(r[:4], np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5], np.float32))
