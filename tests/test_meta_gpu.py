"""Tree metadata on the GPU is bit-exact: depth, ancestor bitmask, and the cumulative
log-decay accumulated in fp32 from the root down (also within 1e-6 of the fp64 sum)."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _fp32_root_down(parent, log_a):
    cl = np.zeros(log_a.shape, dtype=np.float32)
    for i, p in enumerate(parent):
        cl[i] = (np.float32(0) if p < 0 else cl[p]) + log_a[i]
    return cl


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_meta_bit_exact(idx):
    w = W.config(idx)
    d = to_device(w)
    depth, anc, cl = L.tree_meta(d["parent"], d["node_offsets"], d["log_a"],
                                 max_nodes=w.max_nodes)
    depth, anc, cl = depth.cpu().numpy(), anc.cpu().numpy().view(np.uint64), cl.cpu().numpy()
    Wd = (w.max_nodes + 63) // 64
    for s in range(w.B):
        lo, hi = int(w.node_offsets[s]), int(w.node_offsets[s + 1])
        par = w.parent[lo:hi]
        dep, ancs, cl64 = O.tree_meta(par, w.log_a[lo:hi])
        np.testing.assert_array_equal(depth[lo:hi], dep)
        for n in range(hi - lo):
            words = np.zeros(Wd, dtype=np.uint64)
            for i in ancs[n]:
                words[i // 64] |= np.uint64(1) << np.uint64(i % 64)
            np.testing.assert_array_equal(anc[lo + n], words)
        np.testing.assert_array_equal(cl[lo:hi], _fp32_root_down(par, w.log_a[lo:hi]))
        np.testing.assert_allclose(cl[lo:hi], cl64, rtol=1e-6, atol=1e-7)


def test_meta_bad_tree_sets_status():
    w = W.config(2)
    d = to_device(w)
    d["parent"][5] = 7          # not topological
    ws = L.new_workspace(L.make_problem(w.B, w.H, 16, 16, w.T, w.max_nodes))
    L.tree_meta(d["parent"], d["node_offsets"], d["log_a"], max_nodes=w.max_nodes, workspace=ws)
    assert L.get_status(ws) == L.binding.TV_ERR_BAD_TREE
    assert L.get_status(ws) == 0          # read clears
