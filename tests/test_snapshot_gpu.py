"""The per-node-snapshot baseline (tv_snapshot_verify / tv_snapshot_commit) against the
float64 oracle: its outputs, its committed state, and every node's snapshot, which must be
the state the recurrence reaches along that node's path."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close

pytestmark = pytest.mark.gpu


def _run(w):
    d = to_device(w)
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    out, U, snap = L.snapshot_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                                     d["node_offsets"], d["S_root"], max_nodes=w.max_nodes,
                                     mode=w.mode, out_dtype=torch.float32, workspace=ws)
    S_new = L.snapshot_commit(snap, d["S_root"], d["node_offsets"], d["accepted_path"],
                              max_nodes=w.max_nodes, parent=d["parent"], workspace=ws)
    assert L.get_status(ws) == 0
    f64 = lambda t: t.cpu().numpy().astype(np.float64)
    return f64(out), f64(U), f64(snap), f64(S_new)


@pytest.mark.parametrize("name", ["config2", "ragged", "scalar_f32"])
def test_snapshot_baseline_matches_the_oracle(name):
    if name == "config2":
        w = W.config(2)
    elif name == "ragged":
        pars = [W.frontier_tree(40 + i, c, 8, 4)[0] if c else [] for i, c in enumerate([64, 0, 9, 33])]
        w = W.synthetic(pars, H=3, dk=128, dv=128, seed=44, log_a_mean=-5.0)
    else:
        pars = [W.uniform_parent_tree(np.random.default_rng(3), 20, 5)]
        w = W.synthetic(pars, H=2, dk=32, dv=64, seed=45, mode="scalar", in_dtype="f32",
                        log_a_mean=-2.0, s_std=0.1)
    o, U, snap, S_new = _run(w)
    o_ref, U_ref = O.tree_verify(w)
    tol = TOL[w.in_dtype]
    assert_close(o, o_ref, tol, "o")
    assert_close(U, U_ref, tol, "U")
    assert_close(S_new, O.tree_commit(w), tol, "S_new")
    # every node's snapshot is its walked state
    for s in range(w.B):
        lo = int(w.node_offsets[s])
        for h in range(w.H):
            states = O.node_states(w, s, h)
            if len(states):
                assert_close(snap[lo:lo + len(states), h], states, tol, f"snapshots {s} {h}")
