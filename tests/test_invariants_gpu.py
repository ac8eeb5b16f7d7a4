"""Structural invariants of the CUDA path that hold at any size (run on the GPU)."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run

pytestmark = pytest.mark.gpu

KERNELS = ["tc", "simt"]


@pytest.mark.parametrize("kernel", KERNELS)
def test_deterministic_bitwise(kernel):
    w = W.config(3)
    a, _ = run(w, kernel=kernel)
    b, _ = run(w, kernel=kernel)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])


@pytest.mark.parametrize("kernel", KERNELS)
def test_sibling_perturbation_bitwise(kernel):
    """Changing the inputs of nodes off a node's path leaves its o and U bit-identical."""
    par, _ = W.frontier_tree(99, 64, 8, 4)
    w = W.synthetic([par], H=4, dk=128, dv=128, seed=99)
    a, _ = run(w, kernel=kernel, commit=False)
    target = 63
    on_path = set(O.path_to(par, target))
    for j in range(64):
        if j not in on_path:
            w.q[j] = W.bf16_round(w.q[j] * -0.5)
            w.k[j] = W.bf16_round(w.k[j] * 0.25 + 0.1)
            w.v[j] = W.bf16_round(w.v[j] + 1.0)
            w.log_a[j] -= 0.3
            w.b[j] = 0.9
    b, _ = run(w, kernel=kernel, commit=False)
    for n in on_path:
        np.testing.assert_array_equal(b["o"][n], a["o"][n])
        np.testing.assert_array_equal(b["U"][n], a["U"][n])


@pytest.mark.parametrize("kernel", KERNELS)
def test_relabel_permutes(kernel):
    par, _ = W.frontier_tree(7, 48, 8, 4)
    w = W.synthetic([par], H=2, dk=128, dv=128, seed=7)
    a, _ = run(w, kernel=kernel, commit=False)
    dep = W.depths_of(par)
    order = sorted(range(48), key=lambda i: (dep[i], -i))
    new_of = {old: new for new, old in enumerate(order)}
    par2 = [(-1 if par[o] < 0 else new_of[par[o]]) for o in order]
    w2 = W.synthetic([par2], H=2, dk=128, dv=128, seed=7)
    for name in ("q", "k", "v", "log_a", "b"):
        getattr(w2, name)[:] = getattr(w, name)[order]
    w2.S_root[:] = w.S_root
    b, _ = run(w2, kernel=kernel, commit=False)
    tol = TOL["bf16"]
    # the per-node arithmetic may be reordered across nodes, so compare to tolerance
    assert_close(b["o"], a["o"][order], tol * 0.05, "o relabelled")
    assert_close(b["U"], a["U"][order], tol * 0.05, "U relabelled")


@pytest.mark.parametrize("kernel", KERNELS)
def test_b_zero_pure_decay(kernel):
    par, _ = W.frontier_tree(3, 64, 8, 4)
    w = W.synthetic([par], H=2, dk=128, dv=128, seed=3)
    w.b[:] = 0.0
    res, _ = run(w, kernel=kernel)
    assert np.all(res["U"] == 0.0)
    o, _ = O.tree_verify(w)
    assert_close(res["o"], o, TOL["bf16"], "o with b=0")


def test_in_place_commit_equals_out_of_place():
    w = W.config(3)
    d = to_device(w)
    out, U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                           d["node_offsets"], d["S_root"], max_nodes=w.max_nodes)
    S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                          d["accepted_path"], max_nodes=w.max_nodes, parent=d["parent"])
    S_inplace = d["S_root"].clone()
    L.tree_commit(U, d["k"], d["log_a"], S_inplace, d["node_offsets"], d["accepted_path"],
                  max_nodes=w.max_nodes, S_new=S_inplace)
    torch.testing.assert_close(S_inplace, S_new, rtol=0, atol=0)


def test_empty_path_commits_root():
    w = W.config(3)
    d = to_device(w)
    U = torch.zeros((w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    paths = torch.full((w.B, 4), -1, dtype=torch.int32, device="cuda")
    S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"], paths,
                          max_nodes=w.max_nodes, parent=d["parent"])
    torch.testing.assert_close(S_new, d["S_root"], rtol=0, atol=0)


def test_chain_equals_sequential_and_commit_matches_last_state():
    n = 64
    w = W.synthetic([[i - 1 for i in range(n)]], H=2, dk=128, dv=128, seed=12)
    res, _ = run(w)
    o, U = O.tree_verify(w)
    assert_close(res["o"], o, TOL["bf16"], "chain o")
    assert_close(res["S_new"], O.tree_commit(w), TOL["bf16"], "chain S_new")
