"""The streaming commit (dk = dv = 128) against the float64 oracle at its edges: paths
longer than the rows it stages in shared memory, path lengths either side of that limit,
and many (sequence, head) items per CTA, so that each CTA's range crosses sequence
boundaries, with one sequence's path malformed."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run
from linear_attention_tree_b200.tensors import to_device

pytestmark = pytest.mark.gpu


def _check_all_states(w, res):
    want = np.array([[O.commit_sequence(w, s, h, w.accepted_path[s]) for h in range(w.H)]
                     for s in range(w.B)])
    assert_close(res["S_new"], want, TOL["bf16"], "S_new")


def test_full_chain_path_reads_rows_from_hbm():
    """A 64-node chain committed to its leaf: 56 of the 64 path rows come from HBM."""
    w = W.synthetic([[i - 1 for i in range(64)]], H=3, dk=128, dv=128, seed=21,
                    log_a_mean=-5.0, paths=[list(range(64))])
    res, _ = run(w)
    _check_all_states(w, res)


def test_path_lengths_around_the_staged_rows():
    lengths = [0, 7, 8, 9, 20]
    w = W.synthetic([[i - 1 for i in range(24)] for _ in lengths], H=2, dk=128, dv=128,
                    seed=22, log_a_mean=-5.0, paths=[list(range(n)) for n in lengths])
    res, _ = run(w)
    _check_all_states(w, res)


def test_many_items_per_cta_with_a_bad_sequence():
    """480 items over the SMs: CTA ranges cross sequence boundaries (12 heads per
    sequence), and sequence 7's path is malformed; every other state must be right."""
    pars = [W.frontier_tree(300 + i, 24, 6, 3)[0] for i in range(40)]
    # default paths: root -> last node of every sequence (rows padded to the longest)
    w = W.synthetic(pars, H=12, dk=128, dv=128, seed=23)
    assert w.max_path >= 2
    d = to_device(w)
    out, U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                           d["node_offsets"], d["S_root"], max_nodes=w.max_nodes)
    path = d["accepted_path"].clone()
    path[7, :] = -1
    path[7, 0] = 0
    path[7, 1] = 30                                  # beyond the sequence's 24 nodes
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"], path,
                          max_nodes=w.max_nodes, parent=d["parent"], workspace=ws)
    assert L.get_status(ws) == L.binding.TV_ERR_BAD_PATH
    got = S_new.cpu().numpy().astype(np.float64)
    for s in range(w.B):
        if s == 7:
            continue
        want = np.array([O.commit_sequence(w, s, h, w.accepted_path[s]) for h in range(w.H)])
        assert_close(got[s], want, TOL["bf16"], f"S_new of sequence {s}")


def test_in_place_long_paths():
    """In place (S_new is S_root) with paths past the staged rows."""
    w = W.synthetic([[i - 1 for i in range(32)] for _ in range(6)], H=4, dk=128, dv=128,
                    seed=24, log_a_mean=-5.0,
                    paths=[list(range(n)) for n in (32, 1, 12, 9, 0, 31)])
    d = to_device(w)
    out, U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                           d["node_offsets"], d["S_root"], max_nodes=w.max_nodes)
    S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                          d["accepted_path"], max_nodes=w.max_nodes, parent=d["parent"])
    S = d["S_root"].clone()
    L.tree_commit(U, d["k"], d["log_a"], S, d["node_offsets"], d["accepted_path"],
                  max_nodes=w.max_nodes, S_new=S)
    torch.testing.assert_close(S, S_new, rtol=0, atol=0)


@pytest.mark.parametrize("in_place", [False, True])
def test_two_commits_back_to_back_on_chained_states(in_place):
    """commit -> commit on one stream, the second reading the first one's S_new (a new
    buffer, or S_root itself in place), with nothing between them.  Scalar decay makes
    U = V valid for any root state, so the second commit's pseudo-values need no verify
    on the intermediate state; the oracle walks path A from S_root, then path B."""
    pars = [W.frontier_tree(600 + s, 40, 8, 3)[0] for s in range(40)]
    rng = np.random.default_rng(61)
    paths_a, paths_b = [], []
    for p in pars:
        d = W.depths_of(p)
        paths_a.append(O.path_to(p, int(rng.integers(0, len(p)))))
        paths_b.append(O.path_to(p, int(np.argmax(d))))
    w = W.synthetic(pars, H=8, dk=128, dv=128, seed=61, mode="scalar", paths=paths_a,
                    log_a_mean=-3.0)
    d = to_device(w)
    U = d["v"].float().contiguous()                    # scalar decay: u_n = v_n
    width = max(len(p) for p in paths_a + paths_b)
    pad = lambda ps: torch.tensor([p + [-1] * (width - len(p)) for p in ps],
                                  dtype=torch.int32, device="cuda")
    path_a, path_b = pad(paths_a), pad(paths_b)
    ws = L.new_workspace(L.make_problem(w.B, w.H, 128, 128, w.T, w.max_nodes, width))
    S0 = d["S_root"].clone()
    mid = S0 if in_place else torch.empty_like(S0)
    L.tree_commit(U, d["k"], d["log_a"], S0, d["node_offsets"], path_a,
                  max_nodes=w.max_nodes, parent=d["parent"], S_new=mid, workspace=ws)
    end = mid if in_place else torch.empty_like(S0)
    L.tree_commit(U, d["k"], d["log_a"], mid, d["node_offsets"], path_b,
                  max_nodes=w.max_nodes, parent=d["parent"], S_new=end, workspace=ws)
    assert L.get_status(ws) == 0
    got = end.cpu().numpy().astype(np.float64)
    want = np.empty_like(got)
    for s in range(w.B):
        for h in range(w.H):
            q, k, v, la, b, S, parent = O._head(w, s, h)
            S = O.walk(S, paths_a[s], k, v, la, b, "scalar")[0]
            want[s, h] = O.walk(S, paths_b[s], k, v, la, b, "scalar")[0]
    assert_close(got, want, TOL["bf16"], "S_new after two chained commits")
