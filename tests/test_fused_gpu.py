"""tv_tree_commit_verify: the previous step's commit and the next tree's verify against the
committed state, in one pass over the state.  Its results must be those of the two separate
calls (bit for bit where the fused kernel runs, since it performs the same arithmetic), and a
decode loop driven by it must follow the float64 oracle's own steps."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close

pytestmark = pytest.mark.gpu


def _tree_set(t, counts, fmax=4, max_depth=8, paths=None):
    pars = [W.frontier_tree(900 + 13 * t + i, c, max_depth, fmax)[0] if c else []
            for i, c in enumerate(counts)]
    if paths is None:
        rng = np.random.default_rng(t)
        paths = [O.path_to(p, int(rng.integers(0, len(p)))) if p else [] for p in pars]
    return W.synthetic(pars, H=4, dk=128, dv=128, seed=80 + t, paths=paths, log_a_mean=-5.0)


def _fused(dp, wp, dn, wn, S, S_new, kernel="auto", accepted_path=None, U=None):
    return L.tree_commit_verify(
        dp["U"], dp["k"], dp["log_a"], dp["node_offsets"],
        dp["accepted_path"] if accepted_path is None else accepted_path, S,
        dn["q"], dn["k"], dn["v"], dn["log_a"], dn["b"], dn["parent"], dn["node_offsets"],
        max_nodes_prev=wp.max_nodes, max_nodes=wn.max_nodes, parent_prev=dp["parent"],
        S_new=S_new, out_dtype=torch.float32, kernel=kernel, U=U)


@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_fused_decode_loop_follows_the_oracle(kernel):
    """Four steps on one stream, the state updated in place: verify(0), then
    commit(t-1) + verify(t) fused for t = 1..3, then commit(3).  The oracle runs its own
    four steps (its S_new rounded to fp32 is its next S_root)."""
    ws_ = [_tree_set(t, [64, 40, 64, 17, 64, 5]) for t in range(4)]
    ds = [to_device(w) for w in ws_]
    S = ds[0]["S_root"].clone()
    outs = []
    o, U = L.tree_verify(ds[0]["q"], ds[0]["k"], ds[0]["v"], ds[0]["log_a"], ds[0]["b"],
                         ds[0]["parent"], ds[0]["node_offsets"], S, max_nodes=ws_[0].max_nodes,
                         out_dtype=torch.float32, kernel=kernel)
    ds[0]["U"] = U
    outs.append(o)
    for t in range(1, 4):
        _, o, U = _fused(ds[t - 1], ws_[t - 1], ds[t], ws_[t], S, S, kernel=kernel)
        ds[t]["U"] = U
        outs.append(o)
    L.tree_commit(ds[3]["U"], ds[3]["k"], ds[3]["log_a"], S, ds[3]["node_offsets"],
                  ds[3]["accepted_path"], max_nodes=ws_[3].max_nodes, parent=ds[3]["parent"],
                  S_new=S)
    torch.cuda.synchronize()
    S_ref = ws_[0].S_root.astype(np.float32)
    for t, w in enumerate(ws_):
        w.S_root = S_ref
        o_ref, U_ref = O.tree_verify(w)
        assert_close(outs[t].cpu().numpy(), o_ref, TOL["bf16"], f"o at step {t}")
        assert_close(ds[t]["U"].cpu().numpy(), U_ref, TOL["bf16"], f"U at step {t}")
        S_ref = O.tree_commit(w).astype(np.float32)
    assert_close(S.cpu().numpy(), S_ref, TOL["bf16"], "state after the last step")


@pytest.mark.parametrize("in_place", [False, True])
def test_fused_equals_the_two_calls_bitwise(in_place):
    wp, wn = _tree_set(1, [64, 33, 64, 1]), _tree_set(2, [50, 64, 12, 64])
    dp, dn = to_device(wp), to_device(wn)
    _, Up = L.tree_verify(dp["q"], dp["k"], dp["v"], dp["log_a"], dp["b"], dp["parent"],
                          dp["node_offsets"], dp["S_root"], max_nodes=wp.max_nodes,
                          out_dtype=torch.float32)
    dp["U"] = Up
    S_sep = L.tree_commit(Up, dp["k"], dp["log_a"], dp["S_root"], dp["node_offsets"],
                          dp["accepted_path"], max_nodes=wp.max_nodes, parent=dp["parent"])
    o_sep, U_sep = L.tree_verify(dn["q"], dn["k"], dn["v"], dn["log_a"], dn["b"], dn["parent"],
                                 dn["node_offsets"], S_sep, max_nodes=wn.max_nodes,
                                 out_dtype=torch.float32)
    S0 = dp["S_root"].clone()
    S_new, o, U = _fused(dp, wp, dn, wn, S0, S0 if in_place else None)
    torch.cuda.synchronize()
    torch.testing.assert_close(S_new, S_sep, rtol=0, atol=0)
    torch.testing.assert_close(o, o_sep, rtol=0, atol=0)
    torch.testing.assert_close(U, U_sep, rtol=0, atol=0)


def test_fused_edges():
    """Next trees that are empty or one node, previous paths of length 0 and of 32 (the
    longest the single pass takes), and one malformed path: that sequence is reported, the
    others are exact."""
    counts_p = [64, 40, 33, 64, 20]
    pars_p = [[i - 1 for i in range(64)]] + \
        [W.frontier_tree(950 + i, c, 8, 4)[0] for i, c in enumerate(counts_p[1:])]
    paths = [list(range(32)), [], O.path_to(pars_p[2], 20), O.path_to(pars_p[3], 63), [0]]
    wp = W.synthetic(pars_p, H=2, dk=128, dv=128, seed=95, paths=paths, log_a_mean=-5.0)
    wn = _tree_set(9, [0, 1, 64, 10, 0])
    wn.H, wn.q, wn.k, wn.v, wn.log_a, wn.b = 2, wn.q[:, :2], wn.k[:, :2], wn.v[:, :2], \
        wn.log_a[:, :2], wn.b[:, :2]
    wn.S_root = wn.S_root[:, :2]
    dp, dn = to_device(wp), to_device(wn)
    _, Up = L.tree_verify(dp["q"], dp["k"], dp["v"], dp["log_a"], dp["b"], dp["parent"],
                          dp["node_offsets"], dp["S_root"], max_nodes=wp.max_nodes,
                          out_dtype=torch.float32)
    dp["U"] = Up
    ap = dp["accepted_path"].clone()
    assert ap.shape[1] == 32
    ap[4, 0] = 7                         # sequence 4: node 7 is not a root child
    ws = L.new_workspace(L.make_problem(wn.B, 2, 128, 128, wn.T, wn.max_nodes, 32))
    S0 = dp["S_root"].clone()
    S_new, o, U = L.tree_commit_verify(
        Up, dp["k"], dp["log_a"], dp["node_offsets"], ap, S0, dn["q"], dn["k"], dn["v"],
        dn["log_a"], dn["b"], dn["parent"], dn["node_offsets"], max_nodes_prev=wp.max_nodes,
        max_nodes=wn.max_nodes, parent_prev=dp["parent"], out_dtype=torch.float32,
        workspace=ws)
    assert L.get_status(ws) == L.binding.TV_ERR_BAD_PATH
    S_ref = np.array([[O.commit_sequence(wp, s, h, wp.accepted_path[s]) for h in range(2)]
                      for s in range(wp.B)])
    got = S_new.cpu().numpy().astype(np.float64)
    assert_close(got[:4], S_ref[:4], TOL["bf16"], "S_new of the well-formed sequences")
    wn.S_root = got.astype(np.float32)
    o_ref, U_ref = O.tree_verify(wn, seqs=[1, 2, 3])
    rows = slice(int(wn.node_offsets[1]), int(wn.node_offsets[4]))
    assert_close(o.cpu().numpy()[rows], o_ref[rows], TOL["bf16"], "o")
    assert_close(U.cpu().numpy()[rows], U_ref[rows], TOL["bf16"], "U")
