"""Bad device data sets the status word (first error wins) and never traps; the GPU
keeps working and a following valid call is correct.  Guard regions around the outputs
stay untouched (a stand-in for an out-of-bounds checker)."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run

pytestmark = pytest.mark.gpu


def _verify(w, d, ws, kernel="auto", **kw):
    return L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                         d["node_offsets"], d["S_root"], max_nodes=w.max_nodes, mode=w.mode,
                         workspace=ws, kernel=kernel, **kw)


@pytest.mark.parametrize("kernel", ["tc", "simt"])
@pytest.mark.parametrize("bad", ["self_parent", "forward_parent", "below_minus_one",
                                 "offsets_decreasing", "offsets_too_many"])
def test_bad_tree(kernel, bad):
    w = W.config(3)
    d = to_device(w)
    if bad == "self_parent":
        d["parent"][70] = 6
    elif bad == "forward_parent":
        d["parent"][70] = 20
    elif bad == "below_minus_one":
        d["parent"][70] = -2
    elif bad == "offsets_decreasing":
        d["node_offsets"][3] = 100
    elif bad == "offsets_too_many":
        d["node_offsets"][1] = 0
        d["node_offsets"][2] = 128        # 128 nodes > max_nodes in sequence 1
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes))
    _verify(w, d, ws, kernel)
    assert L.get_status(ws) == L.binding.TV_ERR_BAD_TREE
    # the context is healthy: a valid call afterwards is correct
    res, _ = run(W.config(2))
    o, _ = O.tree_verify(W.config(2))
    assert_close(res["o"], o, TOL["bf16"], "o after error")


@pytest.mark.parametrize("bad", ["not_a_chain", "out_of_range", "hole", "not_root_first"])
def test_bad_path(bad):
    w = W.config(3)
    d = to_device(w)
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    out, U = _verify(w, d, ws)
    path = d["accepted_path"].clone()
    row = [int(x) for x in w.accepted_path[2] if x >= 0]
    if bad == "not_a_chain":
        path[2, 0] = row[0]
        path[2, 1] = 63 if row[0] != 63 and w.parent[128 + 63] != row[0] else 62
    elif bad == "out_of_range":
        path[2, 0] = 64
    elif bad == "hole":
        path[2, :] = -1
        path[2, 0] = row[0]
        path[2, 2] = row[0]
    elif bad == "not_root_first":
        deep = [i for i in range(64) if w.parent[128 + i] >= 0][0]
        path[2, :] = -1
        path[2, 0] = deep
    S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"], path,
                          max_nodes=w.max_nodes, parent=d["parent"], workspace=ws)
    assert L.get_status(ws) == L.binding.TV_ERR_BAD_PATH
    # other sequences committed correctly
    want = O.commit_sequence(w, 5, 3, w.accepted_path[5])
    assert_close(S_new[5, 3].cpu().numpy(), want, TOL["bf16"], "other sequence")


@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_guard_regions_untouched(kernel):
    """Outputs carved out of larger NaN-filled buffers: nothing outside is written."""
    pars = [W.frontier_tree(50 + i, c, 8, 4)[0] for i, c in enumerate([63, 1, 64, 17])]
    w = W.synthetic(pars, H=3, dk=128, dv=128, seed=50)
    d = to_device(w)
    G = 4096
    T, H, dv = w.T, w.H, w.dv
    obuf = torch.full((G + T * H * dv + G,), float("nan"), dtype=torch.bfloat16, device="cuda")
    ubuf = torch.full((G + T * H * dv + G,), float("nan"), dtype=torch.float32, device="cuda")
    sbuf = torch.full((G + w.B * H * dv * w.dk + G,), float("nan"), dtype=torch.float32,
                      device="cuda")
    out = obuf[G:G + T * H * dv].view(T, H, dv)
    U = ubuf[G:G + T * H * dv].view(T, H, dv)
    S_new = sbuf[G:G + w.B * H * dv * w.dk].view(w.B, H, dv, w.dk)
    ws = L.new_workspace(L.make_problem(w.B, H, w.dk, dv, T, w.max_nodes, w.max_path))
    _verify(w, d, ws, kernel, out=out, U=U)
    L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"], d["accepted_path"],
                  max_nodes=w.max_nodes, parent=d["parent"], S_new=S_new, workspace=ws)
    assert L.get_status(ws) == 0
    for buf in (obuf, ubuf, sbuf):
        assert torch.isnan(buf[:G].float()).all() and torch.isnan(buf[-G:].float()).all()
    assert torch.isfinite(out.float()).all() and torch.isfinite(U).all()
    assert torch.isfinite(S_new).all()


def test_unsupported_kernel_raises():
    w = W.config(1)
    d = to_device(w)
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes))
    with pytest.raises(L.TreeVerifyError):
        _verify(w, d, ws, kernel="tc")


def test_wait_that_runs_out_is_reported_and_the_context_survives():
    """A bounded mbarrier wait that never completes (the library's diagnostic kernel) ends
    with TV_ERR_TIMEOUT in the status word instead of a hang; the next call is correct."""
    w = W.config(2)
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    L.binding.selftest_timeout(ws)
    assert L.get_status(ws) == L.binding.TV_ERR_TIMEOUT
    assert L.get_status(ws) == 0                      # read once, then cleared
    res, _ = run(w)
    o, U = O.tree_verify(w)
    assert_close(res["o"], o, TOL["bf16"], "o after a time-out")
    assert_close(res["U"], U, TOL["bf16"], "U after a time-out")
