"""Variants of the hot path: value heads sharing q / k heads, and pseudo-values stored in
bf16.  Each is held to the float64 oracle in full.  bf16 U is rounded to nearest once it is
final, so its bar is the usual 2e-2 of RMS plus one bf16 rounding step of each element
(2^-8 of its size); o, which never goes through the stored U, keeps the plain bar."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run

pytestmark = pytest.mark.gpu


def _trees(seed, counts, max_depth=8, fmax=4):
    return [W.frontier_tree(seed * 100 + i, c, max_depth, fmax)[0] if c else []
            for i, c in enumerate(counts)]


def _bf16_u_close(got, want, what):
    rms = float(np.sqrt(np.mean(want ** 2)))
    bound = TOL["bf16"] * rms + 2.0 ** -8 * np.abs(want)
    assert np.all(np.abs(got - want) <= bound), f"{what}: beyond 2e-2 RMS + half a bf16 step"


@pytest.mark.parametrize("kernel,counts", [("tc", [64, 31, 64]), ("tc", [200, 70]),
                                           ("simt", [64, 31, 64]), ("simt", [200, 70])])
def test_grouped_qk_heads(kernel, counts):
    """8 value heads on 2 q / k heads (4 value heads each), every output and state."""
    w = W.synthetic(_trees(61, counts, 10, 6), H=8, dk=128, dv=128, seed=61, qk_heads=2,
                    log_a_mean=-6.0)
    assert w.q.shape[1] == 2
    res, _ = run(w, kernel=kernel)
    o, U = O.tree_verify(w)
    assert_close(res["o"], o, TOL["bf16"], "o")
    assert_close(res["U"], U, TOL["bf16"], "U")
    assert_close(res["S_new"], O.tree_commit(w), TOL["bf16"], "S_new")


def test_grouped_qk_heads_fused_and_snapshot():
    w0 = W.synthetic(_trees(62, [64, 40]), H=4, dk=128, dv=128, seed=62, qk_heads=1)
    w1 = W.synthetic(_trees(63, [50, 64]), H=4, dk=128, dv=128, seed=63, qk_heads=1)
    d0, d1 = to_device(w0), to_device(w1)
    _, U0 = L.tree_verify(d0["q"], d0["k"], d0["v"], d0["log_a"], d0["b"], d0["parent"],
                          d0["node_offsets"], d0["S_root"], max_nodes=w0.max_nodes,
                          out_dtype=torch.float32)
    S_new, o, U = L.tree_commit_verify(
        U0, d0["k"], d0["log_a"], d0["node_offsets"], d0["accepted_path"], d0["S_root"],
        d1["q"], d1["k"], d1["v"], d1["log_a"], d1["b"], d1["parent"], d1["node_offsets"],
        max_nodes_prev=w0.max_nodes, max_nodes=w1.max_nodes, parent_prev=d0["parent"],
        out_dtype=torch.float32)
    out_s, U_s, _ = L.snapshot_verify(d0["q"], d0["k"], d0["v"], d0["log_a"], d0["b"],
                                      d0["parent"], d0["node_offsets"], d0["S_root"],
                                      max_nodes=w0.max_nodes, out_dtype=torch.float32)
    torch.cuda.synchronize()
    S_ref = O.tree_commit(w0)
    assert_close(S_new.cpu().numpy(), S_ref, TOL["bf16"], "S_new")
    w1.S_root = S_new.cpu().numpy()
    o_ref, U_ref = O.tree_verify(w1)
    assert_close(o.cpu().numpy(), o_ref, TOL["bf16"], "o after the fused commit")
    assert_close(U.cpu().numpy(), U_ref, TOL["bf16"], "U after the fused commit")
    o0, U0_ref = O.tree_verify(w0)
    assert_close(out_s.cpu().numpy(), o0, TOL["bf16"], "snapshot baseline o")
    assert_close(U_s.cpu().numpy(), U0_ref, TOL["bf16"], "snapshot baseline U")


@pytest.mark.parametrize("counts,depth", [([64, 17, 64, 1], 8), ([256, 90], 10),
                                          ([150, 80], 40)])
def test_bf16_pseudo_values(counts, depth):
    """U stored in bf16 by both tensor-core kernels (and the CUDA-core fallback for paths
    deeper than 16 inside the wide one), read back in bf16 by the commit."""
    pars = _trees(64 + depth, counts, depth, 6 if depth <= 10 else 2)
    w = W.synthetic(pars, H=3, dk=128, dv=128, seed=depth, log_a_mean=-6.0,
                    paths=[O.path_to(p, int(np.argmax(W.depths_of(p)))) if p else [] for p in pars])
    res, d = run(w, kernel="tc", u_dtype=torch.bfloat16)
    o, U = O.tree_verify(w)
    assert_close(res["o"], o, TOL["bf16"], "o")
    _bf16_u_close(res["U"], U, "U")
    assert_close(res["S_new"], O.tree_commit(w), TOL["bf16"], "S_new from bf16 U")


def test_bf16_pseudo_values_sliced_commit_and_fused():
    """The sliced commit (dk = dv = 64, fp32 inputs) on bf16 U rounded from the oracle's,
    and a fused commit + verify whose previous and next U are both bf16."""
    pars = _trees(70, [30, 12])
    w = W.synthetic(pars, H=2, dk=64, dv=64, seed=70, in_dtype="f32", log_a_mean=-3.0, s_std=0.1)
    d = to_device(w)
    _, U_ref = O.tree_verify(w)
    U16 = torch.from_numpy(U_ref.astype(np.float32)).to(torch.bfloat16).cuda()
    S_new = L.tree_commit(U16, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                          d["accepted_path"], max_nodes=w.max_nodes, parent=d["parent"])
    torch.cuda.synchronize()
    assert_close(S_new.cpu().numpy(), O.tree_commit(w), TOL["bf16"], "S_new (sliced, bf16 U)")

    w0 = W.synthetic(_trees(71, [64, 33]), H=2, dk=128, dv=128, seed=71)
    w1 = W.synthetic(_trees(72, [20, 64]), H=2, dk=128, dv=128, seed=72)
    d0, d1 = to_device(w0), to_device(w1)
    _, U0 = L.tree_verify(d0["q"], d0["k"], d0["v"], d0["log_a"], d0["b"], d0["parent"],
                          d0["node_offsets"], d0["S_root"], max_nodes=w0.max_nodes,
                          out_dtype=torch.float32, u_dtype=torch.bfloat16)
    assert U0.dtype == torch.bfloat16
    S1, o, U1 = L.tree_commit_verify(
        U0, d0["k"], d0["log_a"], d0["node_offsets"], d0["accepted_path"], d0["S_root"],
        d1["q"], d1["k"], d1["v"], d1["log_a"], d1["b"], d1["parent"], d1["node_offsets"],
        max_nodes_prev=w0.max_nodes, max_nodes=w1.max_nodes, parent_prev=d0["parent"],
        out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert U1.dtype == torch.bfloat16
    assert_close(S1.cpu().numpy(), O.tree_commit(w0), TOL["bf16"], "fused S_new")
    w1.S_root = S1.cpu().numpy()
    o_ref, U1_ref = O.tree_verify(w1)
    assert_close(o.cpu().numpy(), o_ref, TOL["bf16"], "fused o")
    _bf16_u_close(U1.float().cpu().numpy().astype(np.float64), U1_ref, "fused U")
