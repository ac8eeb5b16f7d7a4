"""Helpers shared by the GPU tests: run the library on a Workload, compare with the oracle."""
import numpy as np
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200.tensors import to_device

TOL = {"f32": 1e-4, "bf16": 2e-2}


def run(w, kernel="auto", out_dtype=None, commit=True, parent_check=True, u_dtype=None):
    d = to_device(w, "cuda")
    odt = {"f32": torch.float32, "bf16": torch.bfloat16}[out_dtype or w.out_dtype]
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    out, U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                           d["node_offsets"], d["S_root"], max_nodes=w.max_nodes, mode=w.mode,
                           out_dtype=odt, workspace=ws, kernel=kernel, u_dtype=u_dtype)
    S_new = None
    if commit:
        S_new = L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                              d["accepted_path"], max_nodes=w.max_nodes,
                              parent=d["parent"] if parent_check else None, workspace=ws)
    st = L.get_status(ws)
    assert st == 0, L.binding.status_string(st)
    res = {"o": out.float().cpu().numpy().astype(np.float64),
           "U": U.float().cpu().numpy().astype(np.float64)}
    if commit:
        res["S_new"] = S_new.cpu().numpy().astype(np.float64)
    return res, d


def assert_close(got, want, tol, what):
    want = np.asarray(want, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(want ** 2))) if want.size else 0.0
    err = float(np.max(np.abs(got - want))) if want.size else 0.0
    assert err <= tol * rms, f"{what}: max|err| {err:.3e} > {tol:g} * RMS {rms:.3e}"
    return err / rms if rms else 0.0
