"""Three decode steps back to back on one stream, no synchronisation between them: each
step verifies a new draft tree against the state the previous step's commit wrote in place.
The kernels may start while the previous one drains (programmatic launch), so this checks
that each step still reads the state only after the previous commit has finished.

The oracle runs the same three steps on its own results (its S_new, rounded to fp32, is
its next S_root); nothing from the CUDA path enters it."""
import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close

pytestmark = pytest.mark.gpu

STEPS = 3


def _step_workload(t):
    pars = [W.frontier_tree(700 + 10 * t + i, 64, 8, 4)[0] for i in range(6)]
    return W.synthetic(pars, H=4, dk=128, dv=128, seed=70 + t)


def test_three_steps_in_place():
    ws_ = [_step_workload(t) for t in range(STEPS)]
    devs = [to_device(w, "cuda") for w in ws_]
    S = devs[0]["S_root"].clone()                    # the running state, updated in place
    results = []
    torch.cuda.synchronize()
    for t, (w, d) in enumerate(zip(ws_, devs)):
        out, U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                               d["node_offsets"], S, max_nodes=w.max_nodes,
                               out_dtype=torch.float32)
        L.tree_commit(U, d["k"], d["log_a"], S, d["node_offsets"], d["accepted_path"],
                      max_nodes=w.max_nodes, parent=d["parent"], S_new=S)
        results.append((out, U))
    torch.cuda.synchronize()

    S_ref = ws_[0].S_root.astype(np.float32)
    for t, w in enumerate(ws_):
        w.S_root = S_ref
        o, U = O.tree_verify(w)
        assert_close(results[t][0].cpu().numpy(), o, TOL["bf16"], f"o at step {t}")
        assert_close(results[t][1].cpu().numpy(), U, TOL["bf16"], f"U at step {t}")
        S_ref = O.tree_commit(w).astype(np.float32)
    assert_close(S.cpu().numpy(), S_ref, TOL["bf16"], "state after the last step")
