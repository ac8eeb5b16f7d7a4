"""No per-node state snapshots: a verify + commit step on the 32 x 32 x 64-node workload
allocates no device memory at all beyond the caller's buffers, while one snapshot per node
and head would take T * H * dv * dk * 4 bytes (4.3 GB here)."""
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device

pytestmark = pytest.mark.gpu


def test_step_allocates_no_device_memory():
    w = W.config(3)
    d = to_device(w, "cuda")
    ws = L.new_workspace(L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, w.max_path))
    out = torch.empty((w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    U = torch.empty_like(out)
    S_new = torch.empty_like(d["S_root"])

    def step():
        L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                      d["node_offsets"], d["S_root"], max_nodes=w.max_nodes, out=out, U=U,
                      workspace=ws)
        L.tree_commit(U, d["k"], d["log_a"], d["S_root"], d["node_offsets"],
                      d["accepted_path"], max_nodes=w.max_nodes, S_new=S_new, workspace=ws)

    step()                                   # module loading and first-launch set-up
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    torch.cuda.reset_peak_memory_stats()
    allocated = torch.cuda.memory_allocated()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert L.get_status(ws) == 0
    assert torch.cuda.max_memory_allocated() == allocated
    # device-wide free memory (covers allocations outside torch too); any snapshot-like
    # buffer would be gigabytes, so a small tolerance keeps unrelated activity out of it
    assert free_before - free_after < 64 << 20
    snapshots = w.T * w.H * w.dv * w.dk * 4
    assert snapshots > 4e9 and L.workspace_size(L.make_problem(w.B, w.H, w.dk, w.dv, w.T,
                                                                w.max_nodes)) <= 4096
