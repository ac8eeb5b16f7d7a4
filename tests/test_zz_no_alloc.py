"""tv_tree_verify_noalloc: verification without any device allocation by the library.

Callers that cannot allocate at verification time (allocator callbacks, serving loops
with allocation frozen after start-up, hosts that only lend their own buffers) use this
entry point; it keeps its scratch in a fixed device array inside the library.  Its
results must equal tv_tree_verify's on the same inputs, call after call.  This file is
collected last so that a failure here does not hide the other tests' results.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import workloads as W
from linear_attention_tree_b200.tensors import to_device
from tests._gpu_util import TOL, assert_close

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = L.lib().tv_tree_verify_noalloc
    fn.argtypes = [ctypes.c_void_p] * 11 + [ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


@pytest.mark.parametrize("idx,kernel", [(3, "auto"), (2, "simt")])
def test_noalloc_matches_tree_verify_twice(idx, kernel):
    w = W.config(idx)
    d = to_device(w)
    ref_out, ref_U = L.tree_verify(d["q"], d["k"], d["v"], d["log_a"], d["b"], d["parent"],
                                   d["node_offsets"], d["S_root"], max_nodes=w.max_nodes,
                                   out_dtype=torch.float32, kernel=kernel)
    prob = L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, 1, w.mode, torch.bfloat16,
                          torch.float32, kernel)
    fn = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        U = torch.full_like(ref_U, float("nan"))
        scratch = ctypes.c_void_p()
        torch.cuda.synchronize()
        free_before, _ = torch.cuda.mem_get_info()
        torch.cuda.reset_peak_memory_stats()
        allocated = torch.cuda.memory_allocated()
        st = fn(ctypes.byref(prob), d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(),
                d["log_a"].data_ptr(), d["b"].data_ptr(), d["parent"].data_ptr(),
                d["node_offsets"].data_ptr(), d["S_root"].data_ptr(), out.data_ptr(),
                U.data_ptr(), ctypes.byref(scratch), stream)
        torch.cuda.synchronize()
        assert st == 0, L.binding.status_string(st)
        if call == 1:
            # the call itself allocates nothing: neither through torch's allocator nor
            # anywhere else on the device (the first call may load the module image)
            assert torch.cuda.max_memory_allocated() == allocated
            free_after, _ = torch.cuda.mem_get_info()
            assert free_before - free_after < 2 << 20, (free_before, free_after)
        assert scratch.value, "the static scratch address is reported"
        assert L.lib().tv_get_status(scratch, stream) == 0
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy(), ref_out.cpu().numpy(), TOL["bf16"], f"o call {call}")
        assert_close(U.cpu().numpy(), ref_U.cpu().numpy(), TOL["bf16"], f"U call {call}")
        # the same kernel on the same inputs is deterministic: outputs match bit for bit
        torch.testing.assert_close(out, ref_out, rtol=0, atol=0)
        torch.testing.assert_close(U, ref_U, rtol=0, atol=0)


def test_noalloc_reports_device_errors_through_the_returned_scratch():
    w = W.config(2)
    d = to_device(w)
    d["parent"][3] = 9                     # not topological
    prob = L.make_problem(w.B, w.H, w.dk, w.dv, w.T, w.max_nodes, 1, w.mode, torch.bfloat16,
                          torch.float32)
    out = torch.empty((w.T, w.H, w.dv), dtype=torch.float32, device="cuda")
    U = torch.empty_like(out)
    scratch = ctypes.c_void_p()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _noalloc_fn()(ctypes.byref(prob), d["q"].data_ptr(), d["k"].data_ptr(),
                       d["v"].data_ptr(), d["log_a"].data_ptr(), d["b"].data_ptr(),
                       d["parent"].data_ptr(), d["node_offsets"].data_ptr(),
                       d["S_root"].data_ptr(), out.data_ptr(), U.data_ptr(),
                       ctypes.byref(scratch), stream)
    assert st == 0
    assert L.lib().tv_get_status(scratch, stream) == L.binding.TV_ERR_BAD_TREE
    assert L.lib().tv_get_status(scratch, stream) == 0
