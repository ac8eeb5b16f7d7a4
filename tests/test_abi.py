"""The C-ABI library builds, loads without a GPU, exports what the header declares, and
rejects bad arguments synchronously (before any CUDA call)."""
import ctypes
import os
import re

import pytest

import linear_attention_tree_b200 as L
from linear_attention_tree_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"TV_API\s+[\w\s\*]*?\b(tv_\w+)\s*\(", text))
    return names


def test_library_builds_and_loads():
    path = build.build()
    assert os.path.exists(path)
    assert L.lib()._name == binding.LIB_PATH


def test_exports_every_declared_symbol():
    names = _declared()
    assert {"tv_tree_verify", "tv_tree_commit", "tv_tree_meta", "tv_workspace_size",
            "tv_get_status"} <= names
    for n in names:
        assert hasattr(L.lib(), n), n
    assert set(binding.EXPORTS) <= names


def test_problem_layout_and_version():
    assert ctypes.sizeof(binding.Problem) == 52      # 13 int32 fields
    assert L.lib().tv_version() >> 16 == 2
    assert binding.status_string(0) == "ok"


def _call_verify(prob, ptrs):
    return L.lib().tv_tree_verify(ctypes.byref(prob), *ptrs, ctypes.c_size_t(256), None)


def _fake(n=11, misalign=None):
    # fake device addresses: the call must fail before dereferencing anything
    ptrs = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(n)]
    if misalign is not None:
        ptrs[misalign] = ctypes.c_void_p(0x10000 * (misalign + 1) + 4)
    return ptrs


@pytest.mark.parametrize("field,value,expect", [
    ("H", 0, binding.TV_ERR_INVALID_ARG), ("B", -1, binding.TV_ERR_INVALID_ARG),
    ("dk", 100, binding.TV_ERR_UNSUPPORTED), ("dv", 256, binding.TV_ERR_UNSUPPORTED),
    ("max_nodes", 257, binding.TV_ERR_UNSUPPORTED), ("max_nodes", 0, binding.TV_ERR_INVALID_ARG),
    ("mode", 7, binding.TV_ERR_INVALID_ARG), ("in_dtype", 5, binding.TV_ERR_INVALID_ARG),
    ("kernel", 9, binding.TV_ERR_INVALID_ARG), ("total_nodes", 999999, binding.TV_ERR_INVALID_ARG),
])
def test_bad_problem_rejected(field, value, expect):
    prob = L.make_problem(4, 2, 128, 128, 64, 16, 4)
    setattr(prob, field, value)
    assert _call_verify(prob, _fake()) == expect
    if expect == binding.TV_ERR_INVALID_ARG or expect == binding.TV_ERR_UNSUPPORTED:
        assert L.workspace_size(prob) == 0


def test_null_and_misaligned_pointers_rejected():
    prob = L.make_problem(4, 2, 128, 128, 64, 16, 4)
    for i in range(11):
        ptrs = _fake()
        ptrs[i] = None
        assert _call_verify(prob, ptrs) == binding.TV_ERR_INVALID_ARG, i
        assert _call_verify(prob, _fake(misalign=i)) == binding.TV_ERR_INVALID_ARG, i
    # workspace too small
    assert L.lib().tv_tree_verify(ctypes.byref(prob), *_fake(), ctypes.c_size_t(8), None) == \
        binding.TV_ERR_INVALID_ARG


def test_tc_kernel_refuses_unsupported_shapes():
    prob = L.make_problem(4, 2, 64, 128, 64, 16, 4, kernel="tc")
    assert _call_verify(prob, _fake()) == binding.TV_ERR_UNSUPPORTED
    prob = L.make_problem(4, 2, 128, 128, 64, 16, 4, in_dtype=__import__("torch").float32,
                          kernel="tc")
    assert _call_verify(prob, _fake()) == binding.TV_ERR_UNSUPPORTED


def test_commit_rejects_partial_overlap():
    prob = L.make_problem(2, 2, 16, 16, 8, 4, 3)
    state = 2 * 2 * 16 * 16 * 4
    ptrs = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(9)]
    ptrs[7] = ctypes.c_void_p(ptrs[3].value + 256)     # S_new overlaps S_root, not equal
    assert L.lib().tv_tree_commit(ctypes.byref(prob), *ptrs, ctypes.c_size_t(256), None) == \
        binding.TV_ERR_INVALID_ARG
    prob.max_path = 0
    assert L.lib().tv_tree_commit(ctypes.byref(prob), *ptrs, ctypes.c_size_t(256), None) == \
        binding.TV_ERR_INVALID_ARG


def test_product_path_has_no_cpu_fallback():
    """The package never imports the oracle, and its functions need the CUDA library."""
    import linear_attention_tree_b200.binding as b
    pkg = os.path.dirname(b.__file__)
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            assert "import oracle" not in open(os.path.join(pkg, fn)).read()
            assert "from oracle" not in open(os.path.join(pkg, fn)).read()


def test_workspace_is_constant_size():
    """The workspace holds only the status word: its size does not grow with the number of
    nodes, heads or the state size (there are no per-node state snapshots anywhere)."""
    small = L.workspace_size(L.make_problem(1, 1, 16, 16, 6, 6, 3))
    big = L.workspace_size(L.make_problem(128, 32, 128, 128, 3072, 48, 7))
    wide = L.workspace_size(L.make_problem(8, 32, 128, 128, 2048, 256, 11))
    assert 0 < small == big == wide <= 4096


def test_selftest_rejects_bad_workspace_before_launching():
    f = L.lib().tv_selftest_timeout
    assert f(None, 256, None) == binding.TV_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(0x10004), 256, None) == binding.TV_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(0x10000), 8, None) == binding.TV_ERR_INVALID_ARG


def test_commit_verify_checks_its_arguments():
    """Shapes that differ between the two steps, and new pseudo-values over the previous
    ones, are refused before anything is enqueued."""
    import torch
    fn = L.lib().tv_tree_commit_verify
    ptr = lambda i: ctypes.c_void_p(0x100000 * (i + 1))
    prev = L.make_problem(2, 2, 128, 128, 8, 4, 3)
    nxt = L.make_problem(2, 2, 128, 128, 8, 4, 1)
    # prev, U_prev, 7 more previous-step pointers, next, q..node_offsets (7), out, U, workspace
    args = lambda U_prev, U: [ctypes.byref(prev), U_prev] + [ptr(i) for i in range(1, 8)] + \
        [ctypes.byref(nxt)] + [ptr(i) for i in range(8, 15)] + [ptr(15), U, ptr(18),
                                                               ctypes.c_size_t(256), None]
    # U (8 nodes x 2 heads x 128 fp32 = 8 KiB) starting inside U_prev
    assert fn(*args(ptr(0), ctypes.c_void_p(0x100000 + 4096))) == binding.TV_ERR_INVALID_ARG
    other = L.make_problem(3, 2, 128, 128, 8, 4, 1)
    assert fn(ctypes.byref(prev), ptr(0), *[ptr(i) for i in range(1, 8)], ctypes.byref(other),
              *[ptr(i) for i in range(8, 15)], ptr(15), ptr(17), ptr(18), ctypes.c_size_t(256),
              None) == binding.TV_ERR_INVALID_ARG


def test_grouped_heads_and_u_dtype_are_checked():
    """qk_heads must divide H; bf16 U is refused by the CUDA-core kernel, which reads U back."""
    import torch
    for qk in (-1, 3, 5):
        prob = L.make_problem(4, 4, 128, 128, 64, 16, 4, qk_heads=qk)
        assert _call_verify(prob, _fake()) == binding.TV_ERR_INVALID_ARG, qk
    prob = L.make_problem(4, 4, 64, 64, 64, 16, 4, u_dtype=torch.bfloat16)
    assert _call_verify(prob, _fake()) == binding.TV_ERR_UNSUPPORTED
    prob = L.make_problem(4, 4, 128, 128, 64, 16, 4, u_dtype=torch.bfloat16, kernel="simt")
    assert _call_verify(prob, _fake()) == binding.TV_ERR_UNSUPPORTED
