"""Thin ctypes binding over the C ABI in ``include/tree_verify.h``.

Argument marshalling only: tensors are checked for device, dtype, shape, contiguity and
alignment, their raw pointers and torch's current CUDA stream are passed to the ``tv_*``
entry points, and a non-OK status raises `TreeVerifyError`.  Every step of the method runs
in the library's CUDA kernels; there is no CPU fallback, and a missing library raises.

Python name  -> C entry point
  tree_verify     tv_tree_verify
  tree_commit     tv_tree_commit
  tree_meta       tv_tree_meta
  tree_commit_verify tv_tree_commit_verify
  snapshot_verify tv_snapshot_verify    (the per-node-snapshot baseline)
  snapshot_commit tv_snapshot_commit
  workspace_size  tv_workspace_size
  get_status      tv_get_status
  selftest_timeout tv_selftest_timeout
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtreeverify.so")

TV_OK, TV_ERR_INVALID_ARG, TV_ERR_UNSUPPORTED, TV_ERR_BAD_TREE, TV_ERR_BAD_PATH, \
    TV_ERR_CUDA, TV_ERR_TIMEOUT = range(7)
MODE = {"gdn": 0, "scalar": 1}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
KERNEL = {"auto": 0, "tc": 1, "simt": 2}
EXPORTS = ("tv_workspace_size", "tv_tree_verify", "tv_tree_commit", "tv_tree_meta",
           "tv_tree_commit_verify", "tv_snapshot_verify", "tv_snapshot_commit",
           "tv_get_status", "tv_status_string", "tv_last_cuda_error", "tv_version",
           "tv_selftest_timeout")


class TreeVerifyError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = ""
        if status == TV_ERR_CUDA:
            detail = " [" + lib().tv_last_cuda_error().decode() + "]"
        super().__init__(f"{what}: {status_string(status)} (status {status}){detail}")


class Problem(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "dk", "dv", "total_nodes", "max_nodes", "max_path", "mode",
                 "in_dtype", "out_dtype", "kernel", "u_dtype", "qk_heads")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m linear_attention_tree_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32p = ctypes.c_void_p, ctypes.c_void_p
        P = ctypes.POINTER(Problem)
        L.tv_workspace_size.argtypes = [P]
        L.tv_workspace_size.restype = ctypes.c_size_t
        L.tv_tree_verify.argtypes = [P] + [vp] * 11 + [ctypes.c_size_t, vp]
        L.tv_tree_verify.restype = ctypes.c_int
        L.tv_tree_commit.argtypes = [P] + [vp] * 9 + [ctypes.c_size_t, vp]
        L.tv_tree_commit.restype = ctypes.c_int
        L.tv_tree_meta.argtypes = [P] + [vp] * 7 + [ctypes.c_size_t, vp]
        L.tv_tree_commit_verify.argtypes = [P] + [vp] * 8 + [P] + [vp] * 10 + [ctypes.c_size_t, vp]
        L.tv_tree_commit_verify.restype = ctypes.c_int
        L.tv_snapshot_verify.argtypes = [P] + [vp] * 12 + [ctypes.c_size_t, vp]
        L.tv_snapshot_verify.restype = ctypes.c_int
        L.tv_snapshot_commit.argtypes = [P] + [vp] * 7 + [ctypes.c_size_t, vp]
        L.tv_snapshot_commit.restype = ctypes.c_int
        L.tv_tree_meta.restype = ctypes.c_int
        L.tv_get_status.argtypes = [vp, vp]
        L.tv_get_status.restype = ctypes.c_int
        L.tv_selftest_timeout.argtypes = [vp, ctypes.c_size_t, vp]
        L.tv_selftest_timeout.restype = ctypes.c_int
        L.tv_status_string.argtypes = [ctypes.c_int]
        L.tv_status_string.restype = ctypes.c_char_p
        L.tv_last_cuda_error.argtypes = []
        L.tv_last_cuda_error.restype = ctypes.c_char_p
        L.tv_version.argtypes = []
        L.tv_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tv_status_string(int(status)).decode()


def make_problem(B, H, dk, dv, total_nodes, max_nodes, max_path=1, mode="gdn",
                 in_dtype=torch.bfloat16, out_dtype=None, kernel="auto",
                 u_dtype=torch.float32, qk_heads=0) -> Problem:
    """``qk_heads``: number of q / k heads (0 = H); ``u_dtype``: storage type of U."""
    return Problem(int(B), int(H), int(dk), int(dv), int(total_nodes), int(max_nodes),
                   int(max_path), MODE[mode], DTYPE[in_dtype],
                   DTYPE[out_dtype if out_dtype is not None else in_dtype], KERNEL[kernel],
                   DTYPE[u_dtype], int(qk_heads))


def workspace_size(problem: Problem) -> int:
    return int(lib().tv_workspace_size(ctypes.byref(problem)))


def new_workspace(problem: Problem, device=None) -> torch.Tensor:
    """Zero-filled device workspace for ``problem`` (the status word starts clear)."""
    n = workspace_size(problem)
    if n == 0:
        raise TreeVerifyError(TV_ERR_INVALID_ARG, "workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda" or (device is not None and t.device != device):
        raise ValueError(f"{name} must live on the CUDA device of the call")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != TV_OK:
        raise TreeVerifyError(status, what)


def tree_verify(q, k, v, log_a, b, parent, node_offsets, S_root, *, max_nodes: int,
                mode: str = "gdn", out=None, U=None, out_dtype=None, workspace=None,
                kernel: str = "auto", u_dtype=None, stream=None):
    """Verify every node of every draft tree; returns (out, U).

    q, k [T][Hk][dk] (Hk q / k heads shared by H / Hk value heads each, Hk = H by default);
    v [T][H][dv] (fp32 or bf16); log_a, b [T][H] fp32 (b may be None in scalar mode);
    parent [T], node_offsets [B+1] int32; S_root [B][H][dv][dk] fp32.  out [T][H][dv]
    (out_dtype, default the input dtype) and U [T][H][dv] (u_dtype, default fp32, or the
    dtype of the U given) are allocated when not given.  ``max_nodes`` bounds every
    sequence's node count (<= 256).
    """
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    B = node_offsets.shape[0] - 1
    dev = q.device
    out_dtype = out_dtype or q.dtype
    if out is None:
        out = torch.empty((T, H, dv), dtype=out_dtype, device=dev)
    if U is None:
        U = torch.empty((T, H, dv), dtype=u_dtype or torch.float32, device=dev)
    prob = make_problem(B, H, dk, dv, T, max_nodes, 1, mode, q.dtype, out.dtype, kernel,
                        U.dtype, 0 if Hk == H else Hk)
    if workspace is None:
        workspace = new_workspace(prob, dev)
    fdt = torch.float32
    args = [
        _ptr(q, "q", (torch.float32, torch.bfloat16), (T, Hk, dk), dev),
        _ptr(k, "k", q.dtype, (T, Hk, dk), dev),
        _ptr(v, "v", q.dtype, (T, H, dv), dev),
        _ptr(log_a, "log_a", fdt, (T, H), dev),
        _ptr(b, "b", fdt, (T, H), dev),
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(S_root, "S_root", fdt, (B, H, dv, dk), dev),
        _ptr(out, "out", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(U, "U", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    st = lib().tv_tree_verify(ctypes.byref(prob), *args, ctypes.c_size_t(workspace.numel()),
                              _stream(stream))
    _check(st, "tv_tree_verify")
    return out, U


def tree_commit(U, k, log_a, S_root, node_offsets, accepted_path, *, max_nodes: int,
                parent=None, S_new=None, workspace=None, stream=None):
    """Rebuild every sequence's accepted state; returns S_new [B][H][dv][dk] fp32.

    ``S_new`` may be ``S_root`` itself (in-place commit).  accepted_path is [B][max_path]
    int32, root-first, -1 padded.  With ``parent`` every path is checked against its tree.
    """
    T, H, dv = U.shape
    Hk, dk = k.shape[1], k.shape[2]
    B = node_offsets.shape[0] - 1
    dev = U.device
    if S_new is None:
        S_new = torch.empty_like(S_root)
    max_path = accepted_path.shape[1] if accepted_path.dim() == 2 else 0
    prob = make_problem(B, H, dk, dv, T, max_nodes, max_path, "gdn", k.dtype, k.dtype,
                        u_dtype=U.dtype, qk_heads=0 if Hk == H else Hk)
    if workspace is None:
        workspace = new_workspace(prob, dev)
    fdt = torch.float32
    args = [
        _ptr(U, "U", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(k, "k", (torch.float32, torch.bfloat16), (T, Hk, dk), dev),
        _ptr(log_a, "log_a", fdt, (T, H), dev),
        _ptr(S_root, "S_root", fdt, (B, H, dv, dk), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(accepted_path, "accepted_path", torch.int32, (B, max_path), dev),
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(S_new, "S_new", fdt, (B, H, dv, dk), dev),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    st = lib().tv_tree_commit(ctypes.byref(prob), *args, ctypes.c_size_t(workspace.numel()),
                              _stream(stream))
    _check(st, "tv_tree_commit")
    return S_new


def tree_commit_verify(U_prev, k_prev, log_a_prev, node_offsets_prev, accepted_path, S_root,
                       q, k, v, log_a, b, parent, node_offsets, *, max_nodes_prev: int,
                       max_nodes: int, parent_prev=None, S_new=None, out=None, U=None,
                       mode: str = "gdn", out_dtype=None, workspace=None, kernel: str = "auto",
                       stream=None):
    """The previous step's commit and the next tree's verify against the committed state;
    returns (S_new, out, U).  ``S_new`` may be ``S_root`` (in place); ``U`` must not be
    ``U_prev``.  Argument meanings as in `tree_commit` (previous tree) and `tree_verify`
    (next tree)."""
    Tp, H, dv = U_prev.shape
    Hk, dk = k_prev.shape[1], k_prev.shape[2]
    B = node_offsets.shape[0] - 1
    T = q.shape[0]
    dev = q.device
    out_dtype = out_dtype or q.dtype
    if S_new is None:
        S_new = torch.empty_like(S_root)
    if out is None:
        out = torch.empty((T, H, dv), dtype=out_dtype, device=dev)
    if U is None:
        U = torch.empty((T, H, dv), dtype=U_prev.dtype, device=dev)
    max_path = accepted_path.shape[1]
    qkh = 0 if Hk == H else Hk
    prev = make_problem(B, H, dk, dv, Tp, max_nodes_prev, max_path, mode, k_prev.dtype,
                        k_prev.dtype, u_dtype=U_prev.dtype, qk_heads=qkh)
    nxt = make_problem(B, H, dk, dv, T, max_nodes, 1, mode, q.dtype, out.dtype, kernel,
                       U.dtype, qkh)
    if workspace is None:
        workspace = new_workspace(nxt, dev)
    fdt = torch.float32
    args = [
        _ptr(U_prev, "U_prev", (torch.float32, torch.bfloat16), (Tp, H, dv), dev),
        _ptr(k_prev, "k_prev", (torch.float32, torch.bfloat16), (Tp, Hk, dk), dev),
        _ptr(log_a_prev, "log_a_prev", fdt, (Tp, H), dev),
        _ptr(node_offsets_prev, "node_offsets_prev", torch.int32, (B + 1,), dev),
        _ptr(accepted_path, "accepted_path", torch.int32, (B, max_path), dev),
        _ptr(parent_prev, "parent_prev", torch.int32, (Tp,), dev),
        _ptr(S_root, "S_root", fdt, (B, H, dv, dk), dev),
        _ptr(S_new, "S_new", fdt, (B, H, dv, dk), dev),
    ]
    args2 = [
        _ptr(q, "q", (torch.float32, torch.bfloat16), (T, Hk, dk), dev),
        _ptr(k, "k", q.dtype, (T, Hk, dk), dev),
        _ptr(v, "v", q.dtype, (T, H, dv), dev),
        _ptr(log_a, "log_a", fdt, (T, H), dev),
        _ptr(b, "b", fdt, (T, H), dev),
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(out, "out", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(U, "U", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    st = lib().tv_tree_commit_verify(ctypes.byref(prev), *args, ctypes.byref(nxt), *args2,
                                     ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(st, "tv_tree_commit_verify")
    return S_new, out, U


def snapshot_verify(q, k, v, log_a, b, parent, node_offsets, S_root, *, max_nodes: int,
                    mode: str = "gdn", snapshots=None, out=None, U=None, out_dtype=None,
                    workspace=None, stream=None):
    """The per-node-snapshot baseline; returns (out, U, snapshots [T][H][dv][dk] fp32)."""
    T, Hk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    B = node_offsets.shape[0] - 1
    dev = q.device
    out_dtype = out_dtype or q.dtype
    if out is None:
        out = torch.empty((T, H, dv), dtype=out_dtype, device=dev)
    if U is None:
        U = torch.empty((T, H, dv), dtype=torch.float32, device=dev)
    if snapshots is None:
        snapshots = torch.empty((T, H, dv, dk), dtype=torch.float32, device=dev)
    prob = make_problem(B, H, dk, dv, T, max_nodes, 1, mode, q.dtype, out.dtype,
                        u_dtype=U.dtype, qk_heads=0 if Hk == H else Hk)
    if workspace is None:
        workspace = new_workspace(prob, dev)
    fdt = torch.float32
    args = [
        _ptr(q, "q", (torch.float32, torch.bfloat16), (T, Hk, dk), dev),
        _ptr(k, "k", q.dtype, (T, Hk, dk), dev), _ptr(v, "v", q.dtype, (T, H, dv), dev),
        _ptr(log_a, "log_a", fdt, (T, H), dev), _ptr(b, "b", fdt, (T, H), dev),
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(S_root, "S_root", fdt, (B, H, dv, dk), dev),
        _ptr(out, "out", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(U, "U", (torch.float32, torch.bfloat16), (T, H, dv), dev),
        _ptr(snapshots, "snapshots", fdt, (T, H, dv, dk), dev),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    _check(lib().tv_snapshot_verify(ctypes.byref(prob), *args, ctypes.c_size_t(workspace.numel()),
                                    _stream(stream)), "tv_snapshot_verify")
    return out, U, snapshots


def snapshot_commit(snapshots, S_root, node_offsets, accepted_path, *, max_nodes: int,
                    parent=None, S_new=None, workspace=None, stream=None):
    """The baseline's commit: S_new = the snapshot of each accepted path's last node."""
    T, H, dv, dk = snapshots.shape
    B = node_offsets.shape[0] - 1
    dev = snapshots.device
    if S_new is None:
        S_new = torch.empty_like(S_root)
    max_path = accepted_path.shape[1]
    prob = make_problem(B, H, dk, dv, T, max_nodes, max_path)
    if workspace is None:
        workspace = new_workspace(prob, dev)
    fdt = torch.float32
    args = [
        _ptr(snapshots, "snapshots", fdt, (T, H, dv, dk), dev),
        _ptr(S_root, "S_root", fdt, (B, H, dv, dk), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(accepted_path, "accepted_path", torch.int32, (B, max_path), dev),
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(S_new, "S_new", fdt, (B, H, dv, dk), dev),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    _check(lib().tv_snapshot_commit(ctypes.byref(prob), *args, ctypes.c_size_t(workspace.numel()),
                                    _stream(stream)), "tv_snapshot_commit")
    return S_new


def tree_meta(parent, node_offsets, log_a, *, max_nodes: int, workspace=None, stream=None):
    """(depth [T] int32, anc [T][ceil(max_nodes/64)] int64 bit patterns, cumlog [T][H] fp32)."""
    T, H = log_a.shape
    B = node_offsets.shape[0] - 1
    dev = log_a.device
    W = (max_nodes + 63) // 64
    depth = torch.empty(T, dtype=torch.int32, device=dev)
    anc = torch.empty((T, W), dtype=torch.int64, device=dev)
    cumlog = torch.empty((T, H), dtype=torch.float32, device=dev)
    prob = make_problem(B, H, 16, 16, T, max_nodes, 1, "gdn", torch.float32)
    if workspace is None:
        workspace = new_workspace(prob, dev)
    args = [
        _ptr(parent, "parent", torch.int32, (T,), dev),
        _ptr(node_offsets, "node_offsets", torch.int32, (B + 1,), dev),
        _ptr(log_a, "log_a", torch.float32, (T, H), dev),
        _ptr(depth, "depth"), _ptr(anc, "anc"), _ptr(cumlog, "cumlog"),
        _ptr(workspace, "workspace", torch.uint8, None, dev),
    ]
    st = lib().tv_tree_meta(ctypes.byref(prob), *args, ctypes.c_size_t(workspace.numel()),
                            _stream(stream))
    _check(st, "tv_tree_meta")
    return depth, anc, cumlog


def selftest_timeout(workspace: torch.Tensor, stream=None) -> None:
    """Enqueue the library's time-out diagnostic: a bounded wait that runs out records
    TV_ERR_TIMEOUT in ``workspace`` (read it with `get_status`)."""
    _check(lib().tv_selftest_timeout(_ptr(workspace, "workspace", torch.uint8),
                                     workspace.numel(), _stream(stream)), "selftest_timeout")


def get_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream; return and clear the device-side status of ``workspace``."""
    return int(lib().tv_get_status(_ptr(workspace, "workspace", torch.uint8), _stream(stream)))
