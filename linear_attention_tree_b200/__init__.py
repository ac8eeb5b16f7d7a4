"""B200 (sm_100a) draft-tree verification through a recurrent linear-attention layer.

`tree_verify` gives every node of a speculative draft tree the output the sequential
scalar-decay or gated-delta recurrence would produce along its root-to-node path, without
per-node state snapshots, and writes one pseudo-value row per node; `tree_commit` rebuilds
the accepted path's state from those pseudo-values.  Both are CUDA kernels behind the C
ABI of ``include/tree_verify.h``; this package is the Python binding over it.
"""
from .binding import (TreeVerifyError, get_status, lib, make_problem, new_workspace,
                      snapshot_commit, snapshot_verify, tree_commit, tree_commit_verify,
                      tree_meta, tree_verify, workspace_size)

__all__ = ["tree_verify", "tree_commit", "tree_commit_verify", "snapshot_verify",
           "snapshot_commit", "tree_meta", "get_status", "workspace_size",
           "new_workspace", "make_problem", "lib", "TreeVerifyError"]
