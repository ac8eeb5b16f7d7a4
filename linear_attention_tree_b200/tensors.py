"""Host <-> device marshalling of a `Workload` (no arithmetic of the method)."""
from __future__ import annotations

import numpy as np
import torch

from .workloads import Workload, bf16_bits


def _in_tensor(x: np.ndarray, in_dtype: str, device) -> torch.Tensor:
    if in_dtype == "bf16":
        return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_device(w: Workload, device="cuda", pin: bool = False) -> dict:
    """Tensors of one workload on ``device`` (or pinned host memory when ``device='cpu'``
    and ``pin``): q, k, v, log_a, b, parent, node_offsets, S_root, accepted_path."""
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32))
    host = {
        "q": _in_tensor(w.q, w.in_dtype, "cpu"), "k": _in_tensor(w.k, w.in_dtype, "cpu"),
        "v": _in_tensor(w.v, w.in_dtype, "cpu"), "log_a": f32(w.log_a),
        "b": None if w.b is None else f32(w.b), "parent": i32(w.parent),
        "node_offsets": i32(w.node_offsets), "S_root": f32(w.S_root),
        "accepted_path": i32(w.accepted_path),
    }
    out = {}
    for name, t in host.items():
        if t is None:
            out[name] = None
        elif str(device) == "cpu":
            out[name] = t.pin_memory() if pin else t
        else:
            out[name] = t.to(device)
    return out


def bf16_tensor_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()
