"""Device-side materialisation of the synthetic workloads (inputs only).

Large memory tensors are filled on the GPU by the device generator; planted rows are then
overwritten with the host-computed planted vectors. Small per-layer tensors are generated on the
host and uploaded. Nothing here computes a step of the attention method.
"""
from __future__ import annotations

import numpy as np
import torch

from . import rng
from .workloads import Workload

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def upload(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """float32 host values (already representable in `dtype`) -> device tensor of that dtype (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device).to(TORCH_DT[dtype])


def memory_tensor(w: Workload, layer: int, name: str, device="cuda", out: torch.Tensor | None = None) -> torch.Tensor:
    """A generated memory tensor of `layer` on the device, with the planted rows written in."""
    t_id, shape, row_len = w.memory_tensors(layer)[name]
    if out is None:
        out = torch.empty(shape, dtype=TORCH_DT[w.dtype], device=device)
    rng.fill_device(out, w.seed, t_id)
    if name == w.router_tensor_name():
        plants = w.plants(layer)[0]
        if plants:
            rows = np.concatenate([p.rows for p in plants])
            vals = np.concatenate([np.broadcast_to(p.vec, (len(p.rows), row_len)) for p in plants])
            flat = out.view(shape[0], row_len)
            flat[torch.from_numpy(rows).to(device)] = upload(vals, w.dtype, device)
    return out


def small_tensors(w: Workload, layer: int, device="cuda") -> dict:
    """Per-layer Q^R, Q, new-token K and V of every token of every round, on the device."""
    return {
        "qr": upload(w.qr(layer), w.dtype, device),
        "q": upload(w.q(layer), w.dtype, device),
        "k_new": upload(w.k_new(layer), w.dtype, device),
        "v_new": upload(w.v_new(layer), w.dtype, device),
    }
