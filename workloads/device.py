"""Device copies of seeded inputs (torch tensors).  Storage conversion only: float arrays that hold
bf16 values are copied as their exact bf16 bit patterns."""
from __future__ import annotations

import numpy as np
import torch

from . import to_bf16_bits


def tensor(a, dtype: str, device) -> torch.Tensor | None:
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype.kind in "iu" and a.dtype != np.uint16:
        return torch.from_numpy(a.astype(np.int64)).to(device)
    if dtype == "bf16":
        bits = a if a.dtype == np.uint16 else to_bf16_bits(a.astype(np.float32))
        return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a.astype(np.float32)).to(device)


def to_device(inp, device) -> dict:
    """All tensors of a `workloads.Inputs` on `device` (X and parameters in the workload's dtype,
    bias tables fp32, offsets/timestamps int64)."""
    dt = inp.workload.dtype
    layers = [{k: tensor(getattr(p, k), dt, device) for k in ("W1", "b1", "W2", "b2", "ln_w", "ln_b")}
              for p in inp.layers]
    return {"X": tensor(inp.X, dt, device), "off": tensor(inp.seq_offsets, dt, device),
            "ts": tensor(inp.timestamps, dt, device), "pos": tensor(inp.pos_table, "f32", device),
            "tim": tensor(inp.time_table, "f32", device),
            "ali": tensor(inp.alibi_slopes, "f32", device), "layers": layers}
