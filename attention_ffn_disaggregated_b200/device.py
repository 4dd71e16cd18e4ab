"""Move generated layer inputs into CUDA tensors in the layouts the C ABI expects."""
from __future__ import annotations

import dataclasses
from typing import List

import numpy as np
import torch


@dataclasses.dataclass
class DeviceSlab:
    x: torch.Tensor             # uint8 [cap, H]
    x_scale: torch.Tensor       # float32 [cap, H/128]
    topk_ids: torch.Tensor      # int32 [cap, K]
    topk_weights: torch.Tensor  # float32 [cap, K]
    y: torch.Tensor             # bf16 [cap, H]


def to_device_weights(inp, device="cuda"):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return t(inp.w13), t(inp.w13_scale), t(inp.w2), t(inp.w2_scale)


def to_device_slabs(inp, device="cuda", y_fill: float = float("nan")) -> List[DeviceSlab]:
    out = []
    H = inp.shape.hidden
    for s in inp.slabs:
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        y = torch.full((inp.capacity, H), y_fill, dtype=torch.bfloat16, device=device)
        out.append(DeviceSlab(t(s.x), t(s.x_scale), t(s.topk_ids), t(s.topk_weights), y))
    return out


def to_device_counts(inp, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.asarray(inp.counts, np.int32)).to(device)


def gather_outputs(inp, slabs: List[DeviceSlab]) -> np.ndarray:
    """bf16 outputs of all valid rows in slab-major token order, as uint16 bit patterns."""
    parts = [s.y[:int(n)].view(torch.int16).cpu().numpy().view(np.uint16)
             for s, n in zip(slabs, inp.counts)]
    H = inp.shape.hidden
    return np.concatenate(parts) if parts else np.zeros((0, H), np.uint16)
