"""Move generator arrays (numpy; bf16 as uint16 bit patterns) to torch tensors."""

from __future__ import annotations

import numpy as np
import torch


def to_torch(inputs: dict, device="cuda") -> dict:
    out = {}
    for k, v in inputs.items():
        if v.dtype == np.uint16:
            t = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(v))
        out[k] = t.to(device) if device is not None else t
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch bfloat16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
