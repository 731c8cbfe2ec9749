"""Shared helpers for the GPU parity tests (marshalling only)."""
from __future__ import annotations

import numpy as np
import torch

FMTS = ["e4m3", "e5m2", "e2m3", "e3m2", "e2m1", "int8"]


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_device(x: np.ndarray) -> torch.Tensor:
    """float32 array -> fp32 tensor; uint16 array (bf16 bits) -> bf16 tensor."""
    if x.dtype == np.uint16:
        t = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(dev())


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def first_mismatch(a: np.ndarray, b: np.ndarray, n: int = 8):
    idx = np.argwhere(a != b)
    return [(tuple(int(v) for v in i), int(a[tuple(i)]), int(b[tuple(i)])) for i in idx[:n]]
