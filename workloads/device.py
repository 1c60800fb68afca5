"""Move a seeded workload into device memory (torch is used only as an allocator here).

The layout on the device mirrors the host layout of :mod:`workloads`: one flat buffer of
all A_i and one of all B_i per projection (each adapter 16-byte aligned), x and y row-major.
"""
from __future__ import annotations

import dataclasses
from typing import List

import numpy as np
import torch


def np_to_torch(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def torch_to_np(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


@dataclasses.dataclass
class DeviceProjection:
    A_flat: torch.Tensor
    B_flat: torch.Tensor
    A_ptrs: List[int]
    B_ptrs: List[int]
    ranks: List[int]
    scales: List[float]
    h: int
    o: int
    x: torch.Tensor
    y0: torch.Tensor


def upload_projection(p, dtype: str, device="cuda") -> DeviceProjection:
    A = np_to_torch(p.A_flat, dtype).to(device)
    B = np_to_torch(p.B_flat, dtype).to(device)
    es = 2 if dtype == "bf16" else 4
    a0, b0 = A.data_ptr(), B.data_ptr()
    return DeviceProjection(
        A_flat=A, B_flat=B,
        A_ptrs=[a0 + int(off) * es for off in p.A_off],
        B_ptrs=[b0 + int(off) * es for off in p.B_off],
        ranks=[int(r) for r in p.ranks], scales=[float(s) for s in p.scales],
        h=p.h, o=p.o,
        x=np_to_torch(p.x, dtype).to(device), y0=np_to_torch(p.y0, dtype).to(device))
