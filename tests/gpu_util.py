"""Helpers for the GPU parity tests: upload a seeded workload, call the C ABI through the
binding, compare with the oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from workloads import to_float64
from workloads.device import torch_to_np, upload_projection

DT = {"bf16": L.LORA_BF16, "f32": L.LORA_F32}


def tolerance(ref: np.ndarray) -> float:
    """|gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element, max over the call's output."""
    return 1e-2 * float(np.abs(ref).max()) + 1e-3


def assert_close(y_gpu, ref: np.ndarray, dtype: str, what: str = "") -> float:
    got = to_float64(y_gpu, dtype)
    bound = tolerance(ref)
    err = np.abs(got - ref)
    worst = float(err.max()) if err.size else 0.0
    if not worst <= bound:
        i = np.unravel_index(int(np.argmax(err)), err.shape)
        raise AssertionError("%s: max |gpu-ref| = %.3g > %.3g at %s (gpu %r, ref %r)"
                             % (what, worst, bound, i, got[i], ref[i]))
    return worst


class option:
    """Set a runtime option of the library for the duration of a with-block."""

    def __init__(self, key: str, value: int):
        self.key, self.value = key, value

    def __enter__(self):
        self.old = L.lora_get_option(self.key)
        L.lora_set_option(self.key, self.value)
        return self

    def __exit__(self, *exc):
        L.lora_set_option(self.key, self.old)
        return False


@functools.lru_cache(maxsize=8)
def workload(name: str, delta_only: bool = False, reading: str = "variance", **kw):
    return workloads.generate(name, delta_only=delta_only, reading=reading, **kw)


@functools.lru_cache(maxsize=16)
def reference(name: str, delta_only: bool = False, reading: str = "variance", proj: int = 0):
    wl = workload(name, delta_only, reading)
    return oracle.workload_reference(wl, proj)


class DeviceProj:
    """One projection of a workload on the device with its adapter table."""

    def __init__(self, wl, pi: int = 0):
        self.wl = wl
        self.p = wl.projections[pi]
        self.dtype = wl.dtype
        self.d = upload_projection(self.p, wl.dtype)
        self.table = L.AdapterTable(self.d.A_ptrs, self.d.B_ptrs, self.d.ranks, self.d.scales,
                                    self.p.h, self.p.o, DT[wl.dtype], keep=self.d)
        self.ids = torch.from_numpy(np.ascontiguousarray(wl.ids)).cuda()
        self.T = wl.T

    def y(self) -> torch.Tensor:
        return self.d.y0.clone()

    def workspace(self) -> torch.Tensor:
        return torch.empty(self.table.workspace_bytes(self.T), dtype=torch.uint8, device="cuda")

    def segments(self, ids: torch.Tensor = None, max_seg_len: int = 0):
        ids = self.ids if ids is None else ids
        T = ids.numel()
        n = self.table.n
        t = dict(perm=torch.empty(max(T, 1), dtype=torch.int32, device="cuda"),
                 seg_ptr=torch.empty(n + 1, dtype=torch.int32, device="cuda"),
                 seg_adapter=torch.empty(n, dtype=torch.int32, device="cuda"),
                 num_segs=torch.empty(1, dtype=torch.int32, device="cuda"))
        L.lora_build_segments(self.table.handle, ids, T, t["perm"], t["seg_ptr"], t["seg_adapter"], t["num_segs"])
        seg = L.make_segments(t["perm"], t["seg_ptr"], t["seg_adapter"], t["num_segs"], T, n, max_seg_len)
        return seg, t

    def sgmv(self, y, seg, x=None):
        ws = self.workspace()
        x = self.d.x if x is None else x
        L.lora_sgmv(self.table.handle, seg, x, x.shape[1], y, y.shape[1], 0, ws, ws.numel())
        return y

    def bgmv(self, y, ids=None, x=None):
        ids = self.ids if ids is None else ids
        x = self.d.x if x is None else x
        ws = self.workspace()
        L.lora_bgmv(self.table.handle, ids, ids.numel(), x, x.shape[1], y, y.shape[1], 0, ws, ws.numel())
        return y

    def status(self):
        return L.lora_get_status(self.table.handle, reset=True)

    def to_np(self, y):
        torch.cuda.synchronize()
        return torch_to_np(y, self.dtype)


def kernels_launched(fn) -> set:
    """Names of the library's kernels that fn() launched, from the library's own launch
    counters (lora_kernel_launches: launches the CUDA runtime accepted).  The call's results are
    checked against the oracle separately; this says which path the dispatcher took.  (The torch
    profiler was tried first: late in a long process it recorded only the last of several
    launches, or none.)"""
    before = L.kernel_launches()
    fn()
    torch.cuda.synchronize()
    after = L.kernel_launches()
    return {k for k in after if after[k] > before[k]}


def ran(names: set, kernel: str) -> bool:
    return any(kernel in k for k in names)
