"""Heterogeneous-batch LoRA delta (SGMV / BGMV) for B200 -- Python binding of liblora_sgmv.so.

Argument marshalling only: every function here forwards to the C ABI declared in
``include/lora_sgmv.h`` under the same name.  Tensors are passed by device pointer (any
object with ``data_ptr()``, or a plain int), streams as a ``torch.cuda.Stream``, a raw
``cudaStream_t`` int, or ``None`` for torch's current stream.  Nonzero return codes raise
:class:`LoraError`.  There is no fallback: if the shared library is missing, importing the
functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# LORA_SGMV_LIB selects another build of the same library (e.g. a phase-traced one).
LIB_PATH = os.environ.get("LORA_SGMV_LIB") or os.path.join(_HERE, "liblora_sgmv.so")

LORA_F32 = 0
LORA_BF16 = 1
LORA_OK = 0
LORA_ERR_INVALID_ARG = -1
LORA_ERR_UNSUPPORTED = -2
LORA_ERR_WORKSPACE = -3
LORA_ERR_CUDA = -4
LORA_ERR_TIMEOUT = -5
LORA_ERR_DEVICE_STATUS = -6
LORA_STATUS_BAD_ID = 1
LORA_STATUS_TIMEOUT = 2
LORA_STATUS_BAD_SEGMENT = 4
LORA_MAX_RANK = 128
LORA_MAX_SEGMENT_TOKENS = 8192
LORA_NOALLOC_SCRATCH_FLOATS = 262144
LORA_MAX_GROUP = 4
LORA_SIGMA_NONE = 0
LORA_SIGMA_FULL = 1
LORA_SIGMA_DIAG = 2
LORA_MAX_MERGE = 8
LORA_KERNEL_KINDS = 7

EXPORTS = (
    "lora_table_create", "lora_table_destroy", "lora_table_info", "lora_workspace_bytes",
    "lora_build_segments", "lora_shrink", "lora_expand", "lora_sgmv", "lora_bgmv",
    "lora_get_status", "lora_status_string", "lora_set_option", "lora_get_option",
    "lora_sgmv_noalloc", "lora_sgmv_grouped", "lora_table_set_sigma", "lora_bgmv_merged",
    "lora_sgmv_base", "lora_kernel_name", "lora_kernel_launches",
)


class LoraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s: %s (%d)" % (where, status_string(code), code))


class lora_segments(ctypes.Structure):
    """Mirror of ``struct lora_segments`` (device pointers plus host sizes)."""

    _fields_ = [
        ("perm", ctypes.c_void_p),
        ("seg_ptr", ctypes.c_void_p),
        ("seg_adapter", ctypes.c_void_p),
        ("num_segs", ctypes.c_void_p),
        ("T", ctypes.c_int32),
        ("max_segs", ctypes.c_int32),
        ("max_seg_len", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("liblora_sgmv.so is not built (python -m heterogeneous_adapters_sgmv_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "lora_table_create": ([ctypes.POINTER(P), I32, I32, I32, I32, P, P, P, P, P], ctypes.c_int),
        "lora_table_destroy": ([P], ctypes.c_int),
        "lora_table_set_sigma": ([P, I32, P, P], ctypes.c_int),
        "lora_table_info": ([P, P, P, P, P, P], ctypes.c_int),
        "lora_workspace_bytes": ([P, I32], SZ),
        "lora_build_segments": ([P, P, I32, P, P, P, P, P], ctypes.c_int),
        "lora_shrink": ([P, ctypes.POINTER(lora_segments), P, I64, P, I32, P], ctypes.c_int),
        "lora_expand": ([P, ctypes.POINTER(lora_segments), P, I32, P, I64, I32, P], ctypes.c_int),
        "lora_sgmv": ([P, ctypes.POINTER(lora_segments), P, I64, P, I64, I32, P, SZ, P], ctypes.c_int),
        "lora_bgmv": ([P, P, I32, P, I64, P, I64, I32, P, SZ, P], ctypes.c_int),
        "lora_bgmv_merged": ([P, P, P, I32, I32, P, I64, P, I64, I32, P, SZ, P], ctypes.c_int),
        "lora_sgmv_noalloc": ([P, ctypes.POINTER(lora_segments), P, I64, P, I64, I32, P], ctypes.c_int),
        "lora_sgmv_base": ([P, ctypes.POINTER(lora_segments), P, I64, P, I64, P, I64, I32, I32, P, SZ, P],
                           ctypes.c_int),
        "lora_sgmv_grouped": ([P, I32, ctypes.POINTER(lora_segments), P, P, P, P, P, P, SZ, P], ctypes.c_int),
        "lora_get_status": ([P, ctypes.POINTER(ctypes.c_uint32), I32, P], ctypes.c_int),
        "lora_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "lora_set_option": ([ctypes.c_char_p, I64], ctypes.c_int),
        "lora_get_option": ([ctypes.c_char_p, ctypes.POINTER(I64)], ctypes.c_int),
        "lora_kernel_name": ([I32], ctypes.c_char_p),
        "lora_kernel_launches": ([I32], I64),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _ptr(obj) -> Optional[int]:
    if obj is None:
        return None
    if isinstance(obj, int):
        return obj
    return int(obj.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(rc: int, where: str) -> None:
    if rc != LORA_OK:
        raise LoraError(rc, where)


def status_string(code: int) -> str:
    return _load().lora_status_string(code).decode()


lora_status_string = status_string


def lora_table_create(A_ptrs: Sequence[int], B_ptrs: Sequence[int], ranks: Sequence[int],
                      scales: Sequence[float], h_in: int, h_out: int, dtype: int, stream=None) -> int:
    n = len(A_ptrs)
    Pa = (ctypes.c_void_p * n)(*[int(a) for a in A_ptrs])
    Pb = (ctypes.c_void_p * n)(*[int(b) for b in B_ptrs])
    R = (ctypes.c_int32 * n)(*[int(r) for r in ranks])
    S = (ctypes.c_float * n)(*[float(s) for s in scales])
    out = ctypes.c_void_p()
    _check(_load().lora_table_create(ctypes.byref(out), n, h_in, h_out, dtype, Pa, Pb, R, S, _stream(stream)),
           "lora_table_create")
    return int(out.value)


def lora_table_destroy(table: int) -> None:
    _check(_load().lora_table_destroy(table), "lora_table_destroy")


def lora_table_info(table: int) -> dict:
    vals = [ctypes.c_int32() for _ in range(5)]
    _check(_load().lora_table_info(table, *[ctypes.byref(v) for v in vals]), "lora_table_info")
    return dict(zip(("n_adapters", "h_in", "h_out", "max_rank", "dtype"), (v.value for v in vals)))


def lora_workspace_bytes(table: int, T: int) -> int:
    return int(_load().lora_workspace_bytes(table, T))


def lora_build_segments(table: int, ids, T: int, perm, seg_ptr, seg_adapter, num_segs, stream=None) -> None:
    _check(_load().lora_build_segments(table, _ptr(ids), T, _ptr(perm), _ptr(seg_ptr), _ptr(seg_adapter),
                                       _ptr(num_segs), _stream(stream)), "lora_build_segments")


def make_segments(perm, seg_ptr, seg_adapter, num_segs, T: int, max_segs: int, max_seg_len: int = 0) -> lora_segments:
    return lora_segments(_ptr(perm), _ptr(seg_ptr), _ptr(seg_adapter), _ptr(num_segs), T, max_segs, max_seg_len, 0)


def lora_shrink(table: int, seg: lora_segments, x, ldx: int, v, ldv: int, stream=None) -> None:
    _check(_load().lora_shrink(table, ctypes.byref(seg), _ptr(x), ldx, _ptr(v), ldv, _stream(stream)),
           "lora_shrink")


def lora_expand(table: int, seg: lora_segments, v, ldv: int, y, ldy: int, y_offset: int, stream=None) -> None:
    _check(_load().lora_expand(table, ctypes.byref(seg), _ptr(v), ldv, _ptr(y), ldy, y_offset, _stream(stream)),
           "lora_expand")


def lora_sgmv(table: int, seg: lora_segments, x, ldx: int, y, ldy: int, y_offset: int, ws=None,
              ws_bytes: int = 0, stream=None) -> None:
    _check(_load().lora_sgmv(table, ctypes.byref(seg), _ptr(x), ldx, _ptr(y), ldy, y_offset, _ptr(ws), ws_bytes,
                             _stream(stream)), "lora_sgmv")


def lora_sgmv_base(table: int, seg: lora_segments, x, ldx: int, W, ldw: int, y, ldy: int, y_offset: int,
                   accumulate: bool = False, ws=None, ws_bytes: int = 0, stream=None) -> None:
    """Layer output with the frozen base weight W [o, h]: y = (y if accumulate) + x W^T +
    s_i B_i A_i x, on the tensor cores (contiguous segments, bf16)."""
    _check(_load().lora_sgmv_base(table, ctypes.byref(seg), _ptr(x), ldx, _ptr(W), ldw, _ptr(y), ldy, y_offset,
                                  1 if accumulate else 0, _ptr(ws), ws_bytes, _stream(stream)), "lora_sgmv_base")


def lora_sgmv_grouped(tables, seg: lora_segments, xs, ldxs, ys, ldys, y_offsets, ws=None, ws_bytes: int = 0,
                      stream=None) -> None:
    """One launch for several projections sharing a segment table: projection p applies
    tables[p] to xs[p] and updates ys[p][:, y_offsets[p] : y_offsets[p] + o_p]."""
    P = len(tables)
    if not (len(xs) == len(ldxs) == len(ys) == len(ldys) == len(y_offsets) == P):
        raise ValueError("lora_sgmv_grouped: every per-projection list needs one entry per table")
    t_arr = (ctypes.c_void_p * P)(*tables)
    x_arr = (ctypes.c_void_p * P)(*[_ptr(x) for x in xs])
    y_arr = (ctypes.c_void_p * P)(*[_ptr(y) for y in ys])
    ldx_arr = (ctypes.c_int64 * P)(*ldxs)
    ldy_arr = (ctypes.c_int64 * P)(*ldys)
    off_arr = (ctypes.c_int32 * P)(*y_offsets)
    _check(_load().lora_sgmv_grouped(t_arr, P, ctypes.byref(seg), x_arr, ldx_arr, y_arr, ldy_arr, off_arr,
                                     _ptr(ws), ws_bytes, _stream(stream)), "lora_sgmv_grouped")


def lora_bgmv_merged(table: int, ids, w, T: int, K: int, x, ldx: int, y, ldy: int, y_offset: int, ws=None,
                     ws_bytes: int = 0, stream=None) -> None:
    """Several adapters per token: ids and w are [T, K] device tensors (int32 / fp32, -1 =
    empty slot); y[t] += sum_j w[t, j] s_i B_i A_i x[t]."""
    _check(_load().lora_bgmv_merged(table, _ptr(ids), _ptr(w), T, K, _ptr(x), ldx, _ptr(y), ldy, y_offset, _ptr(ws),
                                    ws_bytes, _stream(stream)), "lora_bgmv_merged")


def lora_sgmv_noalloc(table: int, seg: lora_segments, x, ldx: int, y, ldy: int, y_offset: int, stream=None) -> None:
    """SGMV for callers that cannot allocate device memory: the fp32 intermediate lives in a
    fixed 1 MiB array owned by the library (T * ldv <= LORA_NOALLOC_SCRATCH_FLOATS).  Calls
    that may overlap on the GPU share that array and must be serialised by the caller."""
    _check(_load().lora_sgmv_noalloc(table, ctypes.byref(seg), _ptr(x), ldx, _ptr(y), ldy, y_offset,
                                     _stream(stream)), "lora_sgmv_noalloc")


def lora_bgmv(table: int, ids, T: int, x, ldx: int, y, ldy: int, y_offset: int, ws=None, ws_bytes: int = 0,
              stream=None) -> None:
    _check(_load().lora_bgmv(table, _ptr(ids), T, _ptr(x), ldx, _ptr(y), ldy, y_offset, _ptr(ws), ws_bytes,
                             _stream(stream)), "lora_bgmv")


def lora_get_status(table: int, reset: bool = True, stream=None):
    """Returns (return code, status word); does not raise."""
    w = ctypes.c_uint32()
    rc = _load().lora_get_status(table, ctypes.byref(w), 1 if reset else 0, _stream(stream))
    return rc, int(w.value)


def lora_set_option(key: str, value: int) -> None:
    _check(_load().lora_set_option(key.encode(), int(value)), "lora_set_option")


def lora_get_option(key: str) -> int:
    v = ctypes.c_int64()
    _check(_load().lora_get_option(key.encode(), ctypes.byref(v)), "lora_get_option")
    return int(v.value)


def kernel_launches() -> dict:
    """{kernel name: launches the CUDA runtime accepted so far in this process}."""
    lib = _load()
    return {lib.lora_kernel_name(k).decode(): int(lib.lora_kernel_launches(k)) for k in range(LORA_KERNEL_KINDS)}


def lora_table_set_sigma(table: int, kind: int, sigma: Optional[Sequence] = None, stream=None) -> None:
    arr = None
    if sigma is not None:
        arr = (ctypes.c_void_p * len(sigma))(*[_ptr(sg) for sg in sigma])
    _check(_load().lora_table_set_sigma(table, kind, arr, _stream(stream)), "lora_table_set_sigma")


class AdapterTable:
    """Owns one ``lora_table`` and keeps the weight tensors it points to alive."""

    def __init__(self, A: Sequence, B: Sequence, ranks: Sequence[int], scales: Sequence[float],
                 h_in: int, h_out: int, dtype: int, stream=None, keep=None):
        self._keep = (list(A), list(B), keep)
        self.handle = lora_table_create([_ptr(a) for a in A], [_ptr(b) for b in B], ranks, scales,
                                        h_in, h_out, dtype, stream)
        self.n, self.h, self.o, self.dtype = len(A), h_in, h_out, dtype
        self.max_rank = max(int(r) for r in ranks)

    def close(self) -> None:
        if self.handle:
            lora_table_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, T: int) -> int:
        return lora_workspace_bytes(self.handle, T)

    def set_sigma(self, kind: int, sigma: Optional[Sequence] = None, stream=None) -> None:
        """Three-stage form: register Sigma_i per adapter (device fp32 tensors, [r_i, r_i] for
        LORA_SIGMA_FULL or [r_i] for LORA_SIGMA_DIAG); LORA_SIGMA_NONE removes it."""
        lora_table_set_sigma(self.handle, kind, sigma, stream)
        self._sigma = list(sigma) if sigma is not None else None
