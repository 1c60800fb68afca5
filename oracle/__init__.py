"""CPU oracle for the heterogeneous-batch LoRA delta -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``heterogeneous_adapters_sgmv_b200``) never
imports it, and the two share no code: the only common module is ``workloads`` (seeded
input draws, no arithmetic of the method).

Two independent implementations live here:

* ``lora_oracle.c`` (loaded through ctypes): a plain fp64 loop, one token at a time --
  shrink ``v = A_i x`` with scale 1, then expand ``y = y0 + s_i B_i v`` into a column slice
  of y -- following the LoRA definition of the "TGI Multi-LoRA" page ("Technical
  Foundation: LoRA") and the add_lora_slice pseudocode of the "Compress then Serve"
  review thread (authors' rebuttal on Punica).  Also the stable segment bookkeeping that
  SGMV's grouping of same-adapter requests implies.
  The same file holds the three-stage form of that thread's add_lora_slice_with_sigma
  pseudocode (A with scale 1, then the adapter's small Sigma_i, full or diagonal, with
  scale 1, then B with the scale).
* ``brute.py``: numpy fp64 matrix products per adapter group (a different evaluation
  order), used to cross-check the loop.

Pins (``tests/test_oracle_pins.py``) tie both to closed forms and invariants that the
pages and the mathematics fix; parity of the delta values themselves is not pinned by any
number printed on the pages (they print none).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lora_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblora_oracle.so")
_lib = None

ORACLE_F32 = 0
ORACLE_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, OpenMP over tokens, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int32
    lib.oracle_lora_delta.argtypes = [ctypes.c_int, i64, i64, i64, P, i64, P, i64, i64,
                                      P, i32, P, P, P, P, P, ctypes.c_int]
    lib.oracle_lora_delta.restype = ctypes.c_int
    lib.oracle_lora_shrink.argtypes = [ctypes.c_int, i64, i64, P, i64, P, i32, P, P, P, i64,
                                       ctypes.c_int]
    lib.oracle_lora_shrink.restype = ctypes.c_int
    lib.oracle_lora_expand.argtypes = [ctypes.c_int, i64, i64, P, i64, P, i64, i64, P, i32,
                                       P, P, P, P, ctypes.c_int]
    lib.oracle_lora_expand.restype = ctypes.c_int
    lib.oracle_lora_delta_sigma.argtypes = [ctypes.c_int, i64, i64, i64, P, i64, P, i64, i64,
                                            P, i32, P, P, P, P, ctypes.c_int, P, P, ctypes.c_int]
    lib.oracle_lora_delta_sigma.restype = ctypes.c_int
    lib.oracle_lora_shrink_sigma.argtypes = [ctypes.c_int, i64, i64, P, i64, P, i32, P, P, ctypes.c_int, P, P,
                                             i64, ctypes.c_int]
    lib.oracle_lora_shrink_sigma.restype = ctypes.c_int
    lib.oracle_lora_delta_merged.argtypes = [ctypes.c_int, i64, i64, i64, P, i64, P, i64, i64, i32, P, P, i32,
                                             P, P, P, P, P, ctypes.c_int]
    lib.oracle_lora_delta_merged.restype = ctypes.c_int
    lib.oracle_lora_base_delta.argtypes = [ctypes.c_int, i64, i64, i64, P, i64, P, i64, P, i64, i64, ctypes.c_int,
                                           P, i32, P, P, P, P, P, ctypes.c_int]
    lib.oracle_lora_base_delta.restype = ctypes.c_int
    lib.oracle_build_segments.argtypes = [i64, P, i32, P, P, P, P]
    lib.oracle_build_segments.restype = ctypes.c_int64
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _dtype_code(dtype: str) -> int:
    return {"f32": ORACLE_F32, "bf16": ORACLE_BF16}[dtype]


def _check_store(a: np.ndarray, dtype: str) -> np.ndarray:
    want = np.uint16 if dtype == "bf16" else np.float32
    a = np.ascontiguousarray(a)
    if a.dtype != want:
        raise TypeError("expected %s storage, got %s" % (want, a.dtype))
    return a


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class OracleError(ValueError):
    pass


def lora_delta(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray,
               A: Sequence[np.ndarray], B: Sequence[np.ndarray],
               scales: Sequence[float], y_offset: int = 0, o: Optional[int] = None,
               threads: int = 0) -> np.ndarray:
    """fp64 y_ref[T, o] = y0[:, y_offset:y_offset+o] + s_i * B_i (A_i x[t]) for i = ids[t]."""
    x = _check_store(x, dtype)
    y0 = _check_store(y0, dtype)
    T, h = x.shape
    if o is None:
        o = y0.shape[1] - y_offset
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n = len(A)
    As = [_check_store(a, dtype) for a in A]
    Bs = [_check_store(b, dtype) for b in B]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    for a, b, r in zip(As, Bs, ranks):
        if a.shape != (r, h) or b.shape != (o, r):
            raise ValueError("adapter shapes %s / %s do not match h=%d o=%d" % (a.shape, b.shape, h, o))
    Ap = (ctypes.c_void_p * max(n, 1))(*[_ptr(a) for a in As])
    Bp = (ctypes.c_void_p * max(n, 1))(*[_ptr(b) for b in Bs])
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32).astype(np.float64))
    out = np.empty((T, o), dtype=np.float64)
    rc = _load().oracle_lora_delta(_dtype_code(dtype), T, h, o, _ptr(x), x.shape[1], _ptr(y0),
                                   y0.shape[1], y_offset, _ptr(ids), n, Ap, Bp, _ptr(ranks),
                                   _ptr(sc), _ptr(out), threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return out


def lora_shrink(dtype: str, x: np.ndarray, ids: np.ndarray, A: Sequence[np.ndarray],
                ldv: int, threads: int = 0) -> np.ndarray:
    """fp64 v[T, ldv]: v[t, k] = (A_i x[t])[k] for k < r_i, zero elsewhere."""
    x = _check_store(x, dtype)
    T, h = x.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    As = [_check_store(a, dtype) for a in A]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    Ap = (ctypes.c_void_p * max(len(As), 1))(*[_ptr(a) for a in As])
    v = np.empty((T, ldv), dtype=np.float64)
    rc = _load().oracle_lora_shrink(_dtype_code(dtype), T, h, _ptr(x), x.shape[1], _ptr(ids),
                                    len(As), Ap, _ptr(ranks), _ptr(v), ldv, threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return v


def lora_expand(dtype: str, v: np.ndarray, y0: np.ndarray, ids: np.ndarray,
                B: Sequence[np.ndarray], scales: Sequence[float], y_offset: int = 0,
                o: Optional[int] = None, threads: int = 0) -> np.ndarray:
    """fp64 y_ref[T, o] = y0[:, off:off+o] + s_i * B_i v[t, :r_i] for a given fp32 v."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    y0 = _check_store(y0, dtype)
    T = y0.shape[0]
    if o is None:
        o = y0.shape[1] - y_offset
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    Bs = [_check_store(b, dtype) for b in B]
    ranks = np.array([b.shape[1] for b in Bs], dtype=np.int32)
    Bp = (ctypes.c_void_p * max(len(Bs), 1))(*[_ptr(b) for b in Bs])
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32).astype(np.float64))
    out = np.empty((T, o), dtype=np.float64)
    rc = _load().oracle_lora_expand(_dtype_code(dtype), T, o, _ptr(v), v.shape[1], _ptr(y0),
                                    y0.shape[1], y_offset, _ptr(ids), len(Bs), Bp, _ptr(ranks),
                                    _ptr(sc), _ptr(out), threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return out


SIGMA_NONE, SIGMA_FULL, SIGMA_DIAG = 0, 1, 2


def _sigma_arrays(sigma_kind: int, sigma, ranks: np.ndarray):
    if sigma_kind not in (SIGMA_NONE, SIGMA_FULL, SIGMA_DIAG):
        raise ValueError("sigma_kind")
    if sigma_kind == SIGMA_NONE:
        return [], None
    Ss = [np.ascontiguousarray(sg, dtype=np.float32) for sg in sigma]
    for sg, r in zip(Ss, ranks):
        want = (r, r) if sigma_kind == SIGMA_FULL else (r,)
        if sg.shape != want:
            raise ValueError("Sigma shape %s, want %s" % (sg.shape, want))
    return Ss, (ctypes.c_void_p * max(len(Ss), 1))(*[_ptr(sg) for sg in Ss])


def lora_delta_sigma(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray,
                     A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
                     sigma_kind: int, sigma: Sequence[np.ndarray], y_offset: int = 0,
                     o: Optional[int] = None, threads: int = 0) -> np.ndarray:
    """Three-stage form: fp64 y_ref = y0 + s_i B_i (Sigma_i (A_i x[t])) -- Sigma_i full
    (r_i x r_i) or diagonal (r_i values), fp32 values."""
    x = _check_store(x, dtype)
    y0 = _check_store(y0, dtype)
    T, h = x.shape
    if o is None:
        o = y0.shape[1] - y_offset
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n = len(A)
    As = [_check_store(a, dtype) for a in A]
    Bs = [_check_store(b, dtype) for b in B]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    for a, b, r in zip(As, Bs, ranks):
        if a.shape != (r, h) or b.shape != (o, r):
            raise ValueError("adapter shapes %s / %s do not match h=%d o=%d" % (a.shape, b.shape, h, o))
    Ss, Sp = _sigma_arrays(sigma_kind, sigma, ranks)
    Ap = (ctypes.c_void_p * max(n, 1))(*[_ptr(a) for a in As])
    Bp = (ctypes.c_void_p * max(n, 1))(*[_ptr(b) for b in Bs])
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32).astype(np.float64))
    out = np.empty((T, o), dtype=np.float64)
    rc = _load().oracle_lora_delta_sigma(_dtype_code(dtype), T, h, o, _ptr(x), x.shape[1], _ptr(y0),
                                         y0.shape[1], y_offset, _ptr(ids), n, Ap, Bp, _ptr(ranks),
                                         _ptr(sc), sigma_kind, Sp, _ptr(out), threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return out


def lora_shrink_sigma(dtype: str, x: np.ndarray, ids: np.ndarray, A: Sequence[np.ndarray],
                      sigma_kind: int, sigma: Sequence[np.ndarray], ldv: Optional[int] = None,
                      threads: int = 0) -> np.ndarray:
    """Steps 1 and 2 of the three-stage form: fp64 v[t, :r_i] = Sigma_i (A_i x[t])."""
    x = _check_store(x, dtype)
    T, h = x.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    As = [_check_store(a, dtype) for a in A]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    if ldv is None:
        ldv = int(ranks.max()) if len(ranks) else 1
    Ss, Sp = _sigma_arrays(sigma_kind, sigma, ranks)
    Ap = (ctypes.c_void_p * max(len(As), 1))(*[_ptr(a) for a in As])
    v = np.empty((T, ldv), dtype=np.float64)
    rc = _load().oracle_lora_shrink_sigma(_dtype_code(dtype), T, h, _ptr(x), x.shape[1], _ptr(ids), len(As), Ap,
                                          _ptr(ranks), sigma_kind, Sp, _ptr(v), ldv, threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return v


def lora_delta_merged(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray, w: np.ndarray,
                      A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
                      y_offset: int = 0, o: Optional[int] = None, threads: int = 0) -> np.ndarray:
    """Several adapters per token: fp64 y_ref = y0 + sum_j w[t, j] s_i B_i (A_i x[t]) over the
    K slots of ids[t, :] (-1 = empty); ids and w are [T, K]."""
    x = _check_store(x, dtype)
    y0 = _check_store(y0, dtype)
    T, h = x.shape
    if o is None:
        o = y0.shape[1] - y_offset
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    if ids.ndim != 2 or ids.shape[0] != T or w.shape != ids.shape:
        raise ValueError("ids and w must both be [T, K]")
    K = ids.shape[1]
    n = len(A)
    As = [_check_store(a, dtype) for a in A]
    Bs = [_check_store(b, dtype) for b in B]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    for a, b, r in zip(As, Bs, ranks):
        if a.shape != (r, h) or b.shape != (o, r):
            raise ValueError("adapter shapes %s / %s do not match h=%d o=%d" % (a.shape, b.shape, h, o))
    Ap = (ctypes.c_void_p * max(n, 1))(*[_ptr(a) for a in As])
    Bp = (ctypes.c_void_p * max(n, 1))(*[_ptr(b) for b in Bs])
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32).astype(np.float64))
    out = np.empty((T, o), dtype=np.float64)
    rc = _load().oracle_lora_delta_merged(_dtype_code(dtype), T, h, o, _ptr(x), x.shape[1], _ptr(y0), y0.shape[1],
                                          y_offset, K, _ptr(ids), _ptr(w), n, Ap, Bp, _ptr(ranks), _ptr(sc),
                                          _ptr(out), threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return out


def lora_base_delta(dtype: str, x: np.ndarray, W: np.ndarray, y0: np.ndarray, ids: np.ndarray,
                    A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
                    accumulate: bool = True, y_offset: int = 0, o: Optional[int] = None,
                    threads: int = 0) -> np.ndarray:
    """Layer output with the frozen base weight W [o, h]: fp64 y_ref = (y0 if accumulate)
    + W x[t] + s_i B_i (A_i x[t]) for i = ids[t] (id -1: no adapter term)."""
    x = _check_store(x, dtype)
    W = _check_store(W, dtype)
    y0 = _check_store(y0, dtype)
    T, h = x.shape
    if o is None:
        o = y0.shape[1] - y_offset
    if W.shape[0] != o or W.shape[1] < h:
        raise ValueError("W shape %s does not match h=%d o=%d" % (W.shape, h, o))
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    n = len(A)
    As = [_check_store(a, dtype) for a in A]
    Bs = [_check_store(b, dtype) for b in B]
    ranks = np.array([a.shape[0] for a in As], dtype=np.int32)
    for a, b, r in zip(As, Bs, ranks):
        if a.shape != (r, h) or b.shape != (o, r):
            raise ValueError("adapter shapes %s / %s do not match h=%d o=%d" % (a.shape, b.shape, h, o))
    Ap = (ctypes.c_void_p * max(n, 1))(*[_ptr(a) for a in As])
    Bp = (ctypes.c_void_p * max(n, 1))(*[_ptr(b) for b in Bs])
    sc = np.ascontiguousarray(np.asarray(scales, dtype=np.float32).astype(np.float64))
    out = np.empty((T, o), dtype=np.float64)
    rc = _load().oracle_lora_base_delta(_dtype_code(dtype), T, h, o, _ptr(x), x.shape[1], _ptr(W), W.shape[1],
                                        _ptr(y0), y0.shape[1], y_offset, 1 if accumulate else 0, _ptr(ids), n,
                                        Ap, Bp, _ptr(ranks), _ptr(sc), _ptr(out), threads)
    if rc != 0:
        raise OracleError("adapter id out of range")
    return out


def build_segments(ids: np.ndarray, n_adapters: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Stable counting sort by adapter id -> (perm[valid], seg_ptr[S+1], seg_adapter[S])."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T = ids.size
    perm = np.empty(max(T, 1), dtype=np.int32)
    seg_ptr = np.empty(n_adapters + 1, dtype=np.int32)
    seg_adapter = np.empty(max(n_adapters, 1), dtype=np.int32)
    ns = np.zeros(1, dtype=np.int32)
    valid = _load().oracle_build_segments(T, _ptr(ids), n_adapters, _ptr(perm), _ptr(seg_ptr),
                                          _ptr(seg_adapter), _ptr(ns))
    if valid < 0:
        raise OracleError("adapter id out of range")
    S = int(ns[0])
    return perm[:valid].copy(), seg_ptr[:S + 1].copy(), seg_adapter[:S].copy()


def base_reference(wl, W: np.ndarray, accumulate: bool = True, proj_index: int = 0,
                   threads: int = 0) -> np.ndarray:
    """Oracle layer output (fp64, unrounded) of one projection with the base weight W."""
    p = wl.projections[proj_index]
    A = [p.A(i) for i in range(wl.n)]
    B = [p.B(i) for i in range(wl.n)]
    return lora_base_delta(wl.dtype, p.x, W, p.y0, wl.ids, A, B, p.scales, accumulate=accumulate,
                           threads=threads)


def workload_reference(wl, proj_index: int = 0, threads: int = 0) -> np.ndarray:
    """Oracle output (fp64, unrounded) of one projection of a ``workloads.Workload``."""
    p = wl.projections[proj_index]
    A = [p.A(i) for i in range(wl.n)]
    B = [p.B(i) for i in range(wl.n)]
    return lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, threads=threads)
