"""Second, independent CPU implementation of the LoRA delta -- TEST INFRASTRUCTURE ONLY.

numpy fp64 matrix products per adapter group: for every adapter i, gather the rows of the
tokens that name it and evaluate ``y0 + s_i * (x_g @ A_i^T) @ B_i^T``.  This groups tokens
by adapter (the grouping SGMV performs, "Compress then Serve" review thread, rebuttal on
Punica) and uses library matrix products, so it shares neither loop structure nor
summation order with ``lora_oracle.c``.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

from workloads import to_float64


def lora_delta(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray,
               A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
               y_offset: int = 0, o: int = None) -> np.ndarray:
    ids = np.asarray(ids)
    if ((ids < -1) | (ids >= len(A))).any():
        raise ValueError("adapter id out of range")
    if o is None:
        o = y0.shape[1] - y_offset
    xd = to_float64(x, dtype)
    out = to_float64(y0, dtype)[:, y_offset:y_offset + o].copy()
    for i in np.unique(ids[ids >= 0]):
        rows = np.nonzero(ids == i)[0]
        Ai = to_float64(A[i], dtype)
        Bi = to_float64(B[i], dtype)
        s = float(np.float32(scales[i]))
        out[rows] += s * ((xd[rows] @ Ai.T) @ Bi.T)
    return out


def lora_delta_sigma(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray,
                     A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
                     sigma_kind: int, sigma: Sequence[np.ndarray]) -> np.ndarray:
    """Three-stage form per adapter group: y0 + s_i * ((x_g @ A_i^T) @ Sigma_i^T) @ B_i^T, with
    Sigma_i full (sigma_kind 1) or diagonal (sigma_kind 2)."""
    ids = np.asarray(ids)
    if ((ids < -1) | (ids >= len(A))).any():
        raise ValueError("adapter id out of range")
    xd = to_float64(x, dtype)
    out = to_float64(y0, dtype).copy()
    for i in np.unique(ids[ids >= 0]):
        rows = np.nonzero(ids == i)[0]
        S = np.asarray(sigma[i], dtype=np.float64)
        S = S if sigma_kind == 1 else np.diag(S)
        u = xd[rows] @ to_float64(A[i], dtype).T
        out[rows] += float(np.float32(scales[i])) * ((u @ S.T) @ to_float64(B[i], dtype).T)
    return out


def lora_delta_merged(dtype: str, x: np.ndarray, y0: np.ndarray, ids: np.ndarray, w: np.ndarray,
                      A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float]) -> np.ndarray:
    """Merged ensembles, grouped by (slot, adapter): for every slot j and adapter i, the tokens
    whose slot j names i gain w[t, j] * s_i * (x_g @ A_i^T) @ B_i^T."""
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    if ((ids < -1) | (ids >= len(A))).any():
        raise ValueError("adapter id out of range")
    xd = to_float64(x, dtype)
    out = to_float64(y0, dtype).copy()
    for j in range(ids.shape[1]):
        col = ids[:, j]
        for i in np.unique(col[col >= 0]):
            rows = np.nonzero(col == i)[0]
            d = (xd[rows] @ to_float64(A[i], dtype).T) @ to_float64(B[i], dtype).T
            out[rows] += (w[rows, j] * float(np.float32(scales[i])))[:, None] * d
    return out


def lora_base_delta(dtype: str, x: np.ndarray, W: np.ndarray, y0: np.ndarray, ids: np.ndarray,
                    A: Sequence[np.ndarray], B: Sequence[np.ndarray], scales: Sequence[float],
                    accumulate: bool = True) -> np.ndarray:
    """Layer output with the frozen base weight: one library product x @ W^T for all tokens,
    then the adapter terms grouped by adapter."""
    xd = to_float64(x, dtype)
    base = xd @ to_float64(W, dtype)[:, :xd.shape[1]].T
    y = to_float64(y0, dtype) if accumulate else np.zeros_like(base)
    zero = np.zeros_like(y0)
    delta = lora_delta(dtype, x, zero, ids, A, B, scales)
    return y + base + delta
