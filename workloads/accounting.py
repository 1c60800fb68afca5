"""Byte and FLOP accounting for the LoRA delta (measurement bookkeeping, no method arithmetic).

Algorithmic bytes of one call over one projection:

* x read once:                 T_valid * h * e
* y read and written:          2 * T_valid * o * e
* each distinct touched adapter's weights, once: r_i * (h + o) * e

The rank-space intermediate, the ids and the segment table are not counted.  ``e`` is the
element size (2 for bf16, 4 for fp32).  T_valid counts tokens whose id names an adapter.
"""
from __future__ import annotations

from typing import Iterable, Sequence, Tuple

import numpy as np

ELEM_BYTES = {"bf16": 2, "f32": 4}


def distinct_adapters(ids: np.ndarray) -> np.ndarray:
    ids = np.asarray(ids)
    return np.unique(ids[ids >= 0])


def projection_bytes(T_valid: int, h: int, o: int, ranks_touched: Iterable[int], e: int) -> int:
    w = sum(int(r) * (h + o) * e for r in ranks_touched)
    return T_valid * h * e + 2 * T_valid * o * e + w


def projection_flops(ids: np.ndarray, ranks: np.ndarray, h: int, o: int) -> int:
    """Multiply-adds counted as 2 flops: shrink T*r*h plus expand T*o*r per token."""
    ids = np.asarray(ids)
    r = np.asarray(ranks)[ids[ids >= 0]].astype(np.int64)
    return int(2 * (r * h).sum() + 2 * (r * o).sum())


def workload_bytes(wl, shared_x: bool = False, sigma: str = "none", clusters: int = 0) -> int:
    """Algorithmic bytes of one step of a workload (all projections).  With ``shared_x`` the
    projections that read the same activations (q, k and v) count x once, as one grouped
    launch reads it.  For the three-stage form, ``sigma`` ("full" / "diag") adds each
    touched adapter's fp32 Sigma_i (r^2 or r values), and ``clusters`` > 0 shares A and B
    inside clusters (adapter i uses adapter i mod clusters' weights), so the weights of each
    touched cluster count once."""
    e = ELEM_BYTES[wl.dtype]
    d = distinct_adapters(wl.ids)
    T_valid = int((np.asarray(wl.ids) >= 0).sum())
    leaders = np.unique(d % clusters) if clusters > 0 else d
    tot = 0
    seen = set()
    # projections of one x group hold the same activation array
    groups = [id(p.x) for p in wl.projections] if shared_x else range(len(wl.projections))
    for p, g in zip(wl.projections, groups):
        tot += projection_bytes(T_valid, p.h, p.o, (p.ranks[i] for i in leaders), e)
        if g in seen:
            tot -= T_valid * p.h * e
        seen.add(g)
        if sigma == "full":
            tot += int(sum(4 * int(p.ranks[i]) ** 2 for i in d))
        elif sigma == "diag":
            tot += int(sum(4 * int(p.ranks[i]) for i in d))
    return tot


def merged_bytes(wl, ids2d: np.ndarray) -> int:
    """Algorithmic bytes of one call of the merged form on projection 0: x read and y read and
    written once, and every adapter any slot touches once."""
    e = ELEM_BYTES[wl.dtype]
    p = wl.projections[0]
    ids2d = np.asarray(ids2d)
    d = distinct_adapters(ids2d.ravel())
    T_valid = int((ids2d >= 0).any(axis=1).sum())
    return projection_bytes(T_valid, p.h, p.o, (p.ranks[i] for i in d), e)


def workload_flops(wl) -> int:
    return sum(projection_flops(wl.ids, p.ranks, p.h, p.o) for p in wl.projections)


def adapter_bytes(shapes: Sequence[Tuple[int, int]], rank: int, layers: int, e: int) -> int:
    """Storage of one adapter: for every adapted (h -> o) projection of every layer,
    A is r x h and B is o x r."""
    return layers * sum(rank * (h + o) * e for (h, o) in shapes)


def base_layer_bytes(wl) -> int:
    """Algorithmic bytes of the layer output with a frozen base weight (projection 0, y written
    and not read): x once, W [o, h] once, y written once, every distinct touched adapter once."""
    e = ELEM_BYTES[wl.dtype]
    p = wl.projections[0]
    d = distinct_adapters(wl.ids)
    return wl.T * p.h * e + p.o * p.h * e + wl.T * p.o * e + sum(int(p.ranks[i]) * (p.h + p.o) * e for i in d)


def base_layer_flops(wl) -> int:
    """Multiply-adds (2 flops each) of the layer output: the base product for every token plus
    the adapter shrink and expand of every token with an adapter."""
    p = wl.projections[0]
    return 2 * wl.T * p.o * p.h + projection_flops(wl.ids, p.ranks, p.h, p.o)
