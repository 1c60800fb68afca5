"""Seeded synthetic inputs for the heterogeneous-batch LoRA delta.

This module only draws random numbers and lays them out; it holds none of the
arithmetic of the method (no products, no sums over tokens or adapters).  Both
the CPU oracle (``oracle/``) and the CUDA path (``heterogeneous_adapters_sgmv_b200``)
are fed from here, so that they see bit-identical inputs.

Workload shapes follow the five synthetic workloads of the multi-LoRA serving
pages (Mistral-7B-class layers: hidden 4096, GQA k/v 1024, MLP up_proj 14336):

* ``tiny_sgmv``         h = o = 256, 4 adapters of rank 8, fp32, 16 tokens, uniform ids, s = 2
* ``decode_bgmv``       q_proj 4096 -> 4096, 32 adapters of rank 16, bf16, 64 tokens,
                        uniform ids, s = alpha / r = 2
* ``multirank_decode``  4096 -> 4096, 128 adapters, ranks uniform over {8, 16, 32, 64},
                        256 tokens, ids Zipf(1.0), s_i = 16 / r_i
* ``prefill_sgmv``      up_proj 4096 -> 14336, 8 contiguous segments of 512 tokens, segment k
                        uses adapter k, rank 64, s = 0.5
* ``many_adapter_qkvo`` 1000 adapters of rank 16 on q, o (4096 -> 4096) and k, v (4096 -> 1024),
                        512 tokens, ids Zipf(0.8), one id vector shared by the four projections, s = 2

Recipe (every choice here is a reading of the pages, which print no generator):

* ``numpy.random.default_rng(seed)`` with ``seed = 20260 + index`` of the workload in the list above.
* Draw order: ids; ranks; then per projection, per adapter in ascending id, A_i then B_i;
  then x (one per distinct input: q/k/v share one x, o has its own); then y0 per projection.
* ``N(0, v)`` is read as variance ``v`` (std ``sqrt(v)``); ``reading="std"`` takes ``v`` as the std.
* Normal draws are made in fp64 and rounded to nearest-even to fp32; bf16 workloads round that
  fp32 to nearest-even bf16.  The stored bits are what both sides consume.
* Zipf(s) over n ids is the bounded law ``P(id = k) ~ (k + 1) ** -s``, k = 0 .. n-1.
* y0 ~ N(0, 1) for every workload; ``delta_only=True`` sets y0 = 0 (the sensitive parity run).

Weights of one projection are stored in one flat array with per-adapter element offsets
(``A_off``, ``B_off``), each a multiple of 8 elements so every adapter starts on 16 bytes.
A_i is ``[r_i, h]`` row-major, B_i is ``[o, r_i]`` row-major.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

WORKLOAD_NAMES = (
    "tiny_sgmv",
    "decode_bgmv",
    "multirank_decode",
    "prefill_sgmv",
    "many_adapter_qkvo",
)

SEED_BASE = 20260


@dataclasses.dataclass(frozen=True)
class Spec:
    """Shape and distribution parameters of one workload."""

    name: str
    dtype: str                      # "bf16" or "f32"
    n: int                          # adapters per table
    T: int                          # tokens per batch
    ranks: Tuple[int, ...]          # rank choices (uniform over these)
    ids: str                        # "uniform" | "zipf" | "segments"
    zipf_s: float = 0.0
    seg_len: int = 0                # for ids == "segments"
    scale: str = "const"            # "const" | "16/r"
    scale_value: float = 2.0
    a_var: float = 0.02
    b_var: float = 0.02
    # (projection name, h, o, x group): projections in one x group read the same x
    projections: Tuple[Tuple[str, int, int, int], ...] = (("y", 4096, 4096, 0),)


SPECS: Dict[str, Spec] = {
    "tiny_sgmv": Spec(
        name="tiny_sgmv", dtype="f32", n=4, T=16, ranks=(8,), ids="uniform",
        scale_value=2.0, a_var=0.02, b_var=0.02,
        projections=(("y", 256, 256, 0),)),
    "decode_bgmv": Spec(
        name="decode_bgmv", dtype="bf16", n=32, T=64, ranks=(16,), ids="uniform",
        scale_value=2.0, a_var=1.0 / 4096, b_var=0.02,
        projections=(("q", 4096, 4096, 0),)),
    "multirank_decode": Spec(
        name="multirank_decode", dtype="bf16", n=128, T=256, ranks=(8, 16, 32, 64),
        ids="zipf", zipf_s=1.0, scale="16/r", a_var=1.0 / 4096, b_var=0.02,
        projections=(("q", 4096, 4096, 0),)),
    "prefill_sgmv": Spec(
        name="prefill_sgmv", dtype="bf16", n=8, T=8 * 512, ranks=(64,), ids="segments",
        seg_len=512, scale_value=0.5, a_var=1.0 / 4096, b_var=0.02,
        projections=(("up", 4096, 14336, 0),)),
    "many_adapter_qkvo": Spec(
        name="many_adapter_qkvo", dtype="bf16", n=1000, T=512, ranks=(16,), ids="zipf",
        zipf_s=0.8, scale_value=2.0, a_var=1.0 / 4096, b_var=0.02,
        projections=(("q", 4096, 4096, 0), ("k", 4096, 1024, 0),
                     ("v", 4096, 1024, 0), ("o", 4096, 4096, 1))),
}


@dataclasses.dataclass
class Projection:
    """One adapter table (one layer projection) with its activations."""

    name: str
    h: int
    o: int
    ranks: np.ndarray               # int32 [n]
    scales: np.ndarray              # float32 [n]
    A_flat: np.ndarray              # uint16 (bf16 bits) or float32, all A_i back to back
    A_off: np.ndarray               # int64 [n] element offset of A_i in A_flat
    B_flat: np.ndarray
    B_off: np.ndarray
    x: np.ndarray                   # [T, h] uint16 bits or float32
    y0: np.ndarray                  # [T, o] uint16 bits or float32

    def A(self, i: int) -> np.ndarray:
        r = int(self.ranks[i])
        return self.A_flat[self.A_off[i]: self.A_off[i] + r * self.h].reshape(r, self.h)

    def B(self, i: int) -> np.ndarray:
        r = int(self.ranks[i])
        return self.B_flat[self.B_off[i]: self.B_off[i] + self.o * r].reshape(self.o, r)


@dataclasses.dataclass
class Workload:
    spec: Spec
    seed: int
    reading: str
    delta_only: bool
    dtype: str
    T: int
    n: int
    ids: np.ndarray                 # int32 [T]
    projections: List[Projection]

    @property
    def name(self) -> str:
        return self.spec.name


# ----------------------------------------------------------------------------------------
# rounding helpers (pure bit manipulation)

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to nearest-even bfloat16; return the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_float64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values (bf16 bits or float32) to float64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _store(vals64: np.ndarray, dtype: str) -> np.ndarray:
    f32 = vals64.astype(np.float32)          # RNE fp64 -> fp32
    if dtype == "bf16":
        return f32_to_bf16_bits(f32)
    return f32


def _normal(rng: np.random.Generator, shape, var: float, reading: str, dtype: str) -> np.ndarray:
    std = np.sqrt(var) if reading == "variance" else var
    return _store(rng.standard_normal(shape) * std, dtype)


def _zipf_probs(n: int, s: float) -> np.ndarray:
    p = (np.arange(n, dtype=np.float64) + 1.0) ** (-s)
    return p / p.sum()


def draw_ids(spec: Spec, rng: np.random.Generator, T: int, n: int, seg_len: int) -> np.ndarray:
    if spec.ids == "uniform":
        ids = rng.integers(0, n, size=T)
    elif spec.ids == "zipf":
        ids = rng.choice(n, size=T, p=_zipf_probs(n, spec.zipf_s))
    elif spec.ids == "segments":
        ids = np.repeat(np.arange(T // seg_len), seg_len)
        ids = np.concatenate([ids, np.full(T - ids.size, T // seg_len)])[:T]
    else:
        raise ValueError(spec.ids)
    return np.ascontiguousarray(ids, dtype=np.int32)


def generate(name: str, *, seed: Optional[int] = None, reading: str = "variance",
             delta_only: bool = False, T: Optional[int] = None, n: Optional[int] = None,
             seg_len: Optional[int] = None,
             shapes: Optional[Sequence[Tuple[str, int, int, int]]] = None,
             ranks: Optional[Tuple[int, ...]] = None) -> Workload:
    """Draw one workload.  Overrides (T, n, seg_len, shapes, ranks) keep the workload's
    structure and distributions but shrink it for quick tests."""
    spec = SPECS[name]
    if reading not in ("variance", "std"):
        raise ValueError(reading)
    if seed is None:
        seed = SEED_BASE + WORKLOAD_NAMES.index(name)
    seg_len = seg_len if seg_len is not None else spec.seg_len
    if spec.ids == "segments":
        n_ = n if n is not None else spec.n
        T_ = T if T is not None else n_ * seg_len
        n_ = max(n_, -(-T_ // seg_len))
    else:
        n_ = n if n is not None else spec.n
        T_ = T if T is not None else spec.T
    projs = tuple(shapes) if shapes is not None else spec.projections
    rank_choices = tuple(ranks) if ranks is not None else spec.ranks
    rng = np.random.default_rng(seed)

    ids = draw_ids(spec, rng, T_, n_, seg_len)
    if len(rank_choices) == 1:
        rk = np.full(n_, rank_choices[0], dtype=np.int32)
    else:
        rk = rng.choice(np.asarray(rank_choices, dtype=np.int32), size=n_).astype(np.int32)
    if spec.scale == "16/r":
        sc = (16.0 / rk).astype(np.float32)
    else:
        sc = np.full(n_, spec.scale_value, dtype=np.float32)

    out: List[Projection] = []
    for (pname, h, o, _grp) in projs:
        a_sizes = rk.astype(np.int64) * h
        b_sizes = rk.astype(np.int64) * o
        a_off = np.concatenate([[0], np.cumsum(a_sizes)[:-1]]).astype(np.int64)
        b_off = np.concatenate([[0], np.cumsum(b_sizes)[:-1]]).astype(np.int64)
        store_dt = np.uint16 if spec.dtype == "bf16" else np.float32
        A_flat = np.empty(int(a_sizes.sum()), dtype=store_dt)
        B_flat = np.empty(int(b_sizes.sum()), dtype=store_dt)
        for i in range(n_):
            r = int(rk[i])
            A_flat[a_off[i]: a_off[i] + r * h] = _normal(rng, (r * h,), spec.a_var, reading, spec.dtype)
            B_flat[b_off[i]: b_off[i] + o * r] = _normal(rng, (o * r,), spec.b_var, reading, spec.dtype)
        out.append(Projection(name=pname, h=h, o=o, ranks=rk, scales=sc, A_flat=A_flat,
                              A_off=a_off, B_flat=B_flat, B_off=b_off,
                              x=None, y0=None))  # type: ignore[arg-type]
    xs: Dict[int, np.ndarray] = {}
    for p, (_pn, h, _o, grp) in zip(out, projs):
        if grp not in xs:
            xs[grp] = _normal(rng, (T_, h), 1.0, "variance", spec.dtype)
        p.x = xs[grp]
    for p in out:
        if delta_only:
            p.y0 = np.zeros((T_, p.o), dtype=np.uint16 if spec.dtype == "bf16" else np.float32)
        else:
            p.y0 = _normal(rng, (T_, p.o), 1.0, "variance", spec.dtype)
    return Workload(spec=spec, seed=seed, reading=reading, delta_only=delta_only,
                    dtype=spec.dtype, T=T_, n=n_, ids=ids, projections=out)


def random_intermediate(T: int, R: int, seed: int) -> np.ndarray:
    """A seeded fp32 rank-space intermediate ``v[T, R]`` for expand-only runs."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((T, R)).astype(np.float32)


SIGMA_KINDS = ("none", "full", "diag")


def draw_sigma(ranks: np.ndarray, kind: str, seed: int) -> List[np.ndarray]:
    """Seeded fp32 Sigma_i for the three-stage (compressed) form, one per adapter: "full" is
    r_i x r_i with entries of variance 1/r_i (so Sigma_i u keeps the scale of u), "diag" is
    r_i entries of variance 1.  Values are drawn in fp64 and rounded to fp32."""
    if kind not in ("full", "diag"):
        raise ValueError(kind)
    rng = np.random.default_rng(seed)
    out = []
    for r in np.asarray(ranks, dtype=np.int64):
        r = int(r)
        if kind == "full":
            out.append((rng.standard_normal((r, r)) * np.sqrt(1.0 / r)).astype(np.float32))
        else:
            out.append(rng.standard_normal(r).astype(np.float32))
    return out


def jd_clusters(n: int, clusters: int) -> np.ndarray:
    """Cluster of each adapter for compressed serving with shared A and B: adapter i belongs
    to cluster i mod clusters, and every member uses its cluster leader's (adapter c's)
    A and B."""
    return (np.arange(n) % max(1, clusters)).astype(np.int32)


def draw_merge(ids: np.ndarray, n: int, K: int, seed: int, empty: float = 0.0):
    """Per-token adapter ensembles for the merged form: slot 0 keeps the batch's ids, slots
    1..K-1 draw adapters uniformly from [0, n) (a fraction ``empty`` of them left empty, -1),
    and each token's weights are uniform on (0, 1] normalised to sum to 1 over its filled
    slots.  Returns (ids [T, K] int32, w [T, K] fp32)."""
    rng = np.random.default_rng(seed)
    T = len(ids)
    out = np.empty((T, K), dtype=np.int32)
    out[:, 0] = ids
    if K > 1:
        out[:, 1:] = rng.integers(0, n, size=(T, K - 1))
        if empty > 0:
            drop = rng.random((T, K - 1)) < empty
            out[:, 1:][drop] = -1
    w = rng.uniform(1e-3, 1.0, size=(T, K))
    w[out < 0] = 0.0
    tot = w.sum(axis=1, keepdims=True)
    w = np.where(tot > 0, w / np.where(tot > 0, tot, 1.0), 0.0)
    return out, w.astype(np.float32)


def sweep_ids(T: int, n: int, distinct: int, seed: int) -> np.ndarray:
    """Ids of a batch of T tokens that touch exactly ``distinct`` adapters out of n (distinct
    <= min(T, n)): a seeded random subset of adapters, each carrying floor(T/distinct) or
    ceil(T/distinct) tokens, in a seeded random token order.  Used to vary the number of
    distinct adapters at a fixed batch size."""
    if not 1 <= distinct <= min(T, n):
        raise ValueError("distinct must lie in [1, min(T, n)]")
    rng = np.random.default_rng(seed)
    chosen = rng.choice(n, size=distinct, replace=False)
    ids = np.resize(chosen, T)          # every chosen adapter at least once
    rng.shuffle(ids)
    return np.ascontiguousarray(ids, dtype=np.int32)


def draw_base_weight(o: int, h: int, seed: int, dtype: str = "bf16", reading: str = "variance") -> np.ndarray:
    """Seeded frozen base weight W [o, h] (a linear layer's orientation) for the fused layer
    output: entries N(0, 1/h), so x W^T keeps the unit scale of x, drawn in fp64 and rounded
    to fp32, then to bf16."""
    rng = np.random.default_rng(seed)
    return _normal(rng, (o, h), 1.0 / h, reading, dtype)
