"""Pins for the CPU oracle: closed forms, invariants and brute force that the LoRA
definition and the pages fix.  None of these re-types the oracle's loop; each is chosen so
that a plausible slip in the oracle (a dropped term, a transposed operand, a wrong index, the
scale on the wrong step) fails at least one of them.

Definition pinned: per token, y = y0 + s_i * B_i (A_i x) with i the token's adapter
("TGI Multi-LoRA" page, "Technical Foundation: LoRA"; "Compress then Serve" review thread,
add_lora_slice pseudocode: A with scale 1 into an fp32 buffer, then B with the scale into a
slice of y).
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import oracle.brute as brute
import workloads
from workloads import accounting, bf16_bits_to_f32, f32_to_bf16_bits, to_float64

HERE = os.path.dirname(os.path.abspath(__file__))


def _adapters(p, n):
    return [p.A(i) for i in range(n)], [p.B(i) for i in range(n)]


SMALL = {
    "tiny_sgmv": {},
    "decode_bgmv": dict(shapes=[("q", 512, 384, 0)]),
    "multirank_decode": dict(T=96, n=24, shapes=[("q", 256, 320, 0)]),
    "prefill_sgmv": dict(n=3, seg_len=130, shapes=[("up", 256, 448, 0)]),
    "many_adapter_qkvo": dict(T=64, n=50, shapes=[("q", 256, 256, 0), ("k", 256, 64, 0),
                                                  ("v", 256, 64, 0), ("o", 256, 256, 1)]),
}


@pytest.mark.parametrize("name", workloads.WORKLOAD_NAMES)
@pytest.mark.parametrize("delta_only", [False, True])
def test_loop_matches_grouped_matrix_products(name, delta_only):
    wl = workloads.generate(name, delta_only=delta_only, **SMALL[name])
    for p in wl.projections:
        A, B = _adapters(p, wl.n)
        ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
        alt = brute.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
        scale = max(np.abs(alt).max(), 1e-30)
        assert np.abs(ref - alt).max() <= 1e-12 * scale


@pytest.mark.parametrize("name", ["tiny_sgmv", "decode_bgmv"])
def test_single_adapter_equals_merged_weight(name):
    """A batch whose tokens all use adapter 0 equals y0 + x (W_delta)^T with the merged
    weight W_delta = s * B A formed first (o x h), the LoRA merge of the definition."""
    over = {} if name == "tiny_sgmv" else dict(shapes=[("q", 384, 256, 0)], T=12)
    wl = workloads.generate(name, **over)
    p = wl.projections[0]
    ids = np.zeros(wl.T, dtype=np.int32)
    A, B = _adapters(p, wl.n)
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, ids, A, B, p.scales)
    s = float(p.scales[0])
    dW = s * (to_float64(B[0], wl.dtype) @ to_float64(A[0], wl.dtype))
    merged = to_float64(p.y0, wl.dtype) + to_float64(p.x, wl.dtype) @ dW.T
    assert np.allclose(ref, merged, rtol=0, atol=1e-12 * np.abs(merged).max())


def _int_store(a, dtype):
    a = np.asarray(a, dtype=np.float32)
    return f32_to_bf16_bits(a) if dtype == "bf16" else a


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("h,r,o", [(8, 8, 8), (24, 8, 16), (16, 4, 40)])
def test_selection_matrices_closed_form(dtype, h, r, o):
    """A_i selects coordinates pa (A[k, pa[k]] = 1), B_i selects rank slots pb
    (B[n, pb[n]] = 1): the delta is exactly s * x[t, pa[pb[n]]].  A transposed or mis-indexed
    operand selects different coordinates."""
    rng = np.random.default_rng(7)
    T = 5
    pa = rng.permutation(h)[:r]
    pb = rng.integers(0, r, size=o)
    A = np.zeros((r, h), np.float32)
    A[np.arange(r), pa] = 1
    B = np.zeros((o, r), np.float32)
    B[np.arange(o), pb] = 1
    x = rng.integers(-8, 9, size=(T, h)).astype(np.float32)
    y0 = rng.integers(-8, 9, size=(T, o)).astype(np.float32)
    s = 0.5
    ids = np.zeros(T, np.int32)
    ref = oracle.lora_delta(dtype, _int_store(x, dtype), _int_store(y0, dtype), ids,
                            [_int_store(A, dtype)], [_int_store(B, dtype)], [s])
    want = y0.astype(np.float64) + s * x[:, pa[pb]].astype(np.float64)
    assert np.array_equal(ref, want)


def test_rank_one_closed_form():
    """All rows of A equal u and all columns of B equal w: delta = s * r * (u . x) * w."""
    rng = np.random.default_rng(11)
    T, h, r, o = 6, 32, 5, 12
    u = rng.integers(-3, 4, size=h).astype(np.float32)
    w = rng.integers(-3, 4, size=o).astype(np.float32)
    A = np.tile(u, (r, 1))
    B = np.tile(w[:, None], (1, r))
    x = rng.integers(-4, 5, size=(T, h)).astype(np.float32)
    y0 = rng.integers(-4, 5, size=(T, o)).astype(np.float32)
    s = 0.25
    ref = oracle.lora_delta("f32", x, y0, np.zeros(T, np.int32), [A], [B], [s])
    want = y0 + s * r * (x @ u)[:, None] * w[None, :]
    assert np.array_equal(ref, want.astype(np.float64))


@pytest.mark.parametrize("which", ["B", "s"])
def test_zero_B_or_zero_scale_leaves_y_unchanged(which):
    wl = workloads.generate("multirank_decode", **SMALL["multirank_decode"])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    sc = np.array(p.scales)
    if which == "B":
        B = [np.zeros_like(b) for b in B]
    else:
        sc = np.zeros_like(sc)
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, sc)
    assert np.array_equal(ref, to_float64(p.y0, wl.dtype))


def test_delta_linear_in_scale():
    """Doubling s doubles the delta exactly (a power-of-two scale is exact in fp64); a
    scale applied twice, or to both steps, breaks this."""
    wl = workloads.generate("multirank_decode", delta_only=True, **SMALL["multirank_decode"])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    d1 = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    d2 = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, 2 * p.scales)
    assert np.array_equal(d2, 2 * d1)
    assert np.abs(d1).max() > 0


def test_token_permutation_permutes_output():
    wl = workloads.generate("many_adapter_qkvo", **SMALL["many_adapter_qkvo"])
    p = wl.projections[1]
    A, B = _adapters(p, wl.n)
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    perm = np.random.default_rng(3).permutation(wl.T)
    ref_p = oracle.lora_delta(wl.dtype, p.x[perm], p.y0[perm], wl.ids[perm], A, B, p.scales)
    assert np.array_equal(ref_p, ref[perm])


def test_mixed_ranks_equal_per_adapter_runs():
    """The multi-rank batch equals, row for row, batches that each carry one adapter
    (all other tokens without adapter)."""
    wl = workloads.generate("multirank_decode", **SMALL["multirank_decode"])
    p = wl.projections[0]
    assert len(set(p.ranks.tolist())) > 1
    A, B = _adapters(p, wl.n)
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    for i in np.unique(wl.ids):
        ids_i = np.where(wl.ids == i, wl.ids, -1).astype(np.int32)
        one = oracle.lora_delta(wl.dtype, p.x, p.y0, ids_i, A, B, p.scales)
        rows = wl.ids == i
        assert np.array_equal(one[rows], ref[rows])
        assert np.array_equal(one[~rows], to_float64(p.y0, wl.dtype)[~rows])


def test_zero_padding_rank_changes_nothing():
    wl = workloads.generate("multirank_decode", **SMALL["multirank_decode"])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    R = int(p.ranks.max())
    Ap = [np.concatenate([a, np.zeros((R - a.shape[0], a.shape[1]), a.dtype)]) for a in A]
    Bp = [np.concatenate([b, np.zeros((b.shape[0], R - b.shape[1]), b.dtype)], axis=1) for b in B]
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    pad = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, Ap, Bp, p.scales)
    assert np.array_equal(ref, pad)


def test_no_adapter_rows_and_bad_ids():
    wl = workloads.generate("tiny_sgmv")
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    ids = wl.ids.copy()
    ids[::3] = -1
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, ids, A, B, p.scales)
    assert np.array_equal(ref[ids < 0], p.y0[ids < 0].astype(np.float64))
    for bad in (wl.n, -2):
        ids2 = wl.ids.copy()
        ids2[1] = bad
        with pytest.raises(oracle.OracleError):
            oracle.lora_delta(wl.dtype, p.x, p.y0, ids2, A, B, p.scales)
        with pytest.raises(oracle.OracleError):
            oracle.build_segments(ids2, wl.n)


def test_output_slice_offset():
    """The delta lands in columns [y_offset, y_offset + o) of a wider y (the fused-output
    slice of the pseudocode); the oracle reads y0 only there."""
    wl = workloads.generate("tiny_sgmv")
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    wide = np.random.default_rng(5).standard_normal((wl.T, 3 * p.o)).astype(np.float32)
    wide[:, 96:96 + p.o] = p.y0
    ref_off = oracle.lora_delta(wl.dtype, p.x, wide, wl.ids, A, B, p.scales, y_offset=96, o=p.o)
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    assert np.array_equal(ref_off, ref)


def test_exhaustive_tiny_against_outer_products():
    """T = 3 tokens, two adapters of ranks 2 and 3 plus "no adapter": every one of the
    3**3 id assignments, integer inputs, compared exactly with W_i = s_i * sum_k
    outer(B_i[:, k], A_i[k, :]) in rational arithmetic."""
    rng = np.random.default_rng(13)
    T, h, o = 3, 4, 5
    ranks = [2, 3]
    A = [rng.integers(-3, 4, size=(r, h)).astype(np.float32) for r in ranks]
    B = [rng.integers(-3, 4, size=(o, r)).astype(np.float32) for r in ranks]
    s = [Fraction(1, 2), Fraction(3, 1)]
    x = rng.integers(-3, 4, size=(T, h)).astype(np.float32)
    y0 = rng.integers(-3, 4, size=(T, o)).astype(np.float32)
    W = []
    for i in range(2):
        Wi = [[Fraction(0)] * h for _ in range(o)]
        for k in range(ranks[i]):
            for n_ in range(o):
                for j in range(h):
                    Wi[n_][j] += s[i] * int(B[i][n_, k]) * int(A[i][k, j])
        W.append(Wi)
    for combo in itertools.product([-1, 0, 1], repeat=T):
        ids = np.array(combo, np.int32)
        ref = oracle.lora_delta("f32", x, y0, ids, A, B, [float(v) for v in s])
        for t in range(T):
            for n_ in range(o):
                want = Fraction(int(y0[t, n_]))
                if ids[t] >= 0:
                    want += sum(W[ids[t]][n_][j] * int(x[t, j]) for j in range(h))
                assert Fraction(ref[t, n_]) == want


def test_shrink_and_expand_steps():
    """Shrink alone against a library product; expand alone against a library product on a
    given fp32 intermediate; shrink then expand (fp32 intermediate) against the delta."""
    wl = workloads.generate("multirank_decode", **SMALL["multirank_decode"])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    R = int(p.ranks.max())
    v = oracle.lora_shrink(wl.dtype, p.x, wl.ids, A, ldv=R)
    xd = to_float64(p.x, wl.dtype)
    for t in range(wl.T):
        i = wl.ids[t]
        r = p.ranks[i]
        want = to_float64(A[i], wl.dtype) @ xd[t]
        assert np.allclose(v[t, :r], want, rtol=0, atol=1e-12 * max(1.0, np.abs(want).max()))
        assert not v[t, r:].any()
    v32 = workloads.random_intermediate(wl.T, R, seed=9)
    e = oracle.lora_expand(wl.dtype, v32, p.y0, wl.ids, B, p.scales)
    y0d = to_float64(p.y0, wl.dtype)
    for t in range(wl.T):
        i = wl.ids[t]
        r = p.ranks[i]
        want = y0d[t] + float(p.scales[i]) * (to_float64(B[i], wl.dtype) @ v32[t, :r].astype(np.float64))
        assert np.allclose(e[t], want, rtol=0, atol=1e-12 * np.abs(want).max())
    full = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    composed = oracle.lora_expand(wl.dtype, v.astype(np.float32), p.y0, wl.ids, B, p.scales)
    assert np.abs(composed - full).max() <= 1e-6 * np.abs(full).max()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_segments_equal_stable_argsort(seed):
    rng = np.random.default_rng(seed)
    n = [1, 7, 1000][seed]
    T = [0, 33, 4096][seed]
    ids = rng.integers(-1, n, size=T).astype(np.int32)
    perm, seg_ptr, seg_adapter = oracle.build_segments(ids, n)
    valid = np.nonzero(ids >= 0)[0]
    order = valid[np.argsort(ids[valid], kind="stable")]
    assert np.array_equal(perm, order)
    uniq, counts = np.unique(ids[valid], return_counts=True)
    assert np.array_equal(seg_adapter, uniq)
    assert np.array_equal(seg_ptr, np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))


def test_segments_of_workloads():
    for name in ("decode_bgmv", "multirank_decode", "many_adapter_qkvo"):
        wl = workloads.generate(name, shapes=[("q", 8, 8, 0)])
        perm, seg_ptr, seg_adapter = oracle.build_segments(wl.ids, wl.n)
        for s in range(len(seg_adapter)):
            toks = perm[seg_ptr[s]:seg_ptr[s + 1]]
            assert (wl.ids[toks] == seg_adapter[s]).all()
            assert (np.diff(toks) > 0).all()
        assert (np.diff(seg_adapter) > 0).all()


def test_page_size_figures_pin_byte_accounting():
    g = json.load(open(os.path.join(HERE, "golden", "page_sizes.json")))
    m = g["mistral7b"]
    shapes = {"q": (m["hidden"], m["hidden"]), "k": (m["hidden"], m["kv_out"]),
              "v": (m["hidden"], m["kv_out"]), "o": (m["hidden"], m["hidden"])}
    b = accounting.adapter_bytes([shapes[p] for p in g["reading_projections"]],
                                 g["reading_rank"], m["layers"], 2)
    assert round(b / 1e6, 1) == g["adapter_mb"]
    assert b / (g["base_gb"] * 1e9) < g["adapter_over_base_below"]
    inc = g["n_adapters_for_vram_claim"] * g["adapter_mb"] / (g["base_gb"] * 1e3)
    assert abs(inc - g["vram_increase_roughly"]) < 0.005


def test_workload_byte_accounting_counts_distinct_adapters():
    wl = workloads.generate("decode_bgmv", shapes=[("q", 64, 32, 0)])
    d = np.unique(wl.ids)
    e = 2
    want = wl.T * 64 * e + 2 * wl.T * 32 * e + len(d) * 16 * (64 + 32) * e
    assert accounting.workload_bytes(wl) == want


def test_recipe_is_deterministic_and_rounded():
    a = workloads.generate("decode_bgmv", shapes=[("q", 64, 32, 0)])
    b = workloads.generate("decode_bgmv", shapes=[("q", 64, 32, 0)])
    assert np.array_equal(a.ids, b.ids)
    assert np.array_equal(a.projections[0].A_flat, b.projections[0].A_flat)
    x32 = bf16_bits_to_f32(a.projections[0].x)
    assert np.array_equal(f32_to_bf16_bits(x32), a.projections[0].x)
    # variance vs std reading of N(0, 1/4096): std 1/64 vs 1/4096
    s_var = np.std(bf16_bits_to_f32(a.projections[0].A_flat))
    c = workloads.generate("decode_bgmv", shapes=[("q", 64, 32, 0)], reading="std")
    s_std = np.std(bf16_bits_to_f32(c.projections[0].A_flat))
    assert 0.8 / 64 < s_var < 1.2 / 64 and 0.8 / 4096 < s_std < 1.2 / 4096
    z = workloads.generate("multirank_decode", shapes=[("q", 8, 8, 0)])
    counts = np.bincount(z.ids, minlength=z.n)
    assert counts[0] == counts.max() and set(z.projections[0].ranks) <= {8, 16, 32, 64}
    pf = workloads.generate("prefill_sgmv", shapes=[("up", 8, 8, 0)])
    assert np.array_equal(pf.ids, np.repeat(np.arange(8), 512))


# ------------------------------------------------------------------ three-stage form (Sigma)
# "Compress then Serve" review thread, add_lora_slice_with_sigma pseudocode: A with scale 1,
# then the adapter's Sigma with scale 1, then B with the scale into the y slice.

def _sigma_case(dtype="bf16"):
    if dtype == "f32":
        wl = workloads.generate("tiny_sgmv", T=30, n=5)
    else:
        wl = workloads.generate("multirank_decode", T=40, n=7, shapes=[("q", 192, 136, 0)], ranks=(3, 8, 16))
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    return wl, p, A, B


@pytest.mark.parametrize("kind", ["full", "diag"])
def test_sigma_identity_is_the_plain_delta(kind):
    """Sigma_i = I (full) or all ones (diagonal) multiplies by exactly 1 and adds exact zeros,
    so the three-stage result equals the two-stage one bit for bit."""
    wl, p, A, B = _sigma_case()
    sig = [np.eye(a.shape[0], dtype=np.float32) if kind == "full" else np.ones(a.shape[0], np.float32) for a in A]
    plain = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    three = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales,
                                    oracle.SIGMA_FULL if kind == "full" else oracle.SIGMA_DIAG, sig)
    assert np.array_equal(plain, three)


def test_sigma_diagonal_of_powers_of_two_folds_into_B():
    """A diagonal Sigma of powers of two can be folded into B exactly (B' = B diag(d), every
    product exact in fp32): the three-stage result equals the plain one with B'."""
    wl, p, A, B = _sigma_case("f32")
    rng = np.random.default_rng(3)
    d = [np.ldexp(1.0, rng.integers(-3, 4, size=a.shape[0])).astype(np.float32) for a in A]
    Bf = [(b * di[None, :]).astype(np.float32) for b, di in zip(B, d)]
    plain = oracle.lora_delta("f32", p.x, p.y0, wl.ids, A, Bf, p.scales)
    three = oracle.lora_delta_sigma("f32", p.x, p.y0, wl.ids, A, B, p.scales, oracle.SIGMA_DIAG, d)
    assert np.array_equal(plain, three)


@pytest.mark.parametrize("kind", ["full", "diag"])
def test_sigma_equals_merged_three_factor_weight(kind):
    """Per token, y = y0 + s_i (B_i Sigma_i A_i) x with the o x h product formed first in
    fp64 (a different evaluation order); a non-symmetric Sigma catches a transposed Sigma."""
    wl, p, A, B = _sigma_case()
    sig = workloads.draw_sigma(p.ranks, kind, seed=11)
    got = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales,
                                  oracle.SIGMA_FULL if kind == "full" else oracle.SIGMA_DIAG, sig)
    x = to_float64(p.x, wl.dtype)
    want = to_float64(p.y0, wl.dtype).copy()
    for i in range(wl.n):
        S = sig[i].astype(np.float64)
        S = S if kind == "full" else np.diag(S)
        W = float(p.scales[i]) * (to_float64(B[i], wl.dtype) @ S @ to_float64(A[i], wl.dtype))
        rows = wl.ids == i
        want[rows] += x[rows] @ W.T
    scale = np.abs(want).max()
    assert np.abs(got - want).max() <= 1e-12 * scale


def test_sigma_delta_linear_in_sigma():
    """Doubling every Sigma_i doubles the delta exactly (delta-only: y0 = 0)."""
    wl = workloads.generate("multirank_decode", delta_only=True, T=24, n=5, shapes=[("q", 128, 96, 0)])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    sig = workloads.draw_sigma(p.ranks, "full", seed=2)
    one = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, oracle.SIGMA_FULL, sig)
    two = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, oracle.SIGMA_FULL,
                                  [2 * s for s in sig])
    assert np.array_equal(2 * one, two)


def test_sigma_shrink_is_sigma_times_shrink():
    """Steps 1 and 2 alone: v = Sigma_i (A_i x), against numpy applying Sigma to the plain
    shrink (closed form); tokens without an adapter give zero rows."""
    wl, p, A, B = _sigma_case()
    ids = wl.ids.copy()
    ids[::7] = -1
    sig = workloads.draw_sigma(p.ranks, "full", seed=4)
    R = int(p.ranks.max())
    got = oracle.lora_shrink_sigma(wl.dtype, p.x, ids, A, oracle.SIGMA_FULL, sig, ldv=R)
    x = to_float64(p.x, wl.dtype)
    for t in range(wl.T):
        i = ids[t]
        if i < 0:
            assert not got[t].any()
            continue
        r = A[i].shape[0]
        u = to_float64(A[i], wl.dtype) @ x[t]
        w = sig[i].astype(np.float64) @ u
        assert np.abs(got[t, :r] - w).max() <= 1e-12 * max(np.abs(w).max(), 1e-30)
        assert not got[t, r:].any()


def test_sigma_shared_cluster_weights():
    """Compressed serving shares A and B inside a cluster: adapters that point at the same
    A_c, B_c and differ only in Sigma_i give, per token, y0 + s (B_c Sigma_i A_c) x."""
    wl, p, A, B = _sigma_case()
    cl = workloads.jd_clusters(wl.n, 2)
    # members use their leader's weights (same rank inside a cluster by construction here)
    ranks = np.array([A[c].shape[0] for c in cl])
    A2 = [A[c] for c in cl]
    B2 = [B[c] for c in cl]
    sig = workloads.draw_sigma(ranks, "full", seed=8)
    got = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A2, B2, p.scales, oracle.SIGMA_FULL, sig)
    x = to_float64(p.x, wl.dtype)
    want = to_float64(p.y0, wl.dtype).copy()
    for i in range(wl.n):
        W = float(p.scales[i]) * (to_float64(B2[i], wl.dtype) @ sig[i].astype(np.float64) @
                                  to_float64(A2[i], wl.dtype))
        rows = wl.ids == i
        want[rows] += x[rows] @ W.T
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


# ------------------------------------------------------------------ merged adapters per token
# "Lorax" pages: adapters merged per request into a weighted ensemble.  Reading: the merge is
# the weighted sum of the adapters' deltas, y = y0 + sum_j w_j s_j B_j A_j x.

def _merge_case(K=3, empty=0.25, seed=1):
    wl = workloads.generate("multirank_decode", T=36, n=9, shapes=[("q", 160, 96, 0)], ranks=(4, 8, 16))
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    ids, w = workloads.draw_merge(wl.ids, wl.n, K, seed, empty=empty)
    return wl, p, A, B, ids, w


def test_merged_single_slot_unit_weight_is_the_plain_delta():
    wl, p, A, B, _ids, _w = _merge_case()
    ids = wl.ids.reshape(-1, 1).astype(np.int32)
    w = np.ones_like(ids, dtype=np.float32)
    plain = oracle.lora_delta(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales)
    merged = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids, w, A, B, p.scales)
    assert np.array_equal(plain, merged)


def test_merged_zero_weights_leave_y_unchanged():
    wl, p, A, B, ids, w = _merge_case()
    got = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids, np.zeros_like(w), A, B, p.scales)
    assert np.array_equal(got, to_float64(p.y0, wl.dtype))


def test_merged_equals_merged_weight_closed_form():
    """Per token, y0 + x (sum_j w_j s_j B_j A_j)^T with the o x h ensemble weight formed first
    in fp64: pins the per-slot adapter, weight and scale."""
    wl, p, A, B, ids, w = _merge_case()
    got = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids, w, A, B, p.scales)
    x = to_float64(p.x, wl.dtype)
    want = to_float64(p.y0, wl.dtype).copy()
    Wd = [float(p.scales[i]) * (to_float64(B[i], wl.dtype) @ to_float64(A[i], wl.dtype)) for i in range(wl.n)]
    for t in range(wl.T):
        W = np.zeros_like(Wd[0])
        for j in range(ids.shape[1]):
            if ids[t, j] >= 0:
                W += float(w[t, j]) * Wd[ids[t, j]]
        want[t] += W @ x[t]
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


def test_merged_slot_order_and_duplicate_slots():
    """Permuting a token's slots, or splitting one slot's weight over two slots of the same
    adapter, changes nothing beyond fp64 rounding."""
    wl, p, A, B, ids, w = _merge_case(K=2, empty=0.0)
    base = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids, w, A, B, p.scales)
    swapped = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids[:, ::-1].copy(), w[:, ::-1].copy(), A, B, p.scales)
    scale = np.abs(base).max()
    assert np.abs(base - swapped).max() <= 1e-13 * scale
    ids3 = np.concatenate([ids, ids[:, :1]], axis=1)
    w3 = np.concatenate([w, np.zeros_like(w[:, :1])], axis=1)
    w3[:, 2] = np.float32(0.5) * w3[:, 0]
    w3[:, 0] = w3[:, 0] - w3[:, 2]   # exact in fp32: halving, then subtracting the half
    split = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids3, w3, A, B, p.scales)
    assert np.abs(base - split).max() <= 1e-13 * scale


def test_merged_empty_slots_and_bad_ids():
    wl, p, A, B, ids, w = _merge_case()
    only0 = ids.copy()
    only0[:, 1:] = -1
    got = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, only0, w, A, B, p.scales)
    w0 = np.where(only0 >= 0, w, 0).astype(np.float32)
    again = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, only0, w0, A, B, p.scales)
    assert np.array_equal(got, again)
    bad = ids.copy()
    bad[3, 1] = wl.n
    with pytest.raises(oracle.OracleError):
        oracle.lora_delta_merged(wl.dtype, p.x, p.y0, bad, w, A, B, p.scales)


@pytest.mark.parametrize("kind", ["full", "diag"])
@pytest.mark.parametrize("delta_only", [False, True])
def test_sigma_loop_matches_grouped_products(kind, delta_only):
    """The C loop's three-stage form against numpy products per adapter group (a different
    evaluation order and code)."""
    wl = workloads.generate("multirank_decode", delta_only=delta_only, T=60, n=11, shapes=[("q", 200, 120, 0)])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    sig = workloads.draw_sigma(p.ranks, kind, seed=13)
    k = oracle.SIGMA_FULL if kind == "full" else oracle.SIGMA_DIAG
    ref = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, k, sig)
    alt = brute.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, k, sig)
    assert np.abs(ref - alt).max() <= 1e-12 * max(np.abs(alt).max(), 1e-30)


@pytest.mark.parametrize("delta_only", [False, True])
def test_merged_loop_matches_grouped_products(delta_only):
    wl = workloads.generate("many_adapter_qkvo", delta_only=delta_only, T=48, n=30,
                            shapes=[("q", 128, 96, 0)])
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    ids, w = workloads.draw_merge(wl.ids, wl.n, 3, seed=6, empty=0.3)
    ref = oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids, w, A, B, p.scales)
    alt = brute.lora_delta_merged(wl.dtype, p.x, p.y0, ids, w, A, B, p.scales)
    assert np.abs(ref - alt).max() <= 1e-12 * max(np.abs(alt).max(), 1e-30)


def test_next_row_generators_are_seeded_and_shaped():
    """Sigma, cluster and ensemble draws: deterministic per seed, the stated shapes and laws."""
    ranks = np.array([4, 8, 16, 64], dtype=np.int32)
    s1 = workloads.draw_sigma(ranks, "full", seed=3)
    s2 = workloads.draw_sigma(ranks, "full", seed=3)
    assert all(np.array_equal(a, b) for a, b in zip(s1, s2))
    assert [a.shape for a in s1] == [(4, 4), (8, 8), (16, 16), (64, 64)]
    assert all(a.dtype == np.float32 for a in s1)
    assert 0.8 / 64 < float(np.var(s1[3])) < 1.2 / 64   # variance 1/r at r = 64
    d = workloads.draw_sigma(ranks, "diag", seed=3)
    assert [a.shape for a in d] == [(4,), (8,), (16,), (64,)]
    assert np.array_equal(workloads.jd_clusters(7, 3), np.array([0, 1, 2, 0, 1, 2, 0]))
    ids = np.arange(50, dtype=np.int32) % 9
    m1, w1 = workloads.draw_merge(ids, 9, 3, seed=5, empty=0.4)
    m2, w2 = workloads.draw_merge(ids, 9, 3, seed=5, empty=0.4)
    assert np.array_equal(m1, m2) and np.array_equal(w1, w2)
    assert m1.shape == w1.shape == (50, 3) and np.array_equal(m1[:, 0], ids)
    assert ((m1 >= -1) & (m1 < 9)).all() and (m1[:, 1:] == -1).any()
    assert (w1[m1 < 0] == 0).all() and (w1[m1 >= 0] > 0).all()
    assert np.allclose(w1.sum(axis=1), 1.0, atol=1e-6)


def test_byte_accounting_of_the_bench_variants():
    """The bench's algorithmic bytes for its option variants, against hand counts: a grouped
    launch reads the shared x once; Sigma adds 4 r^2 (full) or 4 r (diagonal) bytes per touched
    adapter; shared cluster weights count once per touched cluster; one merged slot is the
    plain call."""
    wl = workloads.generate("many_adapter_qkvo", T=40, n=30, shapes=[("q", 64, 64, 0), ("k", 64, 16, 0),
                                                                      ("v", 64, 16, 0), ("o", 64, 64, 1)])
    e = 2
    T_valid = int((wl.ids >= 0).sum())
    base = accounting.workload_bytes(wl)
    assert accounting.workload_bytes(wl, shared_x=True) == base - 2 * T_valid * 64 * e
    d = accounting.distinct_adapters(wl.ids)
    r = wl.projections[0].ranks
    assert accounting.workload_bytes(wl, sigma="full") == base + 4 * 4 * int(sum(int(r[i]) ** 2 for i in d))
    assert accounting.workload_bytes(wl, sigma="diag") == base + 4 * 4 * int(sum(int(r[i]) for i in d))
    C = 7
    leaders = np.unique(d % C)
    w_all = sum(int(r[i]) * (q.h + q.o) * e for i in d for q in wl.projections)
    w_cl = sum(int(r[i]) * (q.h + q.o) * e for i in leaders for q in wl.projections)
    assert accounting.workload_bytes(wl, sigma="diag", clusters=C) == \
        base - w_all + w_cl + 4 * 4 * int(sum(int(r[i]) for i in d))
    one = wl.ids.reshape(-1, 1)
    p = wl.projections[0]
    assert accounting.merged_bytes(wl, one) == accounting.projection_bytes(
        T_valid, p.h, p.o, (p.ranks[i] for i in d), e)


# ------------------------------------------------------------------ fused base product (layer output)
# "TGI Multi-LoRA" page, "Technical Foundation: LoRA": the frozen base weight's product plus
# the adapter's low-rank term; "predibase/lorax" repository page: one forward pass.

def _base_case(seed=3, T=12, h=96, o=80, n=3, ranks=(8, 16, 8), dtype="bf16", minus_one=True):
    wl = workloads.generate("multirank_decode", T=T, n=n, shapes=[("q", h, o, 0)], ranks=ranks, seed=seed)
    ids = wl.ids.copy()
    if minus_one:
        ids[::4] = -1
    W = workloads.draw_base_weight(o, h, seed=seed + 1, dtype=dtype)
    return wl, ids, W


def test_base_with_zero_weight_is_the_delta():
    """W = 0: the layer output is exactly the delta form y0 + s_i B_i A_i x."""
    wl, ids, W = _base_case()
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    zero = np.zeros_like(W)
    got = oracle.lora_base_delta(wl.dtype, p.x, zero, p.y0, ids, A, B, p.scales)
    want = oracle.lora_delta(wl.dtype, p.x, p.y0, ids, A, B, p.scales)
    assert np.array_equal(got, want)


def test_base_single_adapter_equals_merged_weight():
    """Every token on adapter 0: y = y0 + x (W + s B A)^T with the merged weight formed
    first, the LoRA merge of the definition."""
    wl, _ids, W = _base_case(minus_one=False)
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    ids = np.zeros(wl.T, np.int32)
    got = oracle.lora_base_delta(wl.dtype, p.x, W, p.y0, ids, A, B, p.scales)
    Wm = to_float64(W, wl.dtype) + float(p.scales[0]) * (to_float64(B[0], wl.dtype) @ to_float64(A[0], wl.dtype))
    want = to_float64(p.y0, wl.dtype) + to_float64(p.x, wl.dtype) @ Wm.T
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


def test_base_rows_without_adapter_and_accumulate_flag():
    """Id -1 rows get y0 + x W^T only; without accumulate the result ignores y0 and equals
    the accumulated result minus y0."""
    wl, ids, W = _base_case()
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    ids[:] = -1
    got = oracle.lora_base_delta(wl.dtype, p.x, W, p.y0, ids, A, B, p.scales)
    want = to_float64(p.y0, wl.dtype) + to_float64(p.x, wl.dtype) @ to_float64(W, wl.dtype).T
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()
    wl, ids, W = _base_case()
    garbage = workloads.generate("multirank_decode", T=wl.T, n=wl.n, shapes=[("q", 96, 80, 0)],
                                 ranks=(8, 16, 8), seed=99).projections[0].y0
    fresh = oracle.lora_base_delta(wl.dtype, p.x, W, garbage, ids, A, B, p.scales, accumulate=False)
    zero_y0 = oracle.lora_base_delta(wl.dtype, p.x, W, np.zeros_like(p.y0), ids, A, B, p.scales)
    acc = oracle.lora_base_delta(wl.dtype, p.x, W, p.y0, ids, A, B, p.scales)
    assert np.array_equal(fresh, zero_y0)
    assert np.abs((acc - to_float64(p.y0, wl.dtype)) - fresh).max() <= 1e-12 * np.abs(fresh).max()


@pytest.mark.parametrize("h,o", [(24, 16), (16, 40)])
def test_base_selection_matrix_closed_form(h, o):
    """W selects coordinate sel[n] of x (W[n, sel[n]] = 1) and the adapter terms vanish:
    y = y0 + x[:, sel] exactly.  A transposed W (non-square) selects other coordinates."""
    rng = np.random.default_rng(5)
    T = 6
    sel = rng.integers(0, h, size=o)
    W = np.zeros((o, h), np.float32)
    W[np.arange(o), sel] = 1
    x = rng.integers(-8, 9, size=(T, h)).astype(np.float32)
    y0 = rng.integers(-8, 9, size=(T, o)).astype(np.float32)
    A = [np.ones((8, h), np.float32)]
    B = [np.zeros((o, 8), np.float32)]
    ids = np.zeros(T, np.int32)
    got = oracle.lora_base_delta("bf16", _int_store(x, "bf16"), _int_store(W, "bf16"), _int_store(y0, "bf16"), ids,
                                 [_int_store(a, "bf16") for a in A], [_int_store(b, "bf16") for b in B], [2.0])
    assert np.array_equal(got, y0.astype(np.float64) + x[:, sel].astype(np.float64))


def test_base_linear_in_weight_and_matches_grouped_products():
    """Doubling W doubles the base term exactly (power of two); the loop agrees with numpy
    (one library product for the base term, grouped products for the adapters)."""
    wl, ids, W = _base_case(T=20, h=128, o=96, n=4, ranks=(8, 16, 32, 8))
    p = wl.projections[0]
    A, B = _adapters(p, wl.n)
    y0z = np.zeros_like(p.y0)
    Bz = [np.zeros_like(b) for b in B]
    one = oracle.lora_base_delta(wl.dtype, p.x, W, y0z, ids, A, Bz, p.scales)
    W2 = f32_to_bf16_bits(2 * bf16_bits_to_f32(W))
    two = oracle.lora_base_delta(wl.dtype, p.x, W2, y0z, ids, A, Bz, p.scales)
    assert np.array_equal(two, 2 * one)
    for acc in (True, False):
        got = oracle.lora_base_delta(wl.dtype, p.x, W, p.y0, ids, A, B, p.scales, accumulate=acc)
        alt = brute.lora_base_delta(wl.dtype, p.x, W, p.y0, ids, A, B, p.scales, accumulate=acc)
        assert np.abs(got - alt).max() <= 1e-12 * np.abs(alt).max()
