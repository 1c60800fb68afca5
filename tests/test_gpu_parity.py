"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element,
on the same seeded inputs.  Tolerance: |gpu - ref| <= 1e-2 * max|ref| + 1e-3 (bf16 in, fp32
accumulate, one rounding of the output).  Index bookkeeping must match bit for bit."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, option, reference, workload
from workloads import to_float64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L._load()   # the CUDA library must be present: no fallback
    yield
    L.lora_set_option("split", 0)
    L.lora_set_option("pdl", 1)
    L.lora_set_option("decode_cluster", 0)


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("delta_only", [False, True])
def test_tiny_sgmv_fp32(delta_only):
    wl = workload("tiny_sgmv", delta_only)
    ref = reference("tiny_sgmv", delta_only)
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), ref, wl.dtype, "tiny sgmv")
    y2 = dp.bgmv(dp.y())
    assert_close(dp.to_np(y2), ref, wl.dtype, "tiny bgmv")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("delta_only", [False, True])
def test_decode_bgmv_q_proj(delta_only):
    """The benchmarked call: per-token ids, 64 tokens over 32 rank-16 adapters, 4096 -> 4096."""
    wl = workload("decode_bgmv", delta_only)
    ref = reference("decode_bgmv", delta_only)
    dp = DeviceProj(wl)
    y = dp.bgmv(dp.y())
    assert_close(dp.to_np(y), ref, wl.dtype, "decode bgmv")
    seg, _keep = dp.segments()
    y2 = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y2), ref, wl.dtype, "decode sgmv")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("delta_only", [False, True])
def test_multirank_decode(delta_only):
    wl = workload("multirank_decode", delta_only)
    ref = reference("multirank_decode", delta_only)
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), ref, wl.dtype, "multirank sgmv")
    y2 = dp.bgmv(dp.y())
    assert_close(dp.to_np(y2), ref, wl.dtype, "multirank bgmv")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("delta_only", [False, True])
def test_prefill_sgmv_contiguous(delta_only):
    """8 contiguous segments of 512 tokens, rank 64, 4096 -> 14336; segments passed without
    a permutation (prefill layout), with the long-segment hint."""
    wl = workload("prefill_sgmv", delta_only)
    ref = reference("prefill_sgmv", delta_only)
    dp = DeviceProj(wl)
    n = wl.n
    seg_ptr = torch.arange(0, wl.T + 1, 512, dtype=torch.int32, device="cuda")
    seg_adapter = torch.arange(n, dtype=torch.int32, device="cuda")
    num = torch.tensor([n], dtype=torch.int32, device="cuda")
    seg = L.make_segments(None, seg_ptr, seg_adapter, num, wl.T, n, 512)
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), ref, wl.dtype, "prefill sgmv")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("delta_only", [False, True])
def test_many_adapter_four_projections_share_segments(delta_only):
    """1000 rank-16 adapters on q, k, v, o; one segment table built once, four calls."""
    wl = workload("many_adapter_qkvo", delta_only)
    dps = [DeviceProj(wl, i) for i in range(4)]
    seg, _keep = dps[0].segments()
    ys = [dp.sgmv(dp.y(), seg) for dp in dps]
    for i, (dp, y) in enumerate(zip(dps, ys)):
        ref = reference("many_adapter_qkvo", delta_only, "variance", i)
        assert_close(dp.to_np(y), ref, wl.dtype, "qkvo proj %d" % i)
        assert dp.status() == (0, 0)


@pytest.mark.parametrize("name", ["decode_bgmv", "multirank_decode", "tiny_sgmv"])
def test_std_reading_of_the_weight_law(name):
    """N(0, v) read as standard deviation v: a much smaller delta, still within tolerance of
    the delta-only run."""
    wl = workload(name, True, "std")
    ref = reference(name, True, "std")
    dp = DeviceProj(wl)
    y = dp.bgmv(dp.y())
    assert np.abs(ref).max() > 0
    assert_close(dp.to_np(y), ref, wl.dtype, "std reading")


# ------------------------------------------------------------------ bookkeeping (bit-exact)

@pytest.mark.parametrize("case", ["decode_bgmv", "multirank_decode", "many_adapter_qkvo", "prefill_sgmv",
                                  "edge_empty", "edge_one", "edge_all_none", "edge_max_T", "edge_large_n",
                                  "edge_single_adapter", "edge_count_max", "edge_sort_T", "edge_sort_n",
                                  "edge_heavy", "edge_count_max_T", "edge_radix_T", "edge_heavy_2048"])
def test_build_segments_bit_exact(case):
    """Both bookkeeping kernels (counting sort up to 512 tokens and 8191 adapters, radix sort
    beyond) against the oracle's stable counting sort, including both sides of the switch."""
    rng = np.random.default_rng(17)
    if case.startswith("edge"):
        n, T = {"edge_empty": (5, 0), "edge_one": (5, 1), "edge_all_none": (7, 300),
                "edge_max_T": (1000, L.LORA_MAX_SEGMENT_TOKENS), "edge_large_n": (70000, 3000),
                "edge_single_adapter": (1, 777), "edge_count_max": (8191, 2048), "edge_sort_T": (100, 2049),
                "edge_sort_n": (8192, 2048), "edge_heavy": (5, 512), "edge_count_max_T": (8191, 512),
                "edge_radix_T": (100, 513), "edge_heavy_2048": (5, 2048)}[case]
        ids = rng.integers(-1, n, size=T).astype(np.int32)
        if case == "edge_all_none":
            ids[:] = -1
        if case.startswith("edge_heavy"):   # one adapter carries most tokens: long runs of equal ids
            ids[rng.random(T) < 0.9] = 2
        wl = workload("tiny_sgmv")
        dp = DeviceProj(wl)
        # a table with n adapters that all alias adapter 0's weights (bookkeeping only)
        table = L.AdapterTable([dp.d.A_ptrs[0]] * n, [dp.d.B_ptrs[0]] * n, [8] * n, [1.0] * n, 256, 256,
                               L.LORA_F32, keep=dp)
    else:
        wl = workload(case, shapes=(("q", 64, 64, 0),))
        n, T, ids = wl.n, wl.T, wl.ids
        dp = DeviceProj(wl)
        table = dp.table
    d_ids = torch.from_numpy(ids).cuda() if T else torch.empty(1, dtype=torch.int32, device="cuda")
    perm = torch.full((max(T, 1),), -7, dtype=torch.int32, device="cuda")
    seg_ptr = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    seg_adapter = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    num = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    L.lora_build_segments(table.handle, d_ids, T, perm, seg_ptr, seg_adapter, num)
    torch.cuda.synchronize()
    want_perm, want_ptr, want_ad = oracle.build_segments(ids, n)
    S = int(num.item())
    assert S == len(want_ad)
    assert np.array_equal(seg_ptr[:S + 1].cpu().numpy(), want_ptr)
    assert np.array_equal(seg_adapter[:S].cpu().numpy(), want_ad)
    assert np.array_equal(perm[:len(want_perm)].cpu().numpy(), want_perm)
    rc, word = L.lora_get_status(table.handle)
    assert (rc, word) == (0, 0)


def test_build_segments_flags_bad_ids():
    wl = workload("decode_bgmv", shapes=(("q", 64, 64, 0),))
    dp = DeviceProj(wl)
    ids = wl.ids.copy()
    ids[[3, 10]] = [wl.n, -5]
    d_ids = torch.from_numpy(ids).cuda()
    seg, t = dp.segments(d_ids)
    torch.cuda.synchronize()
    good = ids.copy()
    good[[3, 10]] = -1
    want_perm, want_ptr, want_ad = oracle.build_segments(good, wl.n)
    S = int(t["num_segs"].item())
    assert np.array_equal(t["seg_ptr"][:S + 1].cpu().numpy(), want_ptr)
    assert np.array_equal(t["perm"][:len(want_perm)].cpu().numpy(), want_perm)
    rc, word = dp.status()
    assert rc == L.LORA_ERR_DEVICE_STATUS and word & L.LORA_STATUS_BAD_ID


# ------------------------------------------------------------------ invariants on the device

def _small(name, **kw):
    shapes = {"decode_bgmv": (("q", 1024, 768, 0),), "multirank_decode": (("q", 2048, 1536, 0),)}[name]
    return workloads.generate(name, shapes=shapes, **kw)


@pytest.mark.parametrize("path", ["bgmv", "sgmv", "split"])
def test_zero_B_and_zero_scale_leave_y_bit_identical(path):
    wl = _small("multirank_decode")
    p = wl.projections[0]
    p.B_flat = np.zeros_like(p.B_flat)
    dp = DeviceProj(wl)
    L.lora_set_option("split", 1 if path == "split" else 0)
    try:
        y = dp.y()
        if path == "bgmv":
            dp.bgmv(y)
        else:
            seg, _k = dp.segments()
            dp.sgmv(y, seg)
        assert torch.equal(y, dp.d.y0)
    finally:
        L.lora_set_option("split", 0)
    wl2 = _small("decode_bgmv")
    wl2.projections[0].scales[:] = 0
    dp2 = DeviceProj(wl2)
    y2 = dp2.bgmv(dp2.y())
    assert torch.equal(y2, dp2.d.y0)


@pytest.mark.parametrize("cluster", [1, 2, 4, 8])
def test_paths_agree_bit_for_bit(cluster):
    """At one cluster width, BGMV, SGMV (fused) and shrink-then-expand through the fp32
    workspace perform the same per-token arithmetic in the same order, so they agree exactly;
    repeated runs too."""
    wl = _small("multirank_decode")
    dp = DeviceProj(wl)
    with option("decode_cluster", cluster):
        y_b = dp.bgmv(dp.y())
        seg, _k = dp.segments()
        y_s = dp.sgmv(dp.y(), seg)
        with option("split", 1):
            y_x = dp.sgmv(dp.y(), seg)
        y_b2 = dp.bgmv(dp.y())
    assert torch.equal(y_b, y_s)
    assert torch.equal(y_b, y_x)
    assert torch.equal(y_b, y_b2)
    ref = oracle.workload_reference(wl)
    assert_close(dp.to_np(y_b), ref, wl.dtype, "small multirank")


@pytest.mark.parametrize("name", ["multirank_decode", "many_adapter_qkvo"])
def test_balanced_runs_and_stride_agree_bit_for_bit(name):
    """Segment-table units dealt to the clusters as runs of about equal estimated work or with a
    fixed stride: a unit is computed the same way on whichever cluster takes it, so y is
    bit-identical, and both match the oracle."""
    wl = workload(name)
    ref = reference(name)
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    ys = {}
    for b in (1, 0):
        with option("decode_balance", b):
            ys[b] = dp.sgmv(dp.y(), seg)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1])
    assert_close(dp.to_np(ys[1]), ref, wl.dtype, name + " (balanced runs)")
    assert dp.status() == (0, 0)


def test_token_permutation_permutes_output_exactly():
    wl = _small("multirank_decode")
    dp = DeviceProj(wl)
    y = dp.bgmv(dp.y())
    perm = torch.from_numpy(np.random.default_rng(4).permutation(wl.T)).cuda()
    yp = dp.bgmv(dp.d.y0[perm].clone(), ids=dp.ids[perm].contiguous(), x=dp.d.x[perm].contiguous())
    assert torch.equal(yp, y[perm])


def test_mixed_ranks_equal_single_adapter_calls():
    wl = _small("multirank_decode")
    dp = DeviceProj(wl)
    y = dp.bgmv(dp.y())
    for a in np.unique(wl.ids)[:12]:
        ids_a = torch.from_numpy(np.where(wl.ids == a, wl.ids, -1).astype(np.int32)).cuda()
        ya = dp.bgmv(dp.y(), ids=ids_a)
        rows = torch.from_numpy(wl.ids == a).cuda()
        assert torch.equal(ya[rows], y[rows])
        assert torch.equal(ya[~rows], dp.d.y0[~rows])


def test_shrink_and_expand_entry_points():
    wl = _small("multirank_decode")
    dp = DeviceProj(wl)
    seg, _k = dp.segments()
    R = dp.table.max_rank
    v = torch.full((wl.T, R), float("nan"), dtype=torch.float32, device="cuda")
    L.lora_shrink(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], v, R)
    p = wl.projections[0]
    A = [p.A(i) for i in range(wl.n)]
    B = [p.B(i) for i in range(wl.n)]
    v_ref = oracle.lora_shrink(wl.dtype, p.x, wl.ids, A, ldv=R)
    v_gpu = v.cpu().numpy().astype(np.float64)
    for t in range(wl.T):
        r = p.ranks[wl.ids[t]]
        bound = 1e-2 * np.abs(v_ref[t, :r]).max() + 1e-3
        assert np.abs(v_gpu[t, :r] - v_ref[t, :r]).max() <= bound
    vin = workloads.random_intermediate(wl.T, R, seed=21)
    y = dp.y()
    L.lora_expand(dp.table.handle, seg, torch.from_numpy(vin).cuda(), R, y, y.shape[1], 0)
    ref = oracle.lora_expand(wl.dtype, vin, p.y0, wl.ids, B, p.scales)
    assert_close(dp.to_np(y), ref, wl.dtype, "expand alone")


def test_output_slice_of_a_wider_y():
    """Delta into columns [y_offset, y_offset + o) of a fused output; the rest untouched."""
    wl = _small("decode_bgmv")
    dp = DeviceProj(wl)
    o = wl.projections[0].o
    off = 2 * o
    wide = torch.randn(wl.T, 4 * o, device="cuda").to(torch.bfloat16)
    wide[:, off:off + o] = dp.d.y0
    before = wide.clone()
    L.lora_bgmv(dp.table.handle, dp.ids, wl.T, dp.d.x, dp.d.x.shape[1], wide, wide.shape[1], off)
    ref = oracle.workload_reference(wl)
    assert_close(dp.to_np(wide[:, off:off + o].contiguous()), ref, wl.dtype, "slice")
    assert torch.equal(wide[:, :off], before[:, :off])
    assert torch.equal(wide[:, off + o:], before[:, off + o:])


@pytest.mark.parametrize("h,o,ranks,T", [(8192, 1032, (12, 5, 128), 77), (1032, 14336, (64, 8), 40),
                                         (4096, 1024, (1, 3, 16), 33)])
def test_ragged_shapes_and_odd_ranks(h, o, ranks, T):
    """Several h tiles per CTA, o not a multiple of the tile, ranks that are not multiples of
    8, token counts that are not multiples of the unit size."""
    wl = workloads.generate("multirank_decode", T=T, n=9, shapes=(("q", h, o, 0),), ranks=ranks)
    dp = DeviceProj(wl)
    ref = oracle.workload_reference(wl)
    seg, _k = dp.segments()
    for cluster in (1, 2, 4, 8):
        with option("decode_cluster", cluster):
            y = dp.bgmv(dp.y())
            assert_close(dp.to_np(y), ref, wl.dtype, "ragged bgmv, cluster %d" % cluster)
            y2 = dp.sgmv(dp.y(), seg)
            assert torch.equal(y, y2)


@pytest.mark.parametrize("cluster", [1, 2, 4])
@pytest.mark.parametrize("name", ["decode_bgmv", "multirank_decode", "many_adapter_qkvo"])
def test_every_cluster_width_matches_oracle(name, cluster):
    """The decode kernel at each forced cluster width (8 is what the automatic choice takes
    for the small batches elsewhere in this file), fused and split, at full size."""
    wl = workload(name)
    ref = reference(name)
    dp = DeviceProj(wl)
    seg, _k = dp.segments()
    with option("decode_cluster", cluster):
        y = dp.bgmv(dp.y())
        assert_close(dp.to_np(y), ref, wl.dtype, "%s bgmv, cluster %d" % (name, cluster))
        y2 = dp.sgmv(dp.y(), seg)
        assert_close(dp.to_np(y2), ref, wl.dtype, "%s sgmv, cluster %d" % (name, cluster))
        with option("split", 1):
            y3 = dp.sgmv(dp.y(), seg)
        assert_close(dp.to_np(y3), ref, wl.dtype, "%s split, cluster %d" % (name, cluster))
    assert dp.status() == (0, 0)


def test_long_segment_spans_many_units():
    """One adapter carries 200 tokens: 13 units of at most 16 tokens on one cluster."""
    wl = workloads.generate("decode_bgmv", T=230, shapes=(("q", 2048, 2048, 0),))
    wl.ids[:200] = 3
    dp = DeviceProj(wl)
    ref = oracle.workload_reference(wl)
    y = dp.bgmv(dp.y())
    assert_close(dp.to_np(y), ref, wl.dtype, "long segment")


def test_large_batch_bgmv_goes_through_the_workspace():
    wl = workloads.generate("many_adapter_qkvo", T=2000, n=300, shapes=(("q", 1024, 512, 0),))
    dp = DeviceProj(wl)
    ref = oracle.workload_reference(wl)
    y = dp.bgmv(dp.y())
    assert_close(dp.to_np(y), ref, wl.dtype, "T=2000 bgmv")


# ------------------------------------------------------------------ no-adapter tokens and errors

def test_no_adapter_tokens_untouched_and_bad_ids_flagged():
    wl = _small("decode_bgmv")
    ids = wl.ids.copy()
    ids[::5] = -1
    ids[7] = wl.n + 3
    dp = DeviceProj(wl)
    d_ids = torch.from_numpy(ids).cuda()
    y = dp.bgmv(dp.y(), ids=d_ids)
    good = ids.copy()
    good[7] = -1
    p = wl.projections[0]
    ref = oracle.lora_delta(wl.dtype, p.x, p.y0, good, [p.A(i) for i in range(wl.n)],
                            [p.B(i) for i in range(wl.n)], p.scales)
    assert_close(dp.to_np(y), ref, wl.dtype, "with -1 ids")
    rows = torch.from_numpy(good < 0).cuda()
    assert torch.equal(y[rows], dp.d.y0[rows])
    rc, word = dp.status()
    assert rc == L.LORA_ERR_DEVICE_STATUS and word & L.LORA_STATUS_BAD_ID
    assert dp.status() == (0, 0)


def test_bad_segment_entries_are_skipped_and_flagged():
    wl = _small("decode_bgmv")
    dp = DeviceProj(wl)
    seg, t = dp.segments()
    torch.cuda.synchronize()
    S = int(t["num_segs"].item())
    t["seg_adapter"][0] = wl.n + 1         # segment 0 names a missing adapter
    y = dp.sgmv(dp.y(), seg)
    rc, word = dp.status()
    assert word & L.LORA_STATUS_BAD_SEGMENT
    p0, p1 = int(t["seg_ptr"][0]), int(t["seg_ptr"][1])
    skipped = t["perm"][p0:p1].long()
    assert torch.equal(y[skipped], dp.d.y0[skipped])
    assert S > 1


def test_host_side_errors():
    wl = _small("decode_bgmv")
    dp = DeviceProj(wl)
    h = dp.table.handle
    x, y = dp.d.x, dp.y()
    with pytest.raises(L.LoraError) as e:
        L.lora_bgmv(h, None, wl.T, x, x.shape[1], y, y.shape[1], 0)
    assert e.value.code == L.LORA_ERR_INVALID_ARG
    with pytest.raises(L.LoraError) as e:
        L.lora_bgmv(h, dp.ids, wl.T, x.data_ptr() + 2, x.shape[1], y, y.shape[1], 0)
    assert e.value.code == L.LORA_ERR_UNSUPPORTED
    with pytest.raises(L.LoraError) as e:
        L.lora_bgmv(h, dp.ids, wl.T, x, x.shape[1], y, y.shape[1], 4)   # slice runs past ldy
    assert e.value.code == L.LORA_ERR_INVALID_ARG
    seg, _k = dp.segments()
    L.lora_set_option("split", 1)
    try:
        with pytest.raises(L.LoraError) as e:
            L.lora_sgmv(h, seg, x, x.shape[1], y, y.shape[1], 0, None, 0)
        assert e.value.code == L.LORA_ERR_WORKSPACE
    finally:
        L.lora_set_option("split", 0)
    A0 = dp.d.A_ptrs[0]
    with pytest.raises(L.LoraError) as e:
        L.lora_table_create([A0], [dp.d.B_ptrs[0]], [L.LORA_MAX_RANK + 1], [1.0], 1024, 768, L.LORA_BF16)
    assert e.value.code == L.LORA_ERR_UNSUPPORTED
    with pytest.raises(L.LoraError) as e:
        L.lora_table_create([A0 + 8], [dp.d.B_ptrs[0]], [16], [1.0], 1024, 768, L.LORA_BF16)
    assert e.value.code == L.LORA_ERR_UNSUPPORTED
    with pytest.raises(L.LoraError) as e:
        L.lora_table_create([A0], [dp.d.B_ptrs[0]], [16], [1.0], 1020, 768, L.LORA_BF16)
    assert e.value.code == L.LORA_ERR_UNSUPPORTED
    assert dp.status() == (0, 0)


def test_pdl_on_and_off_agree():
    wl = _small("decode_bgmv")
    dp = DeviceProj(wl)
    L.lora_set_option("pdl", 0)
    try:
        y0 = dp.bgmv(dp.y())
    finally:
        L.lora_set_option("pdl", 1)
    y1 = dp.bgmv(dp.y())
    assert torch.equal(y0, y1)


# ------------------------------------------------------------------ tcgen05 prefill path

def _prefill_case(seg_lens, h, o, ranks, seed=5, delta_only=False):
    T, n = sum(seg_lens), len(seg_lens)
    wl = workloads.generate("prefill_sgmv", T=T, n=n, seg_len=max(seg_lens), shapes=(("up", h, o, 0),),
                            ranks=ranks, seed=seed, delta_only=delta_only)
    wl.ids = np.concatenate([np.full(l, i, np.int32) for i, l in enumerate(seg_lens)])
    dp = DeviceProj(wl)
    ptr = torch.from_numpy(np.concatenate([[0], np.cumsum(seg_lens)]).astype(np.int32)).cuda()
    ad = torch.arange(n, dtype=torch.int32, device="cuda")
    num = torch.tensor([n], dtype=torch.int32, device="cuda")
    seg = L.make_segments(None, ptr, ad, num, T, n, max(seg_lens))
    return wl, dp, seg, (ptr, ad, num)


@pytest.mark.parametrize("seg_lens,h,o,ranks", [
    ([300], 512, 256, (16,)),
    ([130, 100, 700, 1, 256], 1024, 384, (64, 8, 32, 16, 64)),
    ([257, 513, 129], 4096, 1024 + 64, (64, 32, 48)),
])
def test_prefill_tcgen05_ragged_segments_and_ranks(seg_lens, h, o, ranks):
    """Segments that are not multiples of the 128-token tile, o not a multiple of the
    128-column tile, ranks 8..64: the tensor-core path matches the oracle and the CUDA-core
    path within tolerance, and it is the path that ran."""
    wl, dp, seg, _keep = _prefill_case(seg_lens, h, o, ranks)
    ref = oracle.workload_reference(wl)
    names = kernels_launched(lambda: dp.sgmv(dp.y(), seg))
    assert any("prefill_expand_kernel" in k for k in names) and any("prefill_shrink_kernel" in k for k in names)
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), ref, wl.dtype, "tcgen05 prefill")
    L.lora_set_option("prefill_min_seg_len", 0)
    try:
        y2 = dp.sgmv(dp.y(), seg)
    finally:
        L.lora_set_option("prefill_min_seg_len", 256)
    assert_close(dp.to_np(y2), ref, wl.dtype, "decode path on prefill segments")
    assert dp.status() == (0, 0)


def test_prefill_tcgen05_output_slice_untouched_outside():
    wl, dp, seg, _keep = _prefill_case([257, 513], 4096, 1024, (64,))
    o = 1024
    wide = torch.randn(wl.T, o + 192, device="cuda").to(torch.bfloat16)
    wide[:, 128:128 + o] = dp.d.y0
    before = wide.clone()
    ws = dp.workspace()
    L.lora_sgmv(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], wide, wide.shape[1], 128, ws, ws.numel())
    ref = oracle.workload_reference(wl)
    assert_close(dp.to_np(wide[:, 128:128 + o].contiguous()), ref, wl.dtype, "slice")
    assert torch.equal(wide[:, :128], before[:, :128]) and torch.equal(wide[:, 128 + o:], before[:, 128 + o:])


def test_prefill_tcgen05_zero_B_leaves_y_bit_identical():
    wl, dp, seg, _keep = _prefill_case([300, 200], 1024, 512, (64,))
    dp.d.B_flat.zero_()
    y = dp.sgmv(dp.y(), seg)
    assert torch.equal(y, dp.d.y0)


def test_prefill_tcgen05_reuses_one_workspace():
    """Calls on one workspace back to back (the expand deals its last tiles from a counter in the
    workspace, which each call's shrink resets): every call matches the oracle and the first."""
    wl, dp, seg, _keep = _prefill_case([512, 384, 200], 4096, 2048, (64,))
    ref = oracle.workload_reference(wl)
    ws = dp.workspace()
    ys = []
    for _ in range(3):
        y = dp.y()
        L.lora_sgmv(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], y, y.shape[1], 0, ws, ws.numel())
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])
    assert_close(dp.to_np(ys[2]), ref, wl.dtype, "tcgen05 prefill, reused workspace")
    assert dp.status() == (0, 0)


def test_prefill_tcgen05_deterministic():
    wl, dp, seg, _keep = _prefill_case([512, 384], 4096, 2048, (64,))
    y1 = dp.sgmv(dp.y(), seg)
    y2 = dp.sgmv(dp.y(), seg)
    assert torch.equal(y1, y2)
