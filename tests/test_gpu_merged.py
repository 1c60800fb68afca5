"""GPU parity of several adapters merged per token (weighted ensembles) against the oracle.

Two modes.  With the plain workspace the GPU rounds y after each of the K slots and the oracle
once, so the tolerance is the usual |gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element.  With
room for the fp32 sum the slots' terms are summed in fp32 and y is rounded once: every output
then lies within one unit in the last place of the exact fp64 result, give or take the fp32
summation error where y0 and the delta cancel."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, ran, workload
from workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L._load()
    yield


def _merged(dp, ids2, w2, y, ws=None, y_off=0):
    T, K = ids2.shape
    ws = dp.workspace() if ws is None else ws
    L.lora_bgmv_merged(dp.table.handle, torch.from_numpy(ids2).cuda(), torch.from_numpy(w2).cuda(), T, K,
                       dp.d.x, dp.d.x.shape[1], y, y.shape[1], y_off, ws, ws.numel())
    return y


def _sum_workspace(dp, T):
    """The workspace size that holds the fp32 [T, o] sum after the library's own areas."""
    w = (dp.table.workspace_bytes(T) + 255) // 256 * 256
    return torch.empty(w + T * dp.p.o * 4, dtype=torch.uint8, device="cuda")


def _within_one_rounding(got_bits, ref, y0_bits):
    """|got - ref| <= one bf16 ulp of ref plus 2^-16 of the largest |delta|: one rounding of the
    result, with room for the fp32 summation error of the delta, which only shows where y0 and
    the delta cancel to a small result.  Returns the worst ratio of error to bound."""
    got = workloads.to_float64(got_bits, "bf16")
    _, e = np.frexp(np.abs(ref))
    ulp = np.ldexp(1.0, e - 8)
    slack = 2.0 ** -16 * np.abs(ref - workloads.to_float64(y0_bits, "bf16")).max()
    return float((np.abs(got - ref) / (ulp + slack)).max())


def _ulps_bf16(got_bits, ref):
    """Distance in bf16 units in the last place between stored results and the exact values
    rounded to bf16 (through fp32: exact for these magnitudes but for double-rounding ties)."""
    def ordered(b):
        b = np.asarray(b, dtype=np.uint16).astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(got_bits) - ordered(f32_to_bf16_bits(ref.astype(np.float32))))


def _ref(wl, dp, ids2, w2):
    p = dp.p
    return oracle.lora_delta_merged(wl.dtype, p.x, p.y0, ids2, w2, [p.A(i) for i in range(wl.n)],
                                    [p.B(i) for i in range(wl.n)], p.scales)


@pytest.mark.parametrize("K", [2, 3])
@pytest.mark.parametrize("delta_only", [False, True])
def test_merged_decode_batch(K, delta_only):
    """The decode workload (64 tokens, 32 rank-16 adapters, 4096 -> 4096) with K-adapter
    ensembles per token, a quarter of the extra slots empty."""
    wl = workload("decode_bgmv", delta_only)
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, K, seed=40 + K, empty=0.25)
    y = _merged(dp, ids2, w2, dp.y())
    assert_close(dp.to_np(y), _ref(wl, dp, ids2, w2), wl.dtype, "merged K=%d" % K)
    assert dp.status() == (0, 0)


def test_merged_multirank_and_large_batch_path():
    """Mixed ranks, and a 1500-token batch that sorts each slot into the workspace."""
    for T in (200, 1500):
        wl = workloads.generate("multirank_decode", T=T, n=40, shapes=(("q", 1024, 1032, 0),))
        dp = DeviceProj(wl)
        ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 2, seed=T, empty=0.3)
        y = _merged(dp, ids2, w2, dp.y())
        assert_close(dp.to_np(y), _ref(wl, dp, ids2, w2), wl.dtype, "merged T=%d" % T)


def test_single_slot_unit_weight_is_bgmv_bit_for_bit():
    wl = workload("multirank_decode")
    dp = DeviceProj(wl)
    ids2 = wl.ids.reshape(-1, 1).astype(np.int32)
    y = _merged(dp, ids2, np.ones_like(ids2, dtype=np.float32), dp.y())
    assert torch.equal(y, dp.bgmv(dp.y()))


def test_zero_weights_leave_y_bit_identical():
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 3, seed=2)
    y = _merged(dp, ids2, np.zeros_like(w2), dp.y())
    assert torch.equal(y, dp.d.y0)


def test_merged_rejects_bad_slot_counts():
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 2, seed=3)
    di, dw = torch.from_numpy(ids2).cuda(), torch.from_numpy(w2).cuda()
    for K in (0, L.LORA_MAX_MERGE + 1):
        with pytest.raises(L.LoraError) as e:
            L.lora_bgmv_merged(dp.table.handle, di, dw, wl.T, K, dp.d.x, dp.d.x.shape[1], dp.y(), wl.projections[0].o,
                               0)
        assert e.value.code == L.LORA_ERR_INVALID_ARG


@pytest.mark.parametrize("K", [2, 3])
def test_merged_fp32_sum_rounds_once(K):
    """With the larger workspace the K slots are summed in fp32 and y is rounded once by
    merge_finish_kernel: every element within one rounding of the exact result, at least 95% of
    them equal to it rounded, and the total error below that of the K-rounding mode on the same
    inputs."""
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, K, seed=60 + K, empty=0.25)
    ref = _ref(wl, dp, ids2, w2)
    ws = _sum_workspace(dp, wl.T)
    y1 = dp.y()
    names = kernels_launched(lambda: _merged(dp, ids2, w2, y1, ws))
    assert ran(names, "merge_finish_kernel")
    got = dp.to_np(y1)
    worst = _within_one_rounding(got, ref, wl.projections[0].y0)
    assert worst <= 1.0, worst
    d = _ulps_bf16(got, ref)
    assert (d == 0).mean() >= 0.95, "only %.3f of the outputs rounded exactly" % (d == 0).mean()
    yk = _merged(dp, ids2, w2, dp.y())   # plain workspace: rounded after each slot
    got_k = dp.to_np(yk)
    err1 = np.abs(workloads.to_float64(got, wl.dtype) - ref).sum()
    errk = np.abs(workloads.to_float64(got_k, wl.dtype) - ref).sum()
    assert err1 < errk, (err1, errk)
    assert dp.status() == (0, 0)


def test_merged_fp32_sum_sorted_batch_and_offset():
    """The fp32-sum mode on a 1500-token batch (each slot sorted into the workspace ahead of the
    sum) writing a column window of a wider y (offset 8, row stride o + 24)."""
    T = 1500
    wl = workloads.generate("multirank_decode", T=T, n=40, shapes=(("q", 1024, 1032, 0),))
    dp = DeviceProj(wl)
    o = dp.p.o
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 3, seed=71, empty=0.3)
    ref = _ref(wl, dp, ids2, w2)
    wide = torch.randn(T, o + 24, device="cuda").to(torch.bfloat16)
    before = wide.clone()
    wide[:, 8:8 + o] = dp.y()
    ws = _sum_workspace(dp, T)
    names = kernels_launched(lambda: _merged(dp, ids2, w2, wide, ws, y_off=8))
    assert ran(names, "merge_finish_kernel")
    torch.cuda.synchronize()
    assert torch.equal(wide[:, :8], before[:, :8]) and torch.equal(wide[:, 8 + o:], before[:, 8 + o:])
    got = wide[:, 8:8 + o].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    worst = _within_one_rounding(got, ref, wl.projections[0].y0)
    assert worst <= 1.0, worst
    assert (_ulps_bf16(got, ref) == 0).mean() >= 0.95
    assert dp.status() == (0, 0)


def test_merged_small_workspace_keeps_per_slot_rounding():
    """One byte short of the sum's room: the call takes the K-rounding passes (no final
    rounding launch) and matches the call with the plain workspace bit for bit."""
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 2, seed=81, empty=0.25)
    ws = _sum_workspace(dp, wl.T)
    short = ws[:ws.numel() - 1]
    y = dp.y()
    names = kernels_launched(lambda: _merged(dp, ids2, w2, y, short))
    assert not ran(names, "merge_finish_kernel")
    assert torch.equal(y, _merged(dp, ids2, w2, dp.y()))


def test_merged_fp32_sum_f32_outputs():
    """The fp32-sum mode with fp32 y (the 16-token, 4-adapter fp32 workload, K = 3)."""
    wl = workload("tiny_sgmv")
    dp = DeviceProj(wl)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 3, seed=91, empty=0.2)
    y = dp.y()
    names = kernels_launched(lambda: _merged(dp, ids2, w2, y, _sum_workspace(dp, wl.T)))
    assert ran(names, "merge_finish_kernel")
    assert_close(dp.to_np(y), _ref(wl, dp, ids2, w2), wl.dtype, "merged fp32 sum, f32")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("fp32_sum", [False, True])
def test_merged_with_sigma_tables(fp32_sum):
    """Merged ensembles over a table in the three-stage form (full Sigma_i), K = 2, in both
    rounding modes, against the oracle: the three-stage oracle's delta of each slot (y0 = 0),
    weighted per token and added to y0 in fp64 (the update is linear in each slot's term)."""
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    p = dp.p
    sig = workloads.draw_sigma(p.ranks, "full", 53)
    dev = [torch.from_numpy(s).cuda() for s in sig]
    dp.table.set_sigma(L.LORA_SIGMA_FULL, dev)
    ids2, w2 = workloads.draw_merge(wl.ids, wl.n, 2, seed=55, empty=0.25)
    A = [p.A(i) for i in range(wl.n)]
    B = [p.B(i) for i in range(wl.n)]
    zeros = np.zeros_like(p.y0)
    ref = workloads.to_float64(p.y0, wl.dtype).copy()
    for j in range(2):
        dj = oracle.lora_delta_sigma(wl.dtype, p.x, zeros, ids2[:, j].copy(), A, B, p.scales, oracle.SIGMA_FULL, sig)
        ref += w2[:, j:j + 1].astype(np.float64) * dj
    ws = _sum_workspace(dp, wl.T) if fp32_sum else None
    y = dp.y()
    names = kernels_launched(lambda: _merged(dp, ids2, w2, y, ws))
    assert ran(names, "merge_finish_kernel") == fp32_sum
    assert_close(dp.to_np(y), ref, wl.dtype, "merged sigma, fp32 sum %s" % fp32_sum)
    assert dp.status() == (0, 0)
