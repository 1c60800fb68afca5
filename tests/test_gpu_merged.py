"""GPU parity of several adapters merged per token (weighted ensembles) against the oracle.
Tolerance as everywhere: |gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element (the GPU rounds
y after each of the K slots, the oracle once)."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L._load()
    yield


def _merged(dp, ids2, w2, y):
    T, K = ids2.shape
    ws = dp.workspace()
    L.lora_bgmv_merged(dp.table.handle, torch.from_numpy(ids2).cuda(), torch.from_numpy(w2).cuda(), T, K,
                       dp.d.x, dp.d.x.shape[1], y, y.shape[1], 0, ws, ws.numel())
    return y


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
