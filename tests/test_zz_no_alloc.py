"""GPU test of lora_sgmv_noalloc, the SGMV entry point for callers that cannot allocate
device memory (their framework owns all of it, or an allocation would synchronise a
latency-critical path): it keeps the fp32 intermediate in a fixed array inside the library.

Its output must match the regular entry point lora_sgmv on the same inputs, and the fp64
oracle, within the tolerance the other parity tests use, on two calls in a row (the second
call sees the array as the first one left it).  This file is collected last on purpose."""
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close
from workloads import to_float64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("multirank_decode", dict(T=96, n=24, shapes=(("q", 2048, 1536, 0),))),
    ("decode_bgmv", {}),
])
def test_noalloc_matches_regular_sgmv_twice(name, kw):
    assert torch.cuda.is_available()
    wl = workloads.generate(name, **kw)
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    y_ref = dp.sgmv(dp.y(), seg)
    ref64 = to_float64(dp.to_np(y_ref), wl.dtype)
    exact = oracle.workload_reference(wl)
    for _ in range(2):
        y = dp.y()
        L.lora_sgmv_noalloc(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], y, y.shape[1], 0)
        assert_close(dp.to_np(y), ref64, wl.dtype, "noalloc vs lora_sgmv")
        assert_close(dp.to_np(y), exact, wl.dtype, "noalloc vs oracle")
    assert dp.status() == (0, 0)


def test_noalloc_rejects_batches_beyond_its_array():
    wl = workloads.generate("decode_bgmv", shapes=(("q", 64, 64, 0),))
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    ldv = (dp.table.max_rank + 3) // 4 * 4
    seg.T = L.LORA_NOALLOC_SCRATCH_FLOATS // ldv + 1
    y = dp.y()
    with pytest.raises(L.LoraError) as e:
        L.lora_sgmv_noalloc(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], y, y.shape[1], 0)
    assert e.value.code == L.LORA_ERR_WORKSPACE


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs a second GPU")
def test_noalloc_rejects_a_table_of_another_device():
    wl = workloads.generate("decode_bgmv", shapes=(("q", 64, 64, 0),))
    dp = DeviceProj(wl)   # table on device 0
    seg, _keep = dp.segments()
    y = dp.y()
    with torch.cuda.device(1):
        with pytest.raises(L.LoraError) as e:
            L.lora_sgmv_noalloc(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], y, y.shape[1], 0)
    assert e.value.code == L.LORA_ERR_INVALID_ARG
