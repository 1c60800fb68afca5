"""The bounded-wait path on the GPU, in the form that cannot fault or hang the device.

A host-set test option ("inject_stall") makes each kernel arm one pipeline stage per unit
(decode) or per tile (tcgen05 shrink and expand) without ever starting its copies: the
phase of that stage can never complete, like a flag that nothing sets.  With the wait bound
shortened to 20 ms ("wait_limit_ns"), the waits on it run out; the kernel latches
LORA_STATUS_TIMEOUT, waits (bounded) for every copy it did start, releases its tensor memory
and returns.  The test checks the status word, then that a default call on the same table,
same context, runs and matches the oracle, which it could not do if the previous launch had
left copies writing or tensor memory allocated."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, option, ran

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available()
    L._load()
    yield
    L.lora_set_option("inject_stall", 0)
    L.lora_set_option("wait_limit_ns", 0)


def _prefill(dp, wl, seg_len):
    seg_ptr = torch.arange(0, wl.T + 1, seg_len, dtype=torch.int32, device="cuda")
    seg_ad = torch.arange(wl.n, dtype=torch.int32, device="cuda")
    num = torch.tensor([wl.n], dtype=torch.int32, device="cuda")
    return L.make_segments(None, seg_ptr, seg_ad, num, wl.T, wl.n, seg_len), (seg_ptr, seg_ad, num)


@pytest.mark.parametrize("form", ["bgmv", "sgmv", "shrink", "expand"])
def test_decode_wait_runs_out_then_recovers(form):
    wl = workloads.generate("multirank_decode", T=40, n=12, shapes=(("q", 1024, 512, 0),))
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    assert dp.status() == (0, 0)
    with option("wait_limit_ns", LIMIT_NS), option("inject_stall", 1):
        y = dp.y()
        if form == "bgmv":
            dp.bgmv(y)
        elif form == "sgmv":
            dp.sgmv(y, seg)
        else:
            v = torch.zeros(wl.T, 64, dtype=torch.float32, device="cuda")
            if form == "shrink":
                L.lora_shrink(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], v, 64)
            else:
                L.lora_expand(dp.table.handle, seg, v, 64, y, y.shape[1], 0)
        torch.cuda.synchronize()
    rc, word = dp.status()
    assert rc == L.LORA_ERR_TIMEOUT and word & L.LORA_STATUS_TIMEOUT, (rc, word)
    # same context, default bound: the kernels run and match the oracle
    y = dp.bgmv(dp.y())
    assert_close(dp.to_np(y), oracle.workload_reference(wl), wl.dtype, "after timeout (bgmv)")
    y2 = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y2), oracle.workload_reference(wl), wl.dtype, "after timeout (sgmv)")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("bit", [2, 4])
def test_tcgen05_wait_runs_out_then_recovers(bit):
    """bit 2: the shrink's first k-block never lands; bit 4: the expand's first tile never
    lands.  Afterwards the tcgen05 kernels must allocate tensor memory again and match."""
    wl = workloads.generate("prefill_sgmv", n=3, seg_len=256, shapes=(("up", 1024, 512, 0),))
    dp = DeviceProj(wl)
    seg, _keep = _prefill(dp, wl, 256)
    with option("wait_limit_ns", LIMIT_NS), option("inject_stall", bit):
        dp.sgmv(dp.y(), seg)
        torch.cuda.synchronize()
    rc, word = dp.status()
    assert rc == L.LORA_ERR_TIMEOUT and word & L.LORA_STATUS_TIMEOUT, (rc, word)
    names = kernels_launched(lambda: dp.sgmv(dp.y(), seg))
    assert ran(names, "prefill_shrink_kernel") and ran(names, "prefill_expand_kernel")
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), oracle.workload_reference(wl), wl.dtype, "after timeout (tcgen05)")
    assert dp.status() == (0, 0)
