"""Mixed prefill batches on the tensor cores: tokens of several adapters interleaved in batch
order, grouped by lora_build_segments (so the segments carry a permutation), with segments of
very different lengths.  In a batch of at least "tc_min_tokens" tokens, lora_sgmv sends the
segments of at least "tc_min_seg_len" tokens to the tcgen05 kernels, which gather their token
rows through the permutation, and the shorter ones to the decode kernel.  Checked against the
fp64 oracle element by element, and with the launch counters that both kinds of kernel ran."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, option

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available()
    L._load()


def _mixed_ids(T, lens, seed):
    """Ids for segments of the given lengths (adapter i gets lens[i] tokens; -1 for the rest),
    shuffled into a random batch order."""
    ids = np.full(T, -1, np.int32)
    pos = 0
    for a, ln in enumerate(lens):
        ids[pos:pos + ln] = a
        pos += ln
    rng = np.random.default_rng(seed)
    rng.shuffle(ids)
    return ids


def _kernels_ran(fn):
    return kernels_launched(fn)


@pytest.mark.parametrize("delta_only", [False, True])
@pytest.mark.parametrize("lens,h,o,ranks", [
    ((700, 129, 64, 63, 5, 1, 300), 1024, 768, (64, 32, 16, 8)),   # long, ragged, at and below the split
    ((1024, 256), 512, 1024, (64,)),                                  # two long segments, whole tiles
])
def test_mixed_batch_long_segments_on_tcgen05(delta_only, lens, h, o, ranks):
    T = sum(lens) + 40   # 40 tokens without an adapter
    wl = workloads.generate("multirank_decode", T=T, n=len(lens), shapes=(("q", h, o, 0),), ranks=ranks,
                            seed=101, delta_only=delta_only)
    wl.ids = _mixed_ids(T, lens, seed=5)
    dp = DeviceProj(wl)
    seg, _keep = dp.segments()
    ref = oracle.workload_reference(wl)
    with option("tc_min_tokens", 1024), option("tc_min_seg_len", 64):
        y = dp.sgmv(dp.y(), seg)
        assert_close(dp.to_np(y), ref, wl.dtype, "mixed batch (tcgen05 + decode)")
        names = _kernels_ran(lambda: dp.sgmv(dp.y(), seg))
    assert any("prefill_shrink_kernel" in k for k in names), sorted(names)
    assert any("prefill_expand_kernel" in k for k in names), sorted(names)
    assert any("lora_decode_kernel" in k for k in names), sorted(names)
    # the same batch with every segment on the decode kernel agrees within the tolerance
    with option("tc_min_seg_len", 0):
        y2 = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y2), ref, wl.dtype, "mixed batch (decode only)")
    assert dp.status() == (0, 0)


def test_mixed_batch_through_bgmv_large_batch():
    """lora_bgmv on a batch above its direct limit sorts into the workspace and takes the same
    split: long groups on the tensor cores."""
    lens = (900, 300, 7)
    T = 1400
    wl = workloads.generate("multirank_decode", T=T, n=3, shapes=(("q", 512, 512, 0),), ranks=(16, 64), seed=3)
    wl.ids = _mixed_ids(T, lens, seed=9)
    dp = DeviceProj(wl)
    names = _kernels_ran(lambda: dp.bgmv(dp.y()))
    assert any("prefill_expand_kernel" in k for k in names)
    y = dp.bgmv(dp.y())
    assert_close(dp.to_np(y), oracle.workload_reference(wl), wl.dtype, "bgmv large mixed batch")
    assert dp.status() == (0, 0)
