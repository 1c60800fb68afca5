"""GPU parity of lora_sgmv_base, the layer output with a frozen base weight fused with the
adapter term (tcgen05 shrink, then one tensor-core kernel accumulating x W^T and the
intermediate times B_i in the same tile), against the fp64 oracle's lora_base_delta.

Tolerance as everywhere: |gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element.  The base term
dominates the output, so the adapter term is also checked on its own (W = 0), where the
bound is relative to the delta alone."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, ran
from workloads.device import np_to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available()
    L._load()


def _contiguous(seg_ptr_host, seg_ad_host, T, n):
    seg_ptr = torch.tensor(seg_ptr_host, dtype=torch.int32, device="cuda")
    seg_ad = torch.tensor(seg_ad_host, dtype=torch.int32, device="cuda")
    num = torch.tensor([len(seg_ad_host)], dtype=torch.int32, device="cuda")
    seg = L.make_segments(None, seg_ptr, seg_ad, num, T, max(n, len(seg_ad_host)))
    return seg, (seg_ptr, seg_ad, num)


def _ids_of(seg_ptr, seg_ad, T):
    ids = np.full(T, -1, np.int32)
    for s, a in enumerate(seg_ad):
        ids[seg_ptr[s]:seg_ptr[s + 1]] = a
    return ids


def _case(h, o, seg_lens, head, tail, ranks, seed):
    T = head + sum(seg_lens) + tail
    n = len(ranks)
    wl = workloads.generate("multirank_decode", T=T, n=n, shapes=(("q", h, o, 0),), ranks=tuple(ranks), seed=seed)
    # one adapter per segment, ranks as given (the generator draws ranks per adapter)
    seg_ptr = [head]
    for ln in seg_lens:
        seg_ptr.append(seg_ptr[-1] + ln)
    seg_ad = [i % n for i in range(len(seg_lens))]
    return wl, seg_ptr, seg_ad


def _run(dp, seg, W, accumulate, y=None):
    y = dp.y() if y is None else y
    ws = dp.workspace()
    L.lora_sgmv_base(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], W, W.shape[1], y, y.shape[1], 0,
                     accumulate, ws, ws.numel())
    return y


@pytest.mark.parametrize("accumulate", [False, True])
@pytest.mark.parametrize("h,o,seg_lens,head,tail", [
    (1024, 640, (200, 256, 77), 40, 30),      # gaps before and after, ragged segments and N tile
    (512, 512, (128, 384), 0, 0),             # whole tiles only
    (768, 264, (1, 129, 130), 5, 0),          # one-token segment, o just past a 256 tile
])
def test_base_layer_output_matches_oracle(accumulate, h, o, seg_lens, head, tail):
    wl, seg_ptr, seg_ad = _case(h, o, seg_lens, head, tail, (64, 32, 16), seed=71)
    wl.ids = _ids_of(seg_ptr, seg_ad, wl.T)
    dp = DeviceProj(wl)
    seg, _keep = _contiguous(seg_ptr, seg_ad, wl.T, wl.n)
    W_np = workloads.draw_base_weight(o, h, seed=72)
    W = np_to_torch(W_np, "bf16").cuda()
    y = _run(dp, seg, W, accumulate)
    ref = oracle.base_reference(wl, W_np, accumulate=accumulate)
    assert_close(dp.to_np(y), ref, wl.dtype, "base layer output")
    # the adapter term alone (W = 0, no y0): the sensitive check of the delta part
    Z = torch.zeros_like(W)
    y_d = _run(dp, seg, Z, False)
    ref_d = oracle.base_reference(wl, np.zeros_like(W_np), accumulate=False)
    assert np.abs(ref_d).max() > 0
    assert_close(dp.to_np(y_d), ref_d, wl.dtype, "adapter term of the fused kernel")
    assert dp.status() == (0, 0)


def test_base_accumulate_into_zero_is_bit_identical_and_kernels_run():
    wl, seg_ptr, seg_ad = _case(512, 512, (300, 212), 16, 0, (64, 8), seed=5)
    wl.ids = _ids_of(seg_ptr, seg_ad, wl.T)
    dp = DeviceProj(wl)
    seg, _keep = _contiguous(seg_ptr, seg_ad, wl.T, wl.n)
    W = np_to_torch(workloads.draw_base_weight(512, 512, seed=6), "bf16").cuda()
    names = kernels_launched(lambda: _run(dp, seg, W, False))
    assert ran(names, "base_gemm_kernel") and ran(names, "prefill_shrink_kernel")
    a = _run(dp, seg, W, False)
    b = _run(dp, seg, W, True, y=torch.zeros_like(dp.d.y0))
    assert torch.equal(a, b)
    # run to run bit-identical
    c = _run(dp, seg, W, False)
    assert torch.equal(a, c)


def test_base_rejects_what_it_cannot_run():
    wl, seg_ptr, seg_ad = _case(256, 256, (64,), 0, 0, (16,), seed=9)
    dp = DeviceProj(wl)
    seg, _keep = _contiguous(seg_ptr, seg_ad, wl.T, wl.n)
    W = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    y = dp.y()
    ws = dp.workspace()
    perm = torch.arange(wl.T, dtype=torch.int32, device="cuda")
    seg_p = L.make_segments(perm, *(_keep[:3]), wl.T, wl.n)
    with pytest.raises(L.LoraError) as e:
        L.lora_sgmv_base(dp.table.handle, seg_p, dp.d.x, 256, W, 256, y, 256, 0, False, ws, ws.numel())
    assert e.value.code == L.LORA_ERR_UNSUPPORTED
    with pytest.raises(L.LoraError) as e:
        L.lora_sgmv_base(dp.table.handle, seg, dp.d.x, 256, W, 256, y, 256, 0, False, ws, 16)
    assert e.value.code == L.LORA_ERR_WORKSPACE
    with pytest.raises(L.LoraError) as e:
        L.lora_sgmv_base(dp.table.handle, seg, dp.d.x, 256, W, 128, y, 256, 0, False, ws, ws.numel())
    assert e.value.code == L.LORA_ERR_INVALID_ARG


@pytest.mark.slow
def test_base_full_prefill_shape_sampled_rows():
    """The prefill workload's shape (4096 -> 14336, 8 segments of 512 tokens, rank 64) with a
    synthetic base weight, in the launch configuration the benchmark times; the oracle checks
    two tokens of every segment (all 14336 outputs of each)."""
    wl = workloads.generate("prefill_sgmv")
    p = wl.projections[0]
    dp = DeviceProj(wl)
    seg, _keep = _contiguous(list(range(0, wl.T + 1, 512)), list(range(wl.n)), wl.T, wl.n)
    W_np = workloads.draw_base_weight(p.o, p.h, seed=wl.seed + 500)
    W = np_to_torch(W_np, "bf16").cuda()
    y = _run(dp, seg, W, False)
    got = dp.to_np(y)
    rows = np.array([s * 512 + k for s in range(wl.n) for k in (0, 511)])
    sub = bench_sample(wl, rows)
    ref = oracle.base_reference(sub, W_np, accumulate=False)
    assert_close(got[rows], ref, wl.dtype, "full-size fused layer output (sampled rows)")
    assert dp.status() == (0, 0)


def bench_sample(wl, rows):
    import copy
    sub = copy.copy(wl)
    sub.ids = wl.ids[rows].copy()
    sub.T = len(rows)
    sub.projections = []
    for q in wl.projections:
        qq = copy.copy(q)
        qq.x = q.x[rows]
        qq.y0 = q.y0[rows]
        sub.projections.append(qq)
    return sub
