"""GPU parity of the grouped multi-projection call (q, k, v, o of one layer in one launch over
one segment table) against the oracle, and against separate lora_sgmv calls bit for bit.
Tolerance as everywhere: |gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, option, reference, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L._load()
    yield
    L.lora_set_option("decode_cluster", 0)
    L.lora_set_option("split", 0)


def _grouped(dps, seg, xs, ys, offs):
    ws = dps[0].workspace()
    L.lora_sgmv_grouped([d.table.handle for d in dps], seg, xs, [x.shape[1] for x in xs], ys,
                        [y.shape[1] for y in ys], offs, ws, ws.numel())


@pytest.mark.parametrize("delta_only", [False, True])
def test_grouped_qkvo_matches_oracle_and_separate_calls(delta_only):
    """The many-adapter workload's four projections in one launch, q/k/v sharing one x."""
    name = "many_adapter_qkvo"
    wl = workload(name, delta_only)
    dps = [DeviceProj(wl, pi) for pi in range(4)]
    seg, _k = dps[0].segments()
    x_shared = dps[0].d.x
    xs = [x_shared, x_shared, x_shared, dps[3].d.x]
    with option("decode_cluster", 8):
        ys = [d.y() for d in dps]
        _grouped(dps, seg, xs, ys, [0, 0, 0, 0])
        for pi, d in enumerate(dps):
            assert_close(d.to_np(ys[pi]), reference(name, delta_only, proj=pi), wl.dtype, "grouped proj %d" % pi)
            y_sep = d.sgmv(d.y(), seg, x=xs[pi])
            assert torch.equal(ys[pi], y_sep), "projection %d differs from its separate call" % pi
    assert dps[0].status() == (0, 0)


def test_grouped_writes_slices_of_a_fused_qkv_output():
    """q, k and v into column slices [0, 4096), [4096, 5120), [5120, 6144) of one output, o into
    its own; the automatic cluster width; columns outside the slices untouched."""
    name = "many_adapter_qkvo"
    wl = workload(name)
    dps = [DeviceProj(wl, pi) for pi in range(4)]
    seg, _k = dps[0].segments()
    T = wl.T
    qkv = torch.randn(T, 6144 + 64, device="cuda").to(torch.bfloat16)
    offs = [0, 4096, 5120]
    for pi in range(3):
        qkv[:, offs[pi]:offs[pi] + dps[pi].p.o] = dps[pi].d.y0
    before = qkv.clone()
    y_o = dps[3].y()
    x = dps[0].d.x
    ws = dps[0].workspace()
    L.lora_sgmv_grouped([d.table.handle for d in dps], seg, [x, x, x, dps[3].d.x], [x.shape[1]] * 4,
                        [qkv, qkv, qkv, y_o], [qkv.shape[1]] * 3 + [y_o.shape[1]], offs + [0], ws, ws.numel())
    for pi in range(3):
        o = dps[pi].p.o
        got = qkv[:, offs[pi]:offs[pi] + o].contiguous()
        assert_close(dps[pi].to_np(got), reference(name, proj=pi), wl.dtype, "fused slice %d" % pi)
    assert_close(dps[3].to_np(y_o), reference(name, proj=3), wl.dtype, "o projection")
    assert torch.equal(qkv[:, 6144:], before[:, 6144:])


def test_grouped_mixed_shapes_and_ranks():
    """Two projections of different h and o (ragged against the tiles), mixed ranks, ragged
    token count, each with its own x."""
    wl = workloads.generate("multirank_decode", T=77, n=11, shapes=(("a", 2048, 1032, 0), ("b", 1032, 3072, 1)),
                            ranks=(8, 16, 32, 64))
    dps = [DeviceProj(wl, pi) for pi in range(2)]
    seg, _k = dps[0].segments()
    for cluster in (8, 2):
        with option("decode_cluster", cluster):
            ys = [d.y() for d in dps]
            _grouped(dps, seg, [d.d.x for d in dps], ys, [0, 0])
            for pi, d in enumerate(dps):
                assert_close(d.to_np(ys[pi]), oracle.workload_reference(wl, pi), wl.dtype, "mixed proj %d" % pi)
                assert torch.equal(ys[pi], d.sgmv(d.y(), seg))


def test_grouped_single_projection_is_lora_sgmv():
    wl = workload("multirank_decode")
    dp = DeviceProj(wl)
    seg, _k = dp.segments()
    y1 = dp.y()
    _grouped([dp], seg, [dp.d.x], [y1], [0])
    assert torch.equal(y1, dp.sgmv(dp.y(), seg))


def test_grouped_rejects_overlapping_slices_and_mismatched_tables():
    wl = workload("many_adapter_qkvo")
    dps = [DeviceProj(wl, pi) for pi in range(3)]
    seg, _k = dps[0].segments()
    x = dps[0].d.x
    y = torch.zeros(wl.T, 6144, device="cuda", dtype=torch.bfloat16)
    ws = dps[0].workspace()
    tabs = [d.table.handle for d in dps]
    with pytest.raises(L.LoraError) as e:   # k's slice [4000, 5024) overlaps q's [0, 4096)
        L.lora_sgmv_grouped(tabs, seg, [x] * 3, [x.shape[1]] * 3, [y] * 3, [6144] * 3, [0, 4000, 5120],
                            ws, ws.numel())
    assert e.value.code == L.LORA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(y)) == 0
    other = workloads.generate("multirank_decode", T=wl.T, n=17, shapes=(("q", 4096, 1024, 0),))
    dpo = DeviceProj(other)
    with pytest.raises(L.LoraError) as e:   # a table with another adapter count
        L.lora_sgmv_grouped([tabs[0], dpo.table.handle], seg, [x, x], [x.shape[1]] * 2,
                            [y, dpo.y()], [6144, 1024], [0, 0], ws, ws.numel())
    assert e.value.code == L.LORA_ERR_INVALID_ARG


def test_grouped_split_option_runs_separate_calls():
    """With the split option the grouped call falls back to one lora_sgmv per table (shrink
    then expand through the workspace); results stay within tolerance of the oracle."""
    name = "many_adapter_qkvo"
    wl = workload(name)
    dps = [DeviceProj(wl, pi) for pi in range(2)]
    seg, _k = dps[0].segments()
    with option("split", 1):
        ys = [d.y() for d in dps]
        _grouped(dps, seg, [d.d.x for d in dps], ys, [0, 0])
    for pi, d in enumerate(dps):
        assert_close(d.to_np(ys[pi]), reference(name, proj=pi), wl.dtype, "split proj %d" % pi)


@pytest.mark.parametrize("cluster", [8, 4, 1])
def test_shared_exchange_is_bit_identical(cluster):
    """One cluster exchange per unit for all projections (the default) against one per
    projection: the same sums in the same order, so bit-identical outputs, here with three
    projections (a token row of 3 x 16 partial slots) and with four of different ranks."""
    wl = workload("many_adapter_qkvo")
    dps = [DeviceProj(wl, pi) for pi in range(3)]
    seg, _k = dps[0].segments()
    x = dps[0].d.x
    mixed = workloads.generate("multirank_decode", T=150, n=23, ranks=(8, 16, 32, 64),
                               shapes=(("a", 1024, 1032, 0), ("b", 1032, 2048, 1), ("c", 1024, 512, 0),
                                       ("d", 2048, 1024, 2)))
    dpm = [DeviceProj(mixed, pi) for pi in range(4)]
    segm, _km = dpm[0].segments()
    with option("decode_cluster", cluster):
        outs = {}
        for shared in (1, 0):
            with option("decode_shared_exchange", shared):
                ys = [d.y() for d in dps]
                _grouped(dps, seg, [x, x, x], ys, [0, 0, 0])
                ym = [d.y() for d in dpm]
                _grouped(dpm, segm, [d.d.x for d in dpm], ym, [0, 0, 0, 0])
                torch.cuda.synchronize()
                outs[shared] = ys + ym
        for a, b in zip(outs[1], outs[0]):
            assert torch.equal(a, b)
        for pi, d in enumerate(dpm):
            assert_close(d.to_np(outs[1][3 + pi]), oracle.workload_reference(mixed, pi), mixed.dtype,
                         "shared exchange, mixed proj %d" % pi)
    assert dps[0].status() == (0, 0) and dpm[0].status() == (0, 0)
