"""GPU parity of the three-stage (compressed) form y += s_i B_i (Sigma_i (A_i x)) against the
oracle: full and diagonal Sigma, every entry point, adapters sharing cluster weights.
Tolerance as everywhere: |gpu - ref| <= 1e-2 * max|ref| + 1e-3 per element."""
import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, assert_close, kernels_launched, option, workload
from workloads.device import torch_to_np, upload_projection

pytestmark = pytest.mark.gpu

KIND = {"full": L.LORA_SIGMA_FULL, "diag": L.LORA_SIGMA_DIAG}
OKIND = {"full": oracle.SIGMA_FULL, "diag": oracle.SIGMA_DIAG}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L._load()
    yield
    L.lora_set_option("decode_cluster", 0)
    L.lora_set_option("split", 0)


def _with_sigma(dp, kind, seed):
    sig = workloads.draw_sigma(dp.p.ranks, kind, seed)
    dev = [torch.from_numpy(s).cuda() for s in sig]
    dp.table.set_sigma(KIND[kind], dev)
    dp._sigma_keep = dev
    return sig


def _ref(wl, p, sig, kind, ids=None):
    A = [p.A(i) for i in range(wl.n)]
    B = [p.B(i) for i in range(wl.n)]
    return oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids if ids is None else ids, A, B, p.scales,
                                   OKIND[kind], sig)


@pytest.mark.parametrize("kind", ["full", "diag"])
@pytest.mark.parametrize("delta_only", [False, True])
def test_sigma_multirank_every_entry_point(kind, delta_only):
    """Multi-rank decode workload (ranks 8..64, Zipf ids) with Sigma: BGMV, SGMV, shrink then
    expand through the workspace, and the grouped call, against the three-stage oracle."""
    wl = workload("multirank_decode", delta_only)
    dp = DeviceProj(wl)
    sig = _with_sigma(dp, kind, seed=31)
    ref = _ref(wl, dp.p, sig, kind)
    assert_close(dp.to_np(dp.bgmv(dp.y())), ref, wl.dtype, "sigma bgmv")
    seg, _k = dp.segments()
    assert_close(dp.to_np(dp.sgmv(dp.y(), seg)), ref, wl.dtype, "sigma sgmv")
    with option("split", 1):
        assert_close(dp.to_np(dp.sgmv(dp.y(), seg)), ref, wl.dtype, "sigma split")
    y = dp.y()
    ws = dp.workspace()
    L.lora_sgmv_grouped([dp.table.handle], seg, [dp.d.x], [dp.d.x.shape[1]], [y], [y.shape[1]], [0], ws, ws.numel())
    assert_close(dp.to_np(y), ref, wl.dtype, "sigma grouped")
    assert dp.status() == (0, 0)


@pytest.mark.parametrize("cluster", [1, 2, 8])
def test_sigma_every_cluster_width(cluster):
    wl = workloads.generate("multirank_decode", T=70, n=13, shapes=(("q", 2048, 1032, 0),), ranks=(5, 16, 64, 128))
    dp = DeviceProj(wl)
    sig = _with_sigma(dp, "full", seed=5)
    ref = _ref(wl, dp.p, sig, "full")
    seg, _k = dp.segments()
    with option("decode_cluster", cluster):
        y = dp.bgmv(dp.y())
        assert_close(dp.to_np(y), ref, wl.dtype, "sigma bgmv cluster %d" % cluster)
        assert torch.equal(y, dp.sgmv(dp.y(), seg))


def test_sigma_shrink_writes_sigma_times_intermediate():
    wl = workloads.generate("multirank_decode", T=50, n=9, shapes=(("q", 1024, 512, 0),))
    dp = DeviceProj(wl)
    sig = _with_sigma(dp, "full", seed=2)
    seg, _k = dp.segments()
    R = dp.table.max_rank
    v = torch.full((wl.T, R), float("nan"), dtype=torch.float32, device="cuda")
    L.lora_shrink(dp.table.handle, seg, dp.d.x, dp.d.x.shape[1], v, R)
    A = [dp.p.A(i) for i in range(wl.n)]
    want = oracle.lora_shrink_sigma(wl.dtype, dp.p.x, wl.ids, A, oracle.SIGMA_FULL, sig, ldv=R)
    got = v.cpu().numpy().astype(np.float64)
    for t in range(wl.T):
        r = dp.p.ranks[wl.ids[t]]
        bound = 1e-2 * np.abs(want[t, :r]).max() + 1e-3
        assert np.abs(got[t, :r] - want[t, :r]).max() <= bound


@pytest.mark.parametrize("kind", ["full", "diag"])
def test_identity_sigma_is_bit_identical_to_plain(kind):
    """Sigma = I (or ones) multiplies by exactly 1 and adds exact zeros in fp32 too."""
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    plain = dp.bgmv(dp.y())
    dev = [torch.eye(int(r), device="cuda") if kind == "full" else torch.ones(int(r), device="cuda")
           for r in dp.p.ranks]
    dp.table.set_sigma(KIND[kind], dev)
    three = dp.bgmv(dp.y())
    assert torch.equal(plain, three)
    dp.table.set_sigma(L.LORA_SIGMA_NONE)
    assert torch.equal(plain, dp.bgmv(dp.y()))


def test_shared_cluster_weights():
    """Compressed serving: adapters of a cluster point at the leader's A_c, B_c and differ
    only in Sigma_i; the Zipf-head many-adapter batch on the q projection."""
    name = "many_adapter_qkvo"
    wl = workload(name)
    p = wl.projections[0]
    cl = workloads.jd_clusters(wl.n, 16)
    d = upload_projection(p, wl.dtype)
    A_ptrs = [d.A_ptrs[c] for c in cl]
    B_ptrs = [d.B_ptrs[c] for c in cl]
    ranks = [int(p.ranks[c]) for c in cl]
    table = L.AdapterTable(A_ptrs, B_ptrs, ranks, p.scales, p.h, p.o, L.LORA_BF16, keep=d)
    sig = workloads.draw_sigma(np.asarray(ranks), "full", seed=7)
    dev = [torch.from_numpy(s).cuda() for s in sig]
    table.set_sigma(L.LORA_SIGMA_FULL, dev)
    ids = torch.from_numpy(wl.ids).cuda()
    y = d.y0.clone()
    ws = torch.empty(table.workspace_bytes(wl.T), dtype=torch.uint8, device="cuda")
    L.lora_bgmv(table.handle, ids, wl.T, d.x, p.h, y, p.o, 0, ws, ws.numel())
    A = [p.A(c) for c in cl]
    B = [p.B(c) for c in cl]
    ref = oracle.lora_delta_sigma(wl.dtype, p.x, p.y0, wl.ids, A, B, p.scales, oracle.SIGMA_FULL, sig)
    torch.cuda.synchronize()
    assert_close(torch_to_np(y, wl.dtype), ref, wl.dtype, "shared cluster weights")
    table.close()


def test_sigma_long_segments_take_the_decode_kernels():
    """A table with Sigma never takes the tcgen05 path: long contiguous segments still match."""
    wl = workloads.generate("prefill_sgmv", n=3, seg_len=300, shapes=(("up", 1024, 2048, 0),))
    dp = DeviceProj(wl)
    sig = _with_sigma(dp, "diag", seed=9)
    ref = _ref(wl, dp.p, sig, "diag")
    T, n = wl.T, wl.n
    seg_ptr = torch.arange(0, T + 1, 300, dtype=torch.int32, device="cuda")
    seg = L.make_segments(None, seg_ptr, torch.arange(n, dtype=torch.int32, device="cuda"),
                          torch.tensor([n], dtype=torch.int32, device="cuda"), T, n, 300)
    names = " ".join(kernels_launched(lambda: dp.sgmv(dp.y(), seg)))
    assert "prefill" not in names and "lora_decode_kernel" in names
    y = dp.sgmv(dp.y(), seg)
    assert_close(dp.to_np(y), ref, wl.dtype, "sigma long segments")


def test_set_sigma_rejects_bad_arguments():
    wl = workload("decode_bgmv")
    dp = DeviceProj(wl)
    with pytest.raises(L.LoraError) as e:
        dp.table.set_sigma(7, None)
    assert e.value.code == L.LORA_ERR_INVALID_ARG
    with pytest.raises(L.LoraError) as e:
        L.lora_table_set_sigma(dp.table.handle, L.LORA_SIGMA_FULL, [0] * wl.n)
    assert e.value.code == L.LORA_ERR_INVALID_ARG
