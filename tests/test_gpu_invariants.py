"""Exact GPU invariants of the LoRA delta, on top of the tolerance-based parity:

* integer-valued tiny inputs (h, o <= 32, T = 6, every id assignment over {-1, 0, 1}): every
  product and partial sum is an integer well inside fp32, so each GPU path must return the
  oracle's exact value rounded once to the output type -- bit for bit;
* doubling every scale doubles the delta-only output exactly (a power-of-two factor commutes
  with every rounding);
* listing the segments in another order (with their token lists moved along) changes no bit.
"""
import itertools

import numpy as np
import pytest
import torch

import heterogeneous_adapters_sgmv_b200 as L
import oracle
import workloads
from tests.gpu_util import DeviceProj, kernels_launched, option, ran
from workloads import f32_to_bf16_bits
from workloads.device import np_to_torch, torch_to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available()
    L._load()


def _store(a, dtype):
    a = np.asarray(a, dtype=np.float32)
    return f32_to_bf16_bits(a) if dtype == "bf16" else a


def _rounded(ref, dtype):
    """The exact fp64 result rounded once to the output type (as stored bits)."""
    return _store(ref.astype(np.float32), dtype)   # integers < 2^24: fp64 -> fp32 is exact


def _int_problem(dtype, h, o, ranks, seed):
    rng = np.random.default_rng(seed)
    A = [rng.integers(-1, 2, size=(r, h)) for r in ranks]
    B = [rng.integers(-1, 2, size=(o, r)) for r in ranks]
    return rng, [_store(a, dtype) for a in A], [_store(b, dtype) for b in B]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_integer_inputs_every_id_assignment_exact(dtype):
    h, o, T, ranks, scales = 32, 32, 6, (8, 16), (2.0, 0.5)
    rng, A, B = _int_problem(dtype, h, o, ranks, seed=3)
    x = _store(rng.integers(-1, 2, size=(T, h)), dtype)
    y0 = _store(rng.integers(-8, 9, size=(T, o)), dtype)
    dt = L.LORA_BF16 if dtype == "bf16" else L.LORA_F32
    dA = [np_to_torch(a, dtype).cuda() for a in A]
    dB = [np_to_torch(b, dtype).cuda() for b in B]
    table = L.AdapterTable(dA, dB, list(ranks), list(scales), h, o, dt)
    dx = np_to_torch(x, dtype).cuda()
    assigns = np.array(list(itertools.product((-1, 0, 1), repeat=T)), dtype=np.int32)   # 729 x 6
    N = len(assigns)
    ids = torch.from_numpy(assigns).cuda()
    es = 2 if dtype == "bf16" else 4
    y_b = np_to_torch(np.broadcast_to(y0, (N, T, o)).copy(), dtype).cuda()
    y_s = y_b.clone()
    y_x = y_b.clone()
    perm = torch.empty(N, T, dtype=torch.int32, device="cuda")
    sp = torch.empty(N, 3, dtype=torch.int32, device="cuda")
    sa = torch.empty(N, 2, dtype=torch.int32, device="cuda")
    ns = torch.empty(N, dtype=torch.int32, device="cuda")
    ws = torch.empty(table.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    for k in range(N):
        ik = ids.data_ptr() + 4 * T * k
        yb = y_b.data_ptr() + es * T * o * k
        L.lora_bgmv(table.handle, ik, T, dx, h, yb, o, 0)
        pk, spk, sak, nk = (perm.data_ptr() + 4 * T * k, sp.data_ptr() + 12 * k, sa.data_ptr() + 8 * k,
                            ns.data_ptr() + 4 * k)
        L.lora_build_segments(table.handle, ik, T, pk, spk, sak, nk)
        seg = L.make_segments(pk, spk, sak, nk, T, 2)
        L.lora_sgmv(table.handle, seg, dx, h, y_s.data_ptr() + es * T * o * k, o, 0)
        with option("split", 1):
            L.lora_sgmv(table.handle, seg, dx, h, y_x.data_ptr() + es * T * o * k, o, 0, ws, ws.numel())
    torch.cuda.synchronize()
    got = {name: torch_to_np(y, dtype).reshape(N, T, o) for name, y in (("bgmv", y_b), ("sgmv", y_s), ("split", y_x))}
    for k in range(N):
        ref = oracle.lora_delta(dtype, x, y0, assigns[k], A, B, scales)
        want = _rounded(ref, dtype)
        for name, g in got.items():
            assert np.array_equal(g[k].view(np.uint16 if dtype == "bf16" else np.uint32),
                                  want.view(np.uint16 if dtype == "bf16" else np.uint32)), (name, assigns[k])
    assert L.lora_get_status(table.handle) == (0, 0)
    table.close()


def _prefill_segments(T, seg_len, n):
    seg_ptr = torch.arange(0, T + 1, seg_len, dtype=torch.int32, device="cuda")
    seg_ad = torch.arange(n, dtype=torch.int32, device="cuda")
    num = torch.tensor([n], dtype=torch.int32, device="cuda")
    return L.make_segments(None, seg_ptr, seg_ad, num, T, n, seg_len), (seg_ptr, seg_ad, num)


def test_integer_inputs_tcgen05_paths_exact():
    """Contiguous segments of 256 tokens: the tcgen05 shrink and expand, and the fused base
    layer output, on integer inputs -- exact after the one rounding."""
    h, o, n, seg_len = 64, 128, 2, 256
    T = n * seg_len
    rng, A, B = _int_problem("bf16", h, o, (64, 32), seed=11)
    x = _store(rng.integers(-1, 2, size=(T, h)), "bf16")
    y0 = _store(rng.integers(-8, 9, size=(T, o)), "bf16")
    W = _store(rng.integers(-1, 2, size=(o, h)), "bf16")
    ids = np.repeat(np.arange(n, dtype=np.int32), seg_len)
    scales = (2.0, 0.25)
    table = L.AdapterTable([np_to_torch(a, "bf16").cuda() for a in A], [np_to_torch(b, "bf16").cuda() for b in B],
                           [64, 32], list(scales), h, o, L.LORA_BF16)
    seg, _keep = _prefill_segments(T, seg_len, n)
    dx = np_to_torch(x, "bf16").cuda()
    ws = torch.empty(table.workspace_bytes(T), dtype=torch.uint8, device="cuda")
    scratch = np_to_torch(y0, "bf16").cuda()
    names = kernels_launched(lambda: L.lora_sgmv(table.handle, seg, dx, h, scratch, o, 0, ws, ws.numel()))
    assert ran(names, "prefill_expand_kernel")
    y = np_to_torch(y0, "bf16").cuda()
    L.lora_sgmv(table.handle, seg, dx, h, y, o, 0, ws, ws.numel())
    torch.cuda.synchronize()
    want = _rounded(oracle.lora_delta("bf16", x, y0, ids, A, B, scales), "bf16")
    assert np.array_equal(torch_to_np(y, "bf16"), want)
    yb = np_to_torch(y0, "bf16").cuda()
    L.lora_sgmv_base(table.handle, seg, dx, h, np_to_torch(W, "bf16").cuda(), h, yb, o, 0, True, ws, ws.numel())
    torch.cuda.synchronize()
    want_b = _rounded(oracle.lora_base_delta("bf16", x, W, y0, ids, A, B, scales), "bf16")
    assert np.array_equal(torch_to_np(yb, "bf16"), want_b)
    table.close()


@pytest.mark.parametrize("path", ["bgmv", "sgmv", "split", "tcgen05", "base"])
def test_doubling_every_scale_doubles_the_delta_exactly(path):
    if path in ("tcgen05", "base"):
        wl = workloads.generate("prefill_sgmv", n=3, seg_len=256, shapes=(("up", 512, 384, 0),), delta_only=True)
    else:
        wl = workloads.generate("multirank_decode", T=96, n=24, shapes=(("q", 1024, 768, 0),), delta_only=True)
    dp = DeviceProj(wl)
    d = dp.d
    t2 = L.AdapterTable(d.A_ptrs, d.B_ptrs, d.ranks, [2 * s for s in d.scales], d.h, d.o, L.LORA_BF16, keep=d)
    outs = []
    for table in (dp.table, t2):
        y = dp.y()
        ws = dp.workspace()
        if path == "bgmv":
            L.lora_bgmv(table.handle, dp.ids, wl.T, d.x, d.h, y, d.o, 0, ws, ws.numel())
        elif path in ("sgmv", "split"):
            seg, _k = dp.segments()
            with option("split", 1 if path == "split" else 0):
                L.lora_sgmv(table.handle, seg, d.x, d.h, y, d.o, 0, ws, ws.numel())
        else:
            seg, _k = _prefill_segments(wl.T, 256, wl.n)
            if path == "tcgen05":
                L.lora_sgmv(table.handle, seg, d.x, d.h, y, d.o, 0, ws, ws.numel())
            else:
                Z = torch.zeros(d.o, d.h, dtype=torch.bfloat16, device="cuda")
                L.lora_sgmv_base(table.handle, seg, d.x, d.h, Z, d.h, y, d.o, 0, False, ws, ws.numel())
        torch.cuda.synchronize()
        outs.append(y.float())
    assert outs[0].abs().max() > 0
    assert torch.equal(outs[1], 2 * outs[0])
    t2.close()


@pytest.mark.parametrize("cluster", [0, 2])
def test_segment_order_shuffle_changes_no_bit(cluster):
    wl = workloads.generate("multirank_decode", T=200, n=40, shapes=(("q", 1024, 512, 0),))
    dp = DeviceProj(wl)
    seg, t = dp.segments()
    with option("decode_cluster", cluster):
        y_ref = dp.sgmv(dp.y(), seg)
        S = int(t["num_segs"].item())
        ptr = t["seg_ptr"][:S + 1].cpu().numpy()
        ad = t["seg_adapter"][:S].cpu().numpy()
        perm = t["perm"].cpu().numpy()
        order = np.random.default_rng(4).permutation(S)
        new_perm = np.concatenate([perm[ptr[s]:ptr[s + 1]] for s in order]).astype(np.int32)
        new_ptr = np.concatenate([[0], np.cumsum([ptr[s + 1] - ptr[s] for s in order])]).astype(np.int32)
        new_ad = ad[order].astype(np.int32)
        keep = [torch.from_numpy(a).cuda() for a in (new_perm, new_ptr, new_ad, np.array([S], np.int32))]
        seg2 = L.make_segments(keep[0], keep[1], keep[2], keep[3], wl.T, S)
        y2 = dp.sgmv(dp.y(), seg2)
    torch.cuda.synchronize()
    assert torch.equal(y_ref, y2)
    assert dp.status() == (0, 0)
