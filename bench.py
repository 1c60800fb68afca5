#!/usr/bin/env python
"""Throughput of the heterogeneous-batch LoRA delta on B200.

One step = one pass of the hot path over one batch of synthetic, seeded inputs.  The default
workload is the largest one-GPU configuration: an up_proj-shaped layer (4096 -> 14336), 8
contiguous segments of 512 tokens each with its own rank-64 bf16 adapter, scale 0.5, run
through ``lora_sgmv`` (the tcgen05 path).  Other workloads: ``--workload``.  The same JSON line
carries, under ``secondary``, the decode-form workloads (per-token ids on 4096 -> 4096,
multi-rank, many adapters over q/k/v/o), each timed the same way with its own roofline, and
under ``adapter_sweep`` the throughput as the number of distinct adapters in a 256-token batch
grows from 1 to 256.

Timing: the input set (adapter weights, x, y, ids) is replicated into C copies whose total
exceeds 4x the L2 size, and consecutive steps rotate through the copies, so every step reads
its weights from HBM.  Steps are captured into CUDA graphs (all C copies, and the first K % C),
each replayed once before timing.  The timed region is exactly K steps, bracketed by CUDA
events on the launching stream; it is repeated, with a 256 MB buffer written before each
repetition, and the median repetition is reported (max over ranks; a barrier and a synchronize
on both sides of the timed repetitions).  With ``torchrun`` each rank runs its own independent
batches (the path shards by tokens with no exchange): weak scaling.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from workloads import accounting  # noqa: E402

METRIC = "tokens/s of batched multi-LoRA delta; fraction of HBM roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024

DESCRIPTIONS = {
    "tiny_sgmv": "h=o=256, 4 adapters r8 fp32, 16 tokens uniform ids, s=2 (lora_sgmv)",
    "decode_bgmv": "q_proj 4096->4096, 32 adapters r16 bf16, 64 tokens uniform ids, s=2 (lora_bgmv)",
    "multirank_decode": "4096->4096, 128 adapters r in {8,16,32,64} bf16, 256 tokens Zipf(1.0), s=16/r "
                        "(lora_build_segments + lora_sgmv)",
    "prefill_sgmv": "up_proj 4096->14336, 8 contiguous segments x 512 tokens, r64 bf16, s=0.5 (lora_sgmv)",
    "many_adapter_qkvo": "q,o 4096->4096 and k,v 4096->1024, 1000 adapters r16 bf16, 512 tokens Zipf(0.8), "
                         "s=2 (lora_build_segments + 4 x lora_sgmv)",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about one second of work)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_sgmv", choices=list(workloads.WORKLOAD_NAMES))
    ap.add_argument("--copies", type=int, default=0, help="input copies rotated across steps (0: auto)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle CPU-baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=-1, help="end-to-end steps (-1: about 1.5 s; 0: skip)")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode-form lines and the distinct-adapter sweep")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying a graph")
    ap.add_argument("--sigma", default="none", choices=["none", "full", "diag"],
                    help="three-stage (compressed) form: a per-adapter Sigma_i between the A and B steps")
    ap.add_argument("--jd-clusters", type=int, default=0,
                    help="with --sigma: adapters share the A and B of adapter (i mod K), as compressed clusters do")
    ap.add_argument("--merge", type=int, default=1,
                    help="decode_bgmv: K adapters merged per token (weighted ensembles, lora_bgmv_merged)")
    ap.add_argument("--base", action="store_true",
                    help="prefill_sgmv: the layer output with a synthetic frozen base weight, x W^T plus the adapter "
                         "term, through lora_sgmv_base (tensor-core bound)")
    ap.add_argument("--grouped", action="store_true",
                    help="many_adapter_qkvo: one lora_sgmv_grouped launch for q, k, v, o (q, k, v reading one x) "
                         "instead of four lora_sgmv calls")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s sustained under the power cap (the kernels are timed over about a
    second of back-to-back steps): the measured sustained figure, else this machine's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        for key in ("bf16_tflops_sustained", "bf16_tflops"):
            if key in d:
                return float(d[key]), "measured (%s)" % key
    return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def tensor_roofline(flops_step, ms_step, launches_per_step, kname):
    peak, kind = measured_tensor_peak()
    achieved = flops_step / (ms_step / 1e3) / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": None,
            "peak_source": "%s, MEASURED_PEAKS.json" % kind if kind != "fallback"
            else "fallback 1.4 PFLOP/s sustained", "flops_per_step": flops_step, "kernel": kname,
            "basis": "whole step (%d launches): a lower bound on the dominant kernel's own rate" % launches_per_step}


def profile_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel (per step for workloads timed as a whole
    step) from the committed ncu summary, if the summary says it still matches the kernels."""
    path = os.path.join(ROOT, "profiles", "%s_ncu.md" % workload)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip()
    try:
        if vals.get("current", "yes").lower() != "yes":
            return None
        return float(vals.get("dram_bytes_per_launch") or vals["dram_bytes_per_step"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--id=%s" % gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks
# One process per GPU, each an independent replica with its own token batch (the path
# shards by tokens and exchanges nothing).  The job is as slow as its slowest rank.

def rank_seed(workload: str, rank: int) -> int:
    """Seed of rank `rank`'s batch: every replica draws its own inputs."""
    return workloads.SEED_BASE + workloads.WORKLOAD_NAMES.index(workload) + 1000 * rank


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest per-rank value (a time) over all ranks; the value itself without a group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processed `steps` steps in at most `ms` milliseconds."""
    return world * tokens_per_step * steps / (ms / 1e3)


# ----------------------------------------------------------------------------- our arm

class Copy:
    """One replica of the workload's inputs on the device plus its adapter tables."""

    def __init__(self, wl, L, torch, sigma="none", clusters=0, merge=1, base_w=None):
        from workloads.device import np_to_torch, upload_projection
        self.W = np_to_torch(base_w, wl.dtype).cuda() if base_w is not None else None
        self.projs = []
        self.tables = []
        self.sigma = []
        for pi, p in enumerate(wl.projections):
            d = upload_projection(p, wl.dtype)
            A, B, ranks = d.A_ptrs, d.B_ptrs, d.ranks
            if clusters > 0:   # compressed clusters: members use their leader's A and B
                cl = workloads.jd_clusters(wl.n, clusters)
                A, B, ranks = [A[c] for c in cl], [B[c] for c in cl], [ranks[c] for c in cl]
            t = L.AdapterTable(A, B, ranks, d.scales, p.h, p.o,
                               L.LORA_BF16 if wl.dtype == "bf16" else L.LORA_F32, keep=d)
            if sigma != "none":
                sg = [torch.from_numpy(a).cuda()
                      for a in workloads.draw_sigma(np.asarray(ranks), sigma, seed=wl.seed + 77 + pi)]
                t.set_sigma(L.LORA_SIGMA_FULL if sigma == "full" else L.LORA_SIGMA_DIAG, sg)
                self.sigma.append(sg)
            self.projs.append(d)
            self.tables.append(t)
        self.ids = torch.from_numpy(wl.ids).cuda()
        if merge > 1:
            m_ids, m_w = workloads.draw_merge(wl.ids, wl.n, merge, seed=wl.seed + 99)
            self.m_ids = torch.from_numpy(m_ids).cuda()
            self.m_w = torch.from_numpy(m_w).cuda()
        n, T = wl.n, wl.T
        self.seg_t = dict(perm=torch.empty(T, dtype=torch.int32, device="cuda"),
                          seg_ptr=torch.empty(n + 1, dtype=torch.int32, device="cuda"),
                          seg_adapter=torch.empty(n, dtype=torch.int32, device="cuda"),
                          num=torch.empty(1, dtype=torch.int32, device="cuda"))
        ws_bytes = max(t.workspace_bytes(T) for t in self.tables)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        if wl.name == "prefill_sgmv":
            seg_len = wl.spec.seg_len
            self.pf = dict(seg_ptr=torch.arange(0, T + 1, seg_len, dtype=torch.int32, device="cuda"),
                           seg_adapter=torch.arange(n, dtype=torch.int32, device="cuda"),
                           num=torch.tensor([n], dtype=torch.int32, device="cuda"))
            self.seg = L.make_segments(None, self.pf["seg_ptr"], self.pf["seg_adapter"], self.pf["num"], T, n, seg_len)
        else:
            s = self.seg_t
            self.seg = L.make_segments(s["perm"], s["seg_ptr"], s["seg_adapter"], s["num"], T, n)

    def nbytes(self):
        tot = self.ids.numel() * 4 + self.ws.numel()
        if self.W is not None:
            tot += self.W.numel() * self.W.element_size()
        for d in self.projs:
            tot += d.A_flat.numel() * d.A_flat.element_size() + d.B_flat.numel() * d.B_flat.element_size()
            tot += d.x.numel() * d.x.element_size() + d.y0.numel() * d.y0.element_size()
        return tot


def make_step(wl, L, grouped=False, merge=1, base=False):
    """Returns (step(copy, stream_handle), launches per step, name of the dominant kernel)."""
    name = wl.name
    T = wl.T
    if base:
        if name != "prefill_sgmv":
            raise SystemExit("--base applies to prefill_sgmv only")

        def step(c, s):
            d, t = c.projs[0], c.tables[0]
            L.lora_sgmv_base(t.handle, c.seg, d.x, d.h, c.W, d.h, d.y0, d.o, 0, False, c.ws, c.ws.numel(), s)
        return step, 2, "base_gemm_kernel (tcgen05, x W^T plus the adapter term in one accumulator)"
    if merge > 1:
        if name != "decode_bgmv":
            raise SystemExit("--merge applies to decode_bgmv only")

        def step(c, s):
            d, t = c.projs[0], c.tables[0]
            L.lora_bgmv_merged(t.handle, c.m_ids, c.m_w, T, merge, d.x, d.h, d.y0, d.o, 0, c.ws, c.ws.numel(), s)
        return step, merge, "lora_decode_kernel (fused, per-token ids, one pass per merged slot)"
    if grouped:
        if name != "many_adapter_qkvo":
            raise SystemExit("--grouped applies to many_adapter_qkvo only")
        xs_host = [q.x for q in wl.projections]
        src = [next(j for j, xa in enumerate(xs_host) if xa is xh) for xh in xs_host]   # first reader of each x

        def step(c, s):
            st = c.seg_t
            L.lora_build_segments(c.tables[0].handle, c.ids, T, st["perm"], st["seg_ptr"], st["seg_adapter"],
                                  st["num"], s)
            xs = [c.projs[i].x for i in src]
            L.lora_sgmv_grouped([t.handle for t in c.tables], c.seg, xs, [x.shape[1] for x in xs],
                                [d.y0 for d in c.projs], [d.o for d in c.projs], [0] * len(c.projs), c.ws,
                                c.ws.numel(), s)
        return step, 2, "lora_decode_kernel (fused, segments, 4 projections per launch)"

    if name == "decode_bgmv":
        def step(c, s):
            d, t = c.projs[0], c.tables[0]
            L.lora_bgmv(t.handle, c.ids, T, d.x, d.h, d.y0, d.o, 0, c.ws, c.ws.numel(), s)
        return step, 1, "lora_decode_kernel (fused, per-token ids)"
    if name in ("tiny_sgmv", "multirank_decode", "many_adapter_qkvo"):
        def step(c, s):
            st = c.seg_t
            L.lora_build_segments(c.tables[0].handle, c.ids, T, st["perm"], st["seg_ptr"], st["seg_adapter"],
                                  st["num"], s)
            for d, t in zip(c.projs, c.tables):
                L.lora_sgmv(t.handle, c.seg, d.x, d.h, d.y0, d.o, 0, c.ws, c.ws.numel(), s)
        return step, 1 + len(wl.projections), "lora_decode_kernel (fused, segments)"
    if name == "prefill_sgmv":
        def step(c, s):
            d, t = c.projs[0], c.tables[0]
            L.lora_sgmv(t.handle, c.seg, d.x, d.h, d.y0, d.o, 0, c.ws, c.ws.numel(), s)
        return step, 2, "prefill_shrink_kernel + prefill_expand_kernel (tcgen05)"
    raise ValueError(name)


class Timer:
    """Times exactly K steps of a workload through CUDA graphs of its rotating input copies.

    Graphs: one of all C copies (replayed K // C times) and one of the first K % C copies;
    both are replayed once before any timing, so no first-replay upload lands in a timed
    region.  The K-step region is repeated `reps` times; before each repetition a 256 MB
    buffer is written (outside the timed region) so no repetition starts with its inputs in
    L2.  Each repetition is bracketed by CUDA events on the launching stream; the median
    repetition is reported."""

    FLUSH_BYTES = 256 * 1024 * 1024

    def __init__(self, torch, copies, step, K, no_graph=False):
        self.torch, self.copies, self.step, self.K = torch, copies, step, K
        self.no_graph = no_graph
        self.stream = torch.cuda.Stream()
        self.sh = int(self.stream.cuda_stream)
        self.flush_buf = torch.empty(self.FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.g_full = self.g_rem = None

    def warm(self, W):
        torch, C = self.torch, len(self.copies)
        with torch.cuda.stream(self.stream):
            for i in range(W):
                self.step(self.copies[i % C], self.sh)
        torch.cuda.synchronize()
        if self.no_graph:
            return
        K = self.K
        if K >= C:
            self.g_full = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_full, stream=self.stream):
                for i in range(C):
                    self.step(self.copies[i], int(torch.cuda.current_stream().cuda_stream))
        if K % C:
            self.g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_rem, stream=self.stream):
                for i in range(K % C):
                    self.step(self.copies[i], int(torch.cuda.current_stream().cuda_stream))
        with torch.cuda.stream(self.stream):
            for g in (self.g_full, self.g_rem):
                if g is not None:
                    g.replay()
        torch.cuda.synchronize()

    def _region(self):
        C, K = len(self.copies), self.K
        if self.no_graph:
            for i in range(K):
                self.step(self.copies[i % C], self.sh)
            return
        for _ in range(K // C):
            self.g_full.replay()
        if self.g_rem is not None:
            self.g_rem.replay()

    def run(self, reps):
        """Returns the per-repetition region times (ms) of `reps` repetitions."""
        torch = self.torch
        evs = []
        with torch.cuda.stream(self.stream):
            for i in range(reps):
                self.flush_buf.fill_(i & 0xFF)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(self.stream)
                self._region()
                e1.record(self.stream)
                evs.append((e0, e1))
        torch.cuda.synchronize()
        return [float(a.elapsed_time(b)) for a, b in evs]

    def reps_for(self, seconds):
        """Repetitions that fill about `seconds` of GPU time (at least 5, at most 2000)."""
        t = self.run(2)
        per = max(1e-6, min(t) / 1e3 + 50e-6)
        return int(max(5, min(2000, seconds / per)))

    def release(self):
        self.g_full = self.g_rem = None
        self.flush_buf = None


def roofline_of(bytes_step, ms_step, launches_per_step, kname, traffic):
    peak, peak_kind = measured_peaks()
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    one = launches_per_step == 1
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "algorithmic_bytes_per_launch": bytes_step if one else None,
            "algorithmic_bytes_per_step": bytes_step,
            "kernel": kname,
            "kernel_ms_per_launch": round(ms_step, 6) if one else None,
            "basis": "step time (one launch per step)" if one else
            "whole step (%d launches): a lower bound on the dominant kernel's own rate" % launches_per_step}


def make_copies(wl, L, torch, args, plain=False):
    """C replicas of the inputs, C chosen so that together they exceed 4x the L2 size (at
    least 2).  `plain` ignores the three-stage / merged options (secondary lines)."""
    kw = {} if plain else dict(sigma=args.sigma, clusters=args.jd_clusters, merge=args.merge)
    if getattr(args, "base_w", None) is not None and not plain:
        kw["base_w"] = args.base_w
    first = Copy(wl, L, torch, **kw)
    per = first.nbytes()
    C = args.copies or max(2, min(256, -(-4 * L2_BYTES // per)))
    return [first] + [Copy(wl, L, torch, **kw) for _ in range(C - 1)], per


def free_copies(torch, copies):
    for c in copies:
        for t in c.tables:
            t.close()
    copies.clear()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def timed_workload(args, L, torch, wl, grouped, seconds, dist, K=None):
    """Median per-step time of one workload over repeated K-step regions (secondary lines)."""
    step, launches, kname = make_step(wl, L, grouped, 1)
    copies, per = make_copies(wl, L, torch, args, plain=True)
    C = len(copies)
    K = K or C * max(1, -(-32 // C))
    tm = Timer(torch, copies, step, K, args.no_graph)
    tm.warm(max(args.warmup, 3))
    reps = tm.reps_for(seconds)
    if dist:
        dist.barrier()
    times = tm.run(reps)
    ms = max_over_ranks(float(np.median(times)), dist, "cuda") / K
    tm.release()
    free_copies(torch, copies)
    return ms, launches, kname, C, per, K, reps


def secondary_lines(args, L, torch, dist, world):
    """The decode-form workloads, each timed on its own with its own roofline."""
    out = []
    for name, grouped in (("decode_bgmv", False), ("multirank_decode", False), ("many_adapter_qkvo", True)):
        if name == args.workload and grouped == args.grouped:
            continue
        wl = workloads.generate(name, seed=rank_seed(name, int(os.environ.get("RANK", "0"))))
        ms, launches, kname, C, per, K, reps = timed_workload(args, L, torch, wl, grouped, 0.4, dist)
        b = accounting.workload_bytes(wl, shared_x=grouped)
        traffic = profile_traffic(name + ("_grouped" if grouped else ""))
        out.append({"workload": "%s: %s" % (name, workload_description(name, grouped)),
                    "tokens_per_step": wl.T, "value": round(job_throughput(world, wl.T, 1, ms), 1),
                    "unit": UNIT, "ms_per_step": round(ms, 6), "steps": K, "repetitions": reps,
                    "algorithmic_bytes_per_step": b,
                    "l2": "rotating %d input copies, %.0f MB in total; 256 MB written between repetitions" % (
                        C, C * per / 1e6),
                    "roofline": roofline_of(b, ms, launches, kname, traffic)})
    if not args.base:
        out.append(base_layer_line(args, L, torch, dist, world))
    return out


def base_layer_line(args, L, torch, dist, world):
    """The prefill shape's layer output with a synthetic frozen base weight through
    lora_sgmv_base (tensor-core bound), and, for comparison only, the same result computed as
    a library GEMM (torch.matmul) followed by lora_sgmv."""
    wl = workloads.generate("prefill_sgmv", seed=rank_seed("prefill_sgmv", int(os.environ.get("RANK", "0"))))
    p0 = wl.projections[0]
    W = workloads.draw_base_weight(p0.o, p0.h, seed=wl.seed + 500)
    C = max(2, -(-4 * L2_BYTES // (2 * p0.o * p0.h + 2 * wl.T * (p0.h + p0.o))))
    copies = [Copy(wl, L, torch, base_w=W) for _ in range(C)]
    fused, launches, kname = make_step(wl, L, base=True)

    def unfused(c, s):   # comparison only: library GEMM, then the delta
        d, t = c.projs[0], c.tables[0]
        with torch.cuda.stream(torch.cuda.ExternalStream(s)):
            torch.matmul(d.x, c.W.t(), out=d.y0)
        L.lora_sgmv(t.handle, c.seg, d.x, d.h, d.y0, d.o, 0, c.ws, c.ws.numel(), s)

    res = {}
    for name, step in (("fused", fused), ("unfused", unfused)):
        K = C * max(1, -(-8 // C))
        tm = Timer(torch, copies, step, K, args.no_graph)
        tm.warm(max(args.warmup, 3))
        reps = tm.reps_for(0.5)
        if dist:
            dist.barrier()
        res[name] = (max_over_ranks(float(np.median(tm.run(reps))), dist, "cuda") / K, K, reps)
        tm.release()
    free_copies(torch, copies)
    ms, K, reps = res["fused"]
    flops = accounting.base_layer_flops(wl)
    return {"workload": "prefill_base: up_proj 4096->14336 layer output x W^T + s B A x with a synthetic frozen W, "
                        "8 segments x 512 tokens, r64 bf16 (lora_sgmv_base)",
            "tokens_per_step": wl.T, "value": round(job_throughput(world, wl.T, 1, ms), 1), "unit": UNIT,
            "ms_per_step": round(ms, 6), "steps": K, "repetitions": reps,
            "algorithmic_bytes_per_step": accounting.base_layer_bytes(wl),
            "l2": "rotating %d input copies; 256 MB written between repetitions" % C,
            "roofline": tensor_roofline(flops, ms, launches, kname),
            "comparison": {"what": "torch.matmul (cuBLAS) then lora_sgmv, same inputs, same timing",
                           "ms_per_step": round(res["unfused"][0], 6),
                           "fused_speedup": round(res["unfused"][0] / ms, 4)}}


def adapter_sweep(args, L, torch, dist, world):
    """Distinct adapters touched per batch (1 .. 256) at the decode layer shape: 4096 -> 4096,
    rank 16, 256 tokens, a table of 256 adapters, one lora_bgmv per step."""
    from workloads.device import upload_projection
    T, n = 256, 256
    wl = workloads.generate("decode_bgmv", T=T, n=n, seed=rank_seed("decode_bgmv", 0) + 5000)
    p = wl.projections[0]
    e = accounting.ELEM_BYTES[wl.dtype]
    per = sum(a.nbytes for a in (p.A_flat, p.B_flat, p.x, p.y0))
    C = max(2, -(-4 * L2_BYTES // per))
    dev = []
    for _ in range(C):
        d = upload_projection(p, wl.dtype)
        t = L.AdapterTable(d.A_ptrs, d.B_ptrs, d.ranks, d.scales, p.h, p.o, L.LORA_BF16, keep=d)
        dev.append((d, t))
    points = []
    for D in (1, 4, 16, 64, 256):
        ids_np = workloads.sweep_ids(T, n, D, seed=wl.seed + D)
        ids = torch.from_numpy(ids_np).cuda()

        def step(c, s, ids=ids):
            d, t = c
            L.lora_bgmv(t.handle, ids, T, d.x, d.h, d.y0, d.o, 0, None, 0, s)
        K = C * max(1, -(-32 // C))
        tm = Timer(torch, dev, step, K, args.no_graph)
        tm.warm(max(args.warmup, 3))
        reps = tm.reps_for(0.25)
        if dist:
            dist.barrier()
        ms = max_over_ranks(float(np.median(tm.run(reps))), dist, "cuda") / K
        tm.release()
        b = accounting.projection_bytes(T, p.h, p.o, (p.ranks[i] for i in np.unique(ids_np)), e)
        peak, _ = measured_peaks()
        gbs = b / (ms / 1e3) / 1e9
        points.append({"distinct_adapters": D, "value": round(job_throughput(world, T, 1, ms), 1),
                       "ms_per_step": round(ms, 6), "algorithmic_bytes_per_step": b,
                       "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)})
    for d, t in dev:
        t.close()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return {"shape": "4096 -> 4096, rank 16 bf16, 256 tokens, table of 256 adapters, lora_bgmv; "
                     "rotating %d input copies" % C, "unit": UNIT, "points": points}


def workload_description(name, grouped):
    d = DESCRIPTIONS[name]
    return d.replace("4 x lora_sgmv", "one lora_sgmv_grouped, q/k/v sharing x") if grouped else d


def run_ours(args, rank, world, local_rank):
    import torch
    import heterogeneous_adapters_sgmv_b200 as L
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist

    wl = workloads.generate(args.workload, seed=rank_seed(args.workload, rank))
    T = wl.T
    step, launches_per_step, kname = make_step(wl, L, args.grouped, args.merge, args.base)
    if args.jd_clusters and args.sigma == "none":
        raise SystemExit("--jd-clusters needs --sigma")
    bytes_step = accounting.workload_bytes(wl, shared_x=args.grouped, sigma=args.sigma, clusters=args.jd_clusters)
    if args.merge > 1:   # x and y once, every adapter any slot touches once
        m_ids, _m_w = workloads.draw_merge(wl.ids, wl.n, args.merge, seed=wl.seed + 99)
        bytes_step = accounting.merged_bytes(wl, m_ids)
    flops_step = accounting.workload_flops(wl)
    args.base_w = None
    if args.base:
        p0 = wl.projections[0]
        args.base_w = workloads.draw_base_weight(p0.o, p0.h, seed=wl.seed + 500)
        bytes_step = accounting.base_layer_bytes(wl)
        flops_step = accounting.base_layer_flops(wl)
    distinct = int(accounting.distinct_adapters(wl.ids).size)

    copies, ws_bytes = make_copies(wl, L, torch, args)
    C = len(copies)
    torch.cuda.synchronize()
    # the library's own launch counters on one eager step confirm the launches a step makes
    before = L.kernel_launches()
    step(copies[0], int(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    after = L.kernel_launches()
    counted = sum(after[k] - before[k] for k in after)
    if counted != launches_per_step:
        raise SystemExit("a step launched %d kernels, expected %d" % (counted, launches_per_step))
    K = args.steps
    if K <= 0:   # about 20 ms of work per repetition, a whole number of copy rotations
        tm0 = Timer(torch, copies, step, C, args.no_graph)
        tm0.warm(3)
        per = min(tm0.run(3)) / C
        tm0.release()
        K = max(C, int(20.0 / max(per, 1e-4)) // C * C)
    W = max(args.warmup, 3)

    tm = Timer(torch, copies, step, K, args.no_graph)
    tm.warm(W)
    reps = tm.reps_for(1.0)

    gpu_id = torch.cuda.get_device_properties(local_rank).uuid
    gpu_id = "GPU-%s" % gpu_id if not str(gpu_id).startswith("GPU-") else str(gpu_id)
    if dist:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    time.sleep(0.3)   # let the sampler start before the timed region
    times = tm.run(reps)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist:
        dist.barrier(device_ids=[local_rank])
    ms = max_over_ranks(float(np.median(times)), dist, "cuda")
    ms_step = ms / K
    value = job_throughput(world, T, K, ms)
    tm.release()

    traffic = profile_traffic(args.workload + ("_grouped" if args.grouped else "")) if not (
        args.sigma != "none" or args.merge > 1 or args.base) else None
    roofline = roofline_of(bytes_step, ms_step, launches_per_step, kname, traffic)
    if args.base:
        roofline = tensor_roofline(flops_step, ms_step, launches_per_step, kname)

    # end to end through the C ABI with host buffers: H2D inputs, the call, D2H of y.  Two
    # device buffer sets and three streams, as a serving loop would run it: step i + 1's inputs
    # go in (copy engine, host to device) while step i computes and step i - 1's output comes
    # out (the other copy engine); every step still copies all of its inputs in and its result out.
    e2e = None
    if args.e2e_steps != 0:
        nb = 2 if len(copies) >= 2 else 1
        bufs = copies[:nb]
        hx = [torch.empty_like(p.x, device="cpu").pin_memory() for p in bufs[0].projs]
        hy = [torch.empty_like(p.y0, device="cpu").pin_memory() for p in bufs[0].projs]
        hout = [[torch.empty_like(p.y0, device="cpu").pin_memory() for p in bufs[0].projs] for _ in range(nb)]
        hids = torch.from_numpy(wl.ids).pin_memory()
        for i, p in enumerate(bufs[0].projs):
            hx[i].copy_(p.x)
            hy[i].copy_(p.y0)
        h2d = sum(t.numel() * t.element_size() for t in hx + hy) + hids.numel() * 4
        d2h = sum(t.numel() * t.element_size() for t in hout[0])
        s_in, s_run, s_out = torch.cuda.Stream(), tm.stream, torch.cuda.Stream()
        sh = tm.sh
        out_done = [None] * nb

        def e2e_step(k):
            b = k % nb
            c = bufs[b]
            with torch.cuda.stream(s_in):
                if out_done[b] is not None:
                    s_in.wait_event(out_done[b])   # this buffer's previous result is out
                c.ids.copy_(hids, non_blocking=True)
                for i, p in enumerate(c.projs):
                    p.x.copy_(hx[i], non_blocking=True)
                    p.y0.copy_(hy[i], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ev_in)
                step(c, sh)
                ev_run = torch.cuda.Event()
                ev_run.record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run)
                for i, p in enumerate(c.projs):
                    hout[b][i].copy_(p.y0, non_blocking=True)
                out_done[b] = torch.cuda.Event()
                out_done[b].record(s_out)

        for k in range(W):
            e2e_step(k)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e2e_step(0)
        torch.cuda.synchronize()
        Ke = args.e2e_steps if args.e2e_steps > 0 else int(max(20, min(5000, 1.5 / max(time.perf_counter() - t0, 1e-5))))
        if dist:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for k in range(Ke):
            e2e_step(k)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
        ems = max_over_ranks(float(e0.elapsed_time(e1)), dist, "cuda")
        e2e = {"value": round(job_throughput(world, T, Ke, ems), 1), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": Ke, "ms_per_step": round(ems / Ke, 6),
               "path": "pinned host -> cudaMemcpyAsync (copy stream) -> C-ABI call (compute stream) -> "
                       "cudaMemcpyAsync (second copy stream) -> pinned host; %d device buffer sets" % nb}
    pdl = bool(L.lora_get_option("pdl"))
    free_copies(torch, copies)

    secondary = secondary_lines(args, L, torch, dist, world) if not args.no_secondary else None
    sweep = adapter_sweep(args, L, torch, dist, world) if not args.no_secondary else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)
        if args.sigma != "none":
            cpu["sample"] += "; two-stage oracle (the r x r Sigma step adds under 1 % of the work)"

    codes = {"bf16": "bf16", "f32": "f32"}
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_step, 6), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": codes[wl.dtype], "data": "synthetic (seeded; random adapter weights and activations)",
        "config": {"workload": "%s: %s" % (args.workload, workload_description(args.workload, args.grouped)),
                   "tokens_per_step": T, "distinct_adapters_per_step": distinct,
                   "algorithmic_bytes_per_step": bytes_step, "flops_per_step": flops_step,
                   "l2": "rotating %d input copies, %.0f MB in total against a 126 MB L2; a 256 MB buffer is "
                         "written before each timed repetition" % (C, C * ws_bytes / 1e6),
                   "timing": "median of %d repetitions of the %d-step region (graphs warmed before timing)" % (
                       reps, K),
                   "graph": not args.no_graph, "pdl": pdl,
                   "sigma": args.sigma, "jd_clusters": args.jd_clusters, "merge_slots": args.merge,
                   "parallelism": "replicas x%d (independent token batches, no collective)" % world},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": int(K * launches_per_step),
        "secondary": secondary,
        "adapter_sweep": sweep,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_tokens_per_s(wl, T_sample: int, seconds: float, threads: int = 0):
    import oracle
    sub = sample_workload(wl, T_sample)
    reps, t0 = 0, time.perf_counter()
    while True:
        for pi in range(len(sub.projections)):
            oracle.workload_reference(sub, pi, threads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return reps * T_sample / el, reps, el


def sample_workload(wl, T_sample: int):
    """The first T_sample tokens of the batch (same adapters, same weights)."""
    import copy
    if T_sample >= wl.T:
        return wl
    sub = copy.copy(wl)
    sub.ids = wl.ids[:T_sample].copy()
    sub.T = T_sample
    sub.projections = []
    for p in wl.projections:
        q = copy.copy(p)
        q.x = p.x[:T_sample]
        q.y0 = p.y0[:T_sample]
        sub.projections.append(q)
    return sub


def cpu_baseline(wl, seconds: float):
    """The oracle as it stands on the host cores: all threads (OpenMP over tokens) for about
    two thirds of `seconds`, then one thread for the rest."""
    import oracle
    threads = oracle.max_threads()
    out = {}
    for nthr, budget in ((threads, seconds * 2 / 3), (1, seconds / 3)):
        # calibrate on a small sample, then size the sample so one pass is a fraction of the budget
        v, _reps, _el = _oracle_tokens_per_s(wl, min(wl.T, 8), 0.2, nthr)
        T_sample = int(max(1, min(wl.T, budget / 4 * v)))
        v, reps, el = _oracle_tokens_per_s(wl, T_sample, budget, nthr)
        out[nthr if nthr == 1 else "all"] = (v, T_sample, reps, el)
    v, T_sample, reps, el = out["all"]
    v1, T1, reps1, el1 = out[1]
    return {"value": round(v, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": "first %d of %d tokens of one batch, all projections, repeated %d times (%.1f s), "
                      "fp64 C loop with OpenMP over tokens" % (T_sample, wl.T, reps, el),
            "one_thread": {"value": round(v1, 2), "unit": UNIT, "cores": 1,
                           "sample": "first %d tokens, repeated %d times (%.1f s)" % (T1, reps1, el1)}}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    wl = workloads.generate(args.workload)
    threads = oracle.max_threads()
    K, W = (args.steps if args.steps > 0 else 20), max(args.warmup, 3)
    # size one step (a bounded sample of the batch) so that W + K steps take about a minute
    v, _r, _e = _oracle_tokens_per_s(wl, min(wl.T, 4), 0.2, threads)
    per_tok = 1.0 / v
    T_sample = int(max(1, min(wl.T, 60.0 / (K + W) / per_tok)))
    sub = sample_workload(wl, T_sample)
    for _ in range(W):
        for pi in range(len(sub.projections)):
            oracle.workload_reference(sub, pi, threads=threads)
    t0 = time.perf_counter()
    for _ in range(K):
        for pi in range(len(sub.projections)):
            oracle.workload_reference(sub, pi, threads=threads)
    el = time.perf_counter() - t0
    value = K * T_sample / el
    out = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
           "ms_per_step": round(el / K * 1e3, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
           "config": {"workload": "%s: %s" % (args.workload, DESCRIPTIONS[args.workload]),
                      "tokens_per_step": T_sample},
           "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": "first %d of %d tokens per step" % (T_sample, wl.T)},
           "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
