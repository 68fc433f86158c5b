#!/usr/bin/env python3
"""Benchmark of the 1-bit group-128 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Headline workload (one "step"): the decode GEMV sweep -- shapes 4096x4096,
11008x4096 and 4096x11008 (out x in) at batch 1, 4 and 8, weights N(0, 0.02)
binarised to 1-bit group-128 with fp16 scales, activations bf16 N(0, 1).  Each
(shape, batch) pair runs R back-to-back launches (one CUDA graph) over R
rotating copies of the packed weights whose total exceeds 4x the L2 size, so
every launch streams its weights from HBM.  value = packed weight bytes moved
/ device time (GB/s, all ranks, max-over-ranks time).

Also measured and reported under "rows" (outside the timed steps): the
prefill GEMM (M = 2048) TFLOP/s per shape, with an L2 flush before every
launch; the MoE layer tokens/s and the DBF chain when those calls exist.

--impl reference times the CPU oracle (fp64 numpy, the repository's test
oracle) on the host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "1-bit GEMV HBM GB/s (% of peak); prefill GEMM TFLOP/s; MoE-layer tokens/s"
GEMV_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
GEMV_BATCHES = [1, 4, 8]
GEMM_SHAPES = [(14336, 4096), (4096, 14336), (14336, 14336)]
GEMM_M = 2048
WORKLOAD = ("decode GEMV sweep: (out x in) 4096x4096, 11008x4096, 4096x11008 at B = 1, 4, 8; "
            "1-bit signs + fp16 scale per 128 weights; x bf16 N(0,1); W N(0,0.02)")
KERNEL_OF_CHOICE = {"flat": "gemv_flat_kernel", "flat16": "gemv_flat_kernel", "direct": "gemv_direct_kernel",
                    "direct16": "gemv_direct_kernel", "tc": "gemv_tc_kernel", "ring": "gemv_kernel"}
# DRAM bytes of one launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# ncu captures of the decode products, per (N, K, B) pair and kernel choice
# (profiles/ names each capture and its command).  A pair's own figure is
# used as is; the line's traffic is the launch-weighted mean over the
# dominant kernel's pairs, reported only when every one of them has a
# capture for the kernel it chose.
CAPTURED_TRAFFIC = {
    # (N, K, B, choice): bytes per launch (mean over the pair's launches of one
    # eager sweep, profiles/gemv_sweep_traffic.md)
    (4096, 4096, 1, "flat/1"): 2437361,
    (4096, 4096, 4, "flat16/1"): 2462227,
    (4096, 4096, 8, "flat16/1"): 2494788,
    (11008, 4096, 1, "flat/1"): 6443886,
    (11008, 4096, 4, "flat/1"): 6465972,
    (11008, 4096, 8, "flat/1"): 6498901,
    (4096, 11008, 1, "flat16/2"): 6462866,
    (4096, 11008, 4, "flat16/1"): 6498892,
    (4096, 11008, 8, "flat16/1"): 6586883,
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def packed_bytes(N: int, K: int) -> int:
    return N * K // 8 + N * (K // 128) * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock / throttle-reason sampling (NVML, every 10 ms) during the timed region."""

    # NVML clocks-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, pci_bus_id: str | None):
        self.pci = pci_bus_id
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByPciBusId(self.pci) if self.pci else nv.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
        except Exception as e:  # NVML missing: report unsampled
            self.err = repr(e)
        return self

    def _poll(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed

def _backend() -> str:
    """nccl on GPUs; W1_BENCH_BACKEND=gloo runs the rank logic on CPU (tests)."""
    return os.environ.get("W1_BENCH_BACKEND", "nccl")


def _reduce_device() -> str:
    return "cpu" if _backend() == "gloo" else "cuda"


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group(_backend(), timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value: float) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(world, value: float) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ GPU arm

class EagerChain:
    """Stands in for a captured graph: replay() issues the launches directly."""

    def __init__(self, fn):
        self.fn = fn

    def replay(self):
        self.fn()


def build_gemv_sweep(torch, ops, synth, l2_bytes: int, eager: bool = False):
    """Packed weight copies + one CUDA graph of back-to-back launches per pair
    (eager=True: the same launches issued one by one, for ncu launch lists)."""
    dev = torch.device("cuda")
    stream = torch.cuda.Stream()
    combos = []
    for (N, K) in GEMV_SHAPES:
        W, _ = synth.gemv_case(N, K, 1)
        Wd = torch.from_numpy(W).to(dev)
        s0, c0 = ops.w1_pack(Wd)
        del Wd
        pb = packed_bytes(N, K)
        R = max(64, int(math.ceil(4 * l2_bytes / pb)))
        signs = [s0] + [s0.clone() for _ in range(R - 1)]
        scales = [c0] + [c0.clone() for _ in range(R - 1)]
        for B in GEMV_BATCHES:
            x = torch.from_numpy(synth.activations_bf16(synth.rng(100 + B), B, K).view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((B, N), dtype=torch.float32, device=dev)
            # eager warm-up (plans the launch, sets kernel attributes)
            with torch.cuda.stream(stream):
                for r in range(3):
                    ops.w1_gemv(signs[r], scales[r], x, y)
            stream.synchronize()
            def chain(static, signs=signs, scales=scales, x=x, y=y, R=R):
                for r in range(R):
                    ops.w1_gemv(signs[r], scales[r], x, y, static_weights=static)
            with torch.cuda.stream(stream):
                ops.w1_gemv(signs[0], scales[0], x, y, static_weights=True)
            stream.synchronize()
            if eager:
                g = EagerChain(lambda c=chain: c(False))
                gs = EagerChain(lambda c=chain: c(True))
            else:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    chain(False)
                # the same chain with W1_GEMV_STATIC_WEIGHTS (weights written long before)
                gs = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gs, stream=stream):
                    chain(True)
            combos.append({"N": N, "K": K, "B": B, "R": R, "graph": g, "graph_static": gs, "x": x, "y": y,
                           "signs": signs, "scales": scales, "bytes": pb})
    torch.cuda.synchronize()
    return combos, stream


def time_gemv_steps_detailed(torch, combos, stream, steps: int, warmup: int, world: int):
    """Timed region: `steps` sweeps; per-pair device time via events on the stream."""
    for _ in range(warmup):
        with torch.cuda.stream(stream):
            for cb in combos:
                cb["graph"].replay()
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in combos] for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("w1_timed")  # ncu --nvtx-include w1_timed/ selects these launches
    with torch.cuda.stream(stream):
        start.record(stream)
        for s in range(steps):
            for i, cb in enumerate(combos):
                evs[s][i][0].record(stream)
                cb["graph"].replay()
                evs[s][i][1].record(stream)
        end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(end)
    per_pair_ms = [sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(steps)) for i in range(len(combos))]
    return total_ms, per_pair_ms


def time_gemv_static(torch, combos, stream, reps: int = 3):
    """Per-pair device time of the W1_GEMV_STATIC_WEIGHTS chains (outside the timed steps)."""
    out = []
    for cb in combos:
        with torch.cuda.stream(stream):
            cb["graph_static"].replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                cb["graph_static"].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) * 1e3 / (reps * cb["R"]))
    return out


def time_gemv_floor(torch, ops, combos, stream, reps: int = 3):
    """Per pair, the per-launch floor: w1_stream_probe over the same rotating
    weight copies (sign words + scales), in the same CUDA-graph form as the
    products (back-to-back launches, programmatic dependent launch), with the
    loads after the dependency wait (as the headline chain) and before it (as
    W1_GEMV_STATIC_WEIGHTS).  Outside the timed steps."""
    dev = torch.device("cuda")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ctas = 2 * sms
    out = torch.zeros(ctas, dtype=torch.int32, device=dev)
    res = []
    for cb in combos:
        us = {}
        for early in (False, True):
            def chain(cb=cb, early=early):
                for r in range(cb["R"]):
                    ops.w1_stream_probe(cb["signs"][r], cb["scales"][r], out, ctas, early, stream=stream)
            chain()
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                chain()
            with torch.cuda.stream(stream):
                g.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            us["static" if early else "plain"] = e0.elapsed_time(e1) * 1e3 / (reps * cb["R"])
            del g
        res.append(us)
    return res


def gemv_e2e(torch, ops, combos, steps: int):
    """The same sweep through the public API (eager w1_gemv calls, no graphs).
    Every step copies its inputs host->device from pinned memory (each pair's
    x) and reads its results back device->host (each pair's y)."""
    stream = torch.cuda.Stream()
    host = []
    for cb in combos:
        xh = cb["x"].cpu().pin_memory()
        yh = torch.empty(cb["y"].shape, dtype=torch.float32).pin_memory()
        host.append((xh, yh))
    h2d = d2h = 0
    launches = 0
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            for cb, (xh, yh) in zip(combos, host):
                cb["x"].copy_(xh, non_blocking=True)
                h2d += xh.numel() * 2
                for r in range(cb["R"]):
                    ops.w1_gemv(cb["signs"][r], cb["scales"][r], cb["x"], cb["y"])
                    launches += 1
                yh.copy_(cb["y"], non_blocking=True)
                d2h += yh.numel() * 4
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    total_bytes = sum(cb["bytes"] * cb["R"] for cb in combos) * steps
    return {"value": total_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d // steps, "d2h_bytes_per_step": d2h // steps,
            "ms_per_step": ms / steps, "launches": launches}


def gemv_one(torch, ops, synth, shape: str, launches: int = 4):
    """A few eager launches of one GEMV (N, K, B): the small case for ncu."""
    N, K, B = (int(v) for v in shape.split(","))
    W, _ = synth.gemv_case(N, K, 1)
    s, c = ops.w1_pack(torch.from_numpy(W).cuda())
    x = torch.from_numpy(synth.activations_bf16(synth.rng(100 + B), B, K).view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty((B, N), dtype=torch.float32, device="cuda")
    ops.w1_gemv(s, c, x, y)  # the first call chooses the kernel (timing runs)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("w1_timed")  # the chosen kernel's launches, for ncu --nvtx-include
    for _ in range(launches):
        ops.w1_gemv(s, c, x, y)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    return {"N": N, "K": K, "B": B, "launches": launches, "choice": ops.gemv_choice(N, K, B)}


def gemm_rows(torch, ops, synth, peaks, iters: int = 8):
    dev = torch.device("cuda")
    flush = torch.empty(int(512 * 2 ** 20), dtype=torch.uint8, device=dev)
    rows = []
    for (N, K) in GEMM_SHAPES:
        W, x = synth.gemm_case(GEMM_M, N, K)
        Wd = torch.from_numpy(W).to(dev)
        s, c = ops.w1_pack(Wd)
        del Wd
        xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((GEMM_M, N), dtype=torch.float32, device=dev)
        ws = ops.gemm_workspace(GEMM_M, K, device=dev)
        for _ in range(3):
            ops.w1_gemm(s, c, xd, y, workspace=ws)
        torch.cuda.synchronize()
        times = []
        for _ in range(iters):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            ops.w1_gemm(s, c, xd, y, workspace=ws)
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        flops = 2.0 * GEMM_M * N * K
        tf = flops / (ms * 1e-3) / 1e12
        rows.append({"M": GEMM_M, "N": N, "K": K, "ms": ms, "TFLOP/s": tf,
                     "frac_bf16_burst": tf / peaks["bf16_tflops"]})
        del s, c, xd, y, ws
    torch.cuda.synchronize()
    return rows


MOE = dict(T=512, H=2048, I=1024, E=64, top_k=8)
MOE_DECODE_T = (1, 4, 8, 16)   # decode-regime batches
DBF_BATCHES = [1, 2, 4, 8, 512]


def moe_rows(torch, ops, synth, peaks, iters: int = 8, only_t: int | None = None):
    """Routed MoE layer (OLMoE-like): tokens/s and TFLOP/s, L2 flushed per call.
    only_t: just that decode batch (a small case for ncu), no 512-token layer."""
    dev = torch.device("cuda")
    T, H, I, E, K = MOE["T"], MOE["H"], MOE["I"], MOE["E"], MOE["top_k"]
    x, logits, gate, up, down = synth.moe_case(T=T, H=H, I=I, E=E)

    def pack(Wt):
        s, c = ops.w1_pack(torch.from_numpy(Wt.reshape(-1, Wt.shape[-1])).to(dev))
        return s.view(E, Wt.shape[1], -1), c.view(E, Wt.shape[1], -1)
    G, U, D = pack(gate), pack(up), pack(down)
    del gate, up, down
    xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    ld = torch.from_numpy(logits).to(dev)
    ws = ops.moe_workspace(T, H, I, E, K)
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    flush = torch.empty(int(512 * 2 ** 20), dtype=torch.uint8, device=dev)
    for _ in range(0 if only_t else 3):
        ops.w1_moe_grouped(xd, ld, G, U, D, K, out=out, workspace=ws)
    torch.cuda.synchronize()
    times = [] if not only_t else [float("nan")]
    for _ in range(0 if only_t else iters):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        ops.w1_moe_grouped(xd, ld, G, U, D, K, out=out, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    flops = 2.0 * T * K * 3 * H * I
    tf = flops / (ms * 1e-3) / 1e12
    row = {"T": T, "H": H, "I": I, "E": E, "top_k": K, "ms": ms, "tokens/s": T / (ms * 1e-3),
           "TFLOP/s": tf, "frac_bf16_burst": tf / peaks["bf16_tflops"], "launches_per_call": 7}
    # decode regime: Td tokens of the same batch, a different token window
    # per call, each call one CUDA graph replay (no host time inside the
    # events) after an L2 flush; HBM-bound on the experts' packed weights that
    # the call touches.  Both decode forms: per-route products and the
    # products grouped by expert (moe_path knob).
    per_expert = 3 * packed_bytes(I, H)  # gate, up (I x H) and down (H x I) have the same packed size
    ids_all = np.argsort(-logits, axis=1, kind="stable")[:, :K]
    st = torch.cuda.Stream()
    decode = []
    for Td in (MOE_DECODE_T if not only_t else (only_t,)):
        wsd = ops.moe_workspace(Td, H, I, E, K)
        outd = torch.empty((Td, H), dtype=torch.float32, device=dev)
        windows = [(i * Td) % (T - Td + 1) for i in range(iters)]
        touched = [len(np.unique(ids_all[w0:w0 + Td])) * per_expert for w0 in windows]
        entry = {"T": Td}
        for form in ("decode", "grouped"):
            ops.set_knob("moe_path", form)
            try:
                call = lambda w0: ops.w1_moe_grouped(xd[w0:w0 + Td], ld[w0:w0 + Td], G, U, D, K, out=outd,
                                                     workspace=wsd, stream=st)
                with torch.cuda.stream(st):
                    for w0 in windows[:2]:
                        call(w0)
                st.synchronize()
                graphs = []
                for w0 in windows:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=st):
                        call(w0)
                    graphs.append(g)
                tms = []
                for g in graphs:
                    with torch.cuda.stream(st):
                        flush.zero_()
                        a = torch.cuda.Event(enable_timing=True)
                        b = torch.cuda.Event(enable_timing=True)
                        a.record(st)
                        g.replay()
                        b.record(st)
                    st.synchronize()
                    tms.append(a.elapsed_time(b))
                del graphs
            finally:
                ops.set_knob("moe_path", None)
            dms = statistics.median(tms)
            gbs = float(np.mean(touched)) / (dms * 1e-3) / 1e9
            entry[form] = {"us": round(dms * 1e3, 2), "tokens/s": round(Td / (dms * 1e-3), 1),
                           "weight_GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                           "launches_per_call": (2 if Td <= 4 else 3) if form == "decode" else 4}
        decode.append(entry)
    row["decode"] = decode
    return row


def dbf_rows(torch, ops, synth, peaks, l2_bytes: int, iters: int = 5, only_b: int | None = None):
    """DBF chain 4096^3: B = 1, 8 as GB/s of sign bytes (rotating copies > 4x L2,
    CUDA graph of back-to-back calls); B = 512 as TFLOP/s (L2 flushed)."""
    dev = torch.device("cuda")
    m = r = n = 4096
    rows = []
    for B in (DBF_BATCHES if not only_b else (only_b,)):
        a, B1, mid, B2, b, x = synth.dbf_case(m=m, r=r, n=n, B=B)
        to16 = lambda v: torch.from_numpy(v.view(np.int16)).to(dev).view(torch.float16)
        tow = lambda v: torch.from_numpy(v.view(np.int32)).to(dev)
        ad, md, bd = to16(a), to16(mid), to16(b)
        xd = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        y = torch.empty((B, m), dtype=torch.float32, device=dev)
        ws = ops.dbf_workspace(m, r, n, B)
        sign_bytes = (m * r + r * n) // 8
        alg_bytes = sign_bytes + 2 * (m + r + n)
        flops = 2.0 * B * (r * n + m * r)
        if B <= 8:
            R = max(16, int(math.ceil(4 * l2_bytes / sign_bytes)))
            B1s = [tow(B1)] + [None] * (R - 1)
            B2s = [tow(B2)] + [None] * (R - 1)
            for i in range(1, R):
                B1s[i] = B1s[0].clone()
                B2s[i] = B2s[0].clone()
            st = torch.cuda.Stream()

            def graph_us():
                with torch.cuda.stream(st):
                    for i in range(3):
                        ops.dbf_apply(ad, B1s[i], md, B2s[i], bd, xd, y=y, workspace=ws)
                st.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=st):
                    for i in range(R):
                        ops.dbf_apply(ad, B1s[i], md, B2s[i], bd, xd, y=y, workspace=ws)
                g.replay()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(iters):
                    g.replay()
                e1.record()
                torch.cuda.synchronize()
                return e0.elapsed_time(e1) * 1e3 / (iters * R)

            us = graph_us()
            gbs = alg_bytes / (us * 1e-6) / 1e9
            row = {"B": B, "us_per_call": round(us, 3), "GB/s": round(gbs, 1),
                   "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "calls": R}
            # the small-batch chain forms side by side (fused kernel vs two launches)
            forms = {}
            for form, core, warps in (("fused", None, None), ("twostep", None, None), ("twostep", "direct", None),
                                      ("twostep", None, 8)):
                if warps and B <= 2:
                    continue  # 8 warps is already the default there
                ops.set_knob("dbf_path", form)
                if core:
                    ops.set_knob("dbf_core", core)
                if warps:
                    ops.set_knob("dbf_warps", warps)
                try:
                    key = form + ("_" + core if core else "") + (f"_w{warps}" if warps else "")
                    forms[key] = round(graph_us(), 3)
                finally:
                    ops.set_knob("dbf_path", None)
                    ops.set_knob("dbf_core", None)
                    ops.set_knob("dbf_warps", None)
            row["us_by_form"] = forms
            # split rank: r partitioned over the CTAs of a cluster in U . h (two-launch form)
            splits = {}
            for sp in (1, 2, 4, 8):
                ops.set_knob("dbf_path", "twostep")
                ops.set_knob("dbf_rank_split", sp)
                try:
                    splits[str(sp)] = round(graph_us(), 3)
                except RuntimeError:
                    splits[str(sp)] = None  # no plan with this split for the shape
                finally:
                    ops.set_knob("dbf_path", None)
                    ops.set_knob("dbf_rank_split", None)
            row["us_twostep_by_rank_split"] = splits
            rows.append(row)
            del B1s, B2s
        else:
            B1d, B2d = tow(B1), tow(B2)
            flush = torch.empty(int(512 * 2 ** 20), dtype=torch.uint8, device=dev)
            for _ in range(2):
                ops.dbf_apply(ad, B1d, md, B2d, bd, xd, y=y, workspace=ws)
            torch.cuda.synchronize()
            times = []
            for _ in range(iters):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                ops.dbf_apply(ad, B1d, md, B2d, bd, xd, y=y, workspace=ws)
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            ms = statistics.median(times)
            tf = flops / (ms * 1e-3) / 1e12
            rows.append({"B": B, "ms": ms, "TFLOP/s": tf, "frac_bf16_burst": tf / peaks["bf16_tflops"]})
    torch.cuda.synchronize()
    return rows


OKT_FACTORS = {4096: (64, 64), 11008: (86, 128)}


def okt_rows(torch, ops, synth, combos, stream, reps: int = 3):
    """Rotated-activation decode products on the sweep's pairs and weight copies
    (timing only: any packed matrix times the same): per call, w1_okt_gemv
    (rotation + product, weights static), w1_okt_rotate alone, and the plain
    static-weights product on bf16 x for comparison.  CUDA graphs of R
    back-to-back calls over the pair's rotating copies, CUDA events."""
    dev = torch.device("cuda")
    rows = []

    def graph_us(fn, R):
        with torch.cuda.stream(stream):
            for r in range(3):
                fn(r)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(R):
                fn(r)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (reps * R)

    for cb in combos:
        N, K, B, R = cb["N"], cb["K"], cb["B"], cb["R"]
        n1, n2 = OKT_FACTORS[K]
        g = synth.rng(500 + K)
        H = torch.from_numpy(synth.orthogonal_f32(g, n1)).to(dev)
        Rm = torch.from_numpy(synth.orthogonal_f32(g, n2)).to(dev)
        xr = torch.empty((B, K), dtype=torch.float32, device=dev)
        x, y = cb["x"], cb["y"]
        full = graph_us(lambda r: ops.w1_okt_gemv(cb["signs"][r], cb["scales"][r], H, Rm, x, y=y, x_rot=xr,
                                                  static_weights=True), R)
        rot = graph_us(lambda r: ops.w1_okt_rotate(H, Rm, x, x_rot=xr), R)
        plain = graph_us(lambda r: ops.w1_gemv(cb["signs"][r], cb["scales"][r], x, y, static_weights=True), R)
        rows.append({"N": N, "K": K, "B": B, "n1": n1, "n2": n2, "okt_gemv_us": round(full, 3),
                     "rotate_us": round(rot, 3), "gemv_static_us": round(plain, 3),
                     "added_us": round(full - plain, 3),
                     "okt_weight_GB/s": round(cb["bytes"] / (full * 1e-6) / 1e9, 1)})
    torch.cuda.synchronize()
    return rows


FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # CUDA-core FMA: SMs x lanes x 2 flops x max clock


def measure_rows(torch, ops, synth, peaks, iters: int = 5):
    """Approximation residuals on the 4096 x 4096 matrices (each call timed as
    one CUDA graph replay after an L2 flush): the sign-code
    residual sums (GB/s of W and packed bytes read), the DBF
    residual (fp32 TFLOP/s of the reconstruction, 2 m n r), 32-iteration
    power iteration, and the relative Frobenius / spectral residuals of the
    1-bit code on the synthetic Gaussian matrix."""
    dev = torch.device("cuda")
    m = n = r = 4096
    W, _ = synth.gemv_case(m, n, 1)
    Wd = torch.from_numpy(W).to(dev)
    signs, scales = ops.w1_pack(Wd)
    a, B1, mid, B2, b, _ = synth.dbf_case(m=m, r=r, n=n, B=1)
    to16 = lambda v: torch.from_numpy(v.view(np.int16)).to(dev).view(torch.float16)
    tow = lambda v: torch.from_numpy(v.view(np.int32)).to(dev)
    dargs = (to16(a), tow(B1), to16(mid), tow(B2), to16(b))
    ws = ops.measure_workspace(m, n)
    E = torch.empty((m, n), dtype=torch.float32, device=dev)
    v0 = torch.from_numpy(synth.start_vector(n)).to(dev)
    flush = torch.empty(int(512 * 2 ** 20), dtype=torch.uint8, device=dev)

    st = torch.cuda.Stream()

    def timed(fn):
        # one call captured as a CUDA graph, so host time does not enter the
        # events; L2 flushed before each replay
        with torch.cuda.stream(st):
            fn()
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            fn()
        ts = []
        for _ in range(iters):
            with torch.cuda.stream(st):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(st)
                g.replay()
                e1.record(st)
            st.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    res_ms = timed(lambda: ops.w1_residual(Wd, signs, scales, want_E=False, workspace=ws))
    res_bytes = m * n * 4 + packed_bytes(m, n)
    dws = torch.empty(ops.dbf_residual_workspace_size(m, r, n), dtype=torch.uint8, device=dev)
    dbf_ms = timed(lambda: ops.dbf_residual(Wd, *dargs, want_E=False, workspace=dws))
    dbf_tf = 2.0 * m * n * r / (dbf_ms * 1e-3) / 1e12
    pi_ms = timed(lambda: ops.w1_power_iteration(Wd, v0, 32, workspace=ws))
    # least-squares refit of the DBF middle diagonal against W (fp64 Grams,
    # right-hand side and conjugate-gradient solve): 2 x m r^2 / 2 (symmetric
    # Grams) + m n r multiply-adds
    rws = torch.empty(ops.dbf_reproject_workspace_size(m, r, n), dtype=torch.uint8, device=dev)
    rp_out = {}

    def reproject():
        rp_out["r"] = ops.dbf_reproject_mid(Wd, dargs[0], dargs[1], dargs[3], dargs[4], workspace=rws)

    reproject()  # eager: one cooperative launch among a few plain ones, ~10 ms
    st.synchronize()
    rts = []
    for _ in range(3):
        with torch.cuda.stream(st):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            reproject()
            e1.record(st)
        st.synchronize()
        rts.append(e0.elapsed_time(e1))
    rp_ms = statistics.median(rts)
    rp_info = rp_out["r"][2].cpu().tolist()
    rp_fma = m * r * r + m * n * r
    ops.w1_residual(Wd, signs, scales, E=E, workspace=ws)
    _, sums = ops.w1_residual(Wd, signs, scales, want_E=False, workspace=ws)
    se, sw = (float(v) for v in sums.cpu())
    rel_spec = float(ops.w1_power_iteration(E, v0, 32, workspace=ws)) / float(ops.w1_power_iteration(Wd, v0, 32, workspace=ws))
    torch.cuda.synchronize()
    return {"residual_g128": {"ms": round(res_ms, 4), "GB/s": round(res_bytes / (res_ms * 1e-3) / 1e9, 1),
                              "frac_hbm": round(res_bytes / (res_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
            "dbf_residual": {"ms": round(dbf_ms, 4), "TFLOP/s": round(dbf_tf, 1),
                             "note": "2 m n r on the tensor cores (fp16 x +-1 products, fp32 accumulation)",
                             "frac_bf16_burst": round(dbf_tf / peaks["bf16_tflops"], 4)},
            "power_iteration_32": {"ms": round(pi_ms, 4), "launches": 3 * 32 + 3},
            "reproject_mid": {"ms": round(rp_ms, 4), "cg_iterations": rp_info[0], "converged": rp_info[1],
                              "fp64_fma": rp_fma, "fp64_TFLOP/s": round(2.0 * rp_fma / (rp_ms * 1e-3) / 1e12, 2)},
            "g128_gaussian_4096": {"rel_frobenius": round((se / sw) ** 0.5, 5), "rel_spectral": round(rel_spec, 5)}}


def cpu_oracle_sweep(max_pack_rows: int | None = None):
    """The fp64 oracle on the whole decode GEMV sweep on the host cores: each
    shape's weights packed by the oracle (pack_ref_fast), then one product per
    (shape, batch) pair, every pair at full size.  Phases timed separately:
    pack, dequantise (dequant_ref) and the whole product call (matmul_ref, which
    dequantises again, multiplies and forms the tolerance scale).  Returns the
    packed bytes processed, the per-phase seconds and the per-pair rows."""
    from oracle import w1_oracle as O
    from pack_sign_g128_b200 import synth
    rows = []
    t_pack = t_deq = t_prod = 0.0
    nbytes = 0
    for (N, K) in GEMV_SHAPES:
        W, _ = synth.gemv_case(N, K, 1)
        if max_pack_rows is not None:
            W = W[:max_pack_rows]
        n_rows = W.shape[0]
        t0 = time.perf_counter()
        s, c = O.pack_ref_fast(W)
        tp = time.perf_counter() - t0
        t_pack += tp
        for B in GEMV_BATCHES:
            x = O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(100 + B), B, K))
            t0 = time.perf_counter()
            O.dequant_ref(s, c, K)
            td = time.perf_counter() - t0
            t0 = time.perf_counter()
            O.matmul_ref(x, s, c, K)
            tm = time.perf_counter() - t0
            t_deq += td
            t_prod += tm
            nbytes += packed_bytes(n_rows, K)
            rows.append({"N": n_rows, "K": K, "B": B, "dequant_s": round(td, 4), "matmul_ref_s": round(tm, 4),
                         "GB/s": round(packed_bytes(n_rows, K) / tm / 1e9, 5)})
    return nbytes, {"pack_s": round(t_pack, 3), "dequant_s": round(t_deq, 3), "matmul_ref_s": round(t_prod, 3)}, rows


def cpu_oracle_rows(budget_s: float = 40.0):
    """The oracle on the other configurations, full size, in order, until the
    time budget is spent (rows not reached are listed as skipped): prefill
    GEMM per shape (dequantise + fp64 BLAS product + tolerance scale), the
    routed MoE layer, the DBF chain 4096^3 at B = 512."""
    from oracle import w1_oracle as O
    from pack_sign_g128_b200 import synth
    out = {"gemm": [], "moe": None, "dbf": None, "skipped": []}
    spent = 0.0
    for (N, K) in GEMM_SHAPES:
        if spent > budget_s:
            out["skipped"].append(f"gemm {N}x{K}")
            continue
        W, x = synth.gemm_case(GEMM_M, N, K)
        s, c = O.pack_ref_fast(W)
        del W
        xf = O.bf16_bits_to_f64(x)
        t0 = time.perf_counter()
        O.matmul_ref(xf, s, c, K)
        t = time.perf_counter() - t0
        spent += t
        out["gemm"].append({"M": GEMM_M, "N": N, "K": K, "matmul_ref_s": round(t, 3),
                            "TFLOP/s": round(2.0 * GEMM_M * N * K / t / 1e12, 5)})
    if spent <= budget_s:
        T, H, I, E, k = MOE["T"], MOE["H"], MOE["I"], MOE["E"], MOE["top_k"]
        x, logits, gate, up, down = synth.moe_case(T=T, H=H, I=I, E=E)
        pk = []
        for Wt in (gate, up, down):
            s_, c_ = O.pack_ref_fast(Wt.reshape(-1, Wt.shape[-1]))
            pk.append((s_.reshape(E, Wt.shape[1], -1), c_.reshape(E, Wt.shape[1], -1)))
        t0 = time.perf_counter()
        O.moe_ref(O.bf16_bits_to_f64(x), logits, pk[0], pk[1], pk[2], H, I, E, k)
        t = time.perf_counter() - t0
        spent += t
        out["moe"] = {"T": T, "s": round(t, 3), "tokens/s": round(T / t, 2)}
    else:
        out["skipped"].append("moe")
    if spent <= budget_s:
        a, B1, mid, B2, b, x = synth.dbf_case(m=4096, r=4096, n=4096, B=512)
        t0 = time.perf_counter()
        O.dbf_ref(a, B1, mid, B2, b, O.bf16_bits_to_f64(x), 4096, 4096, 4096)
        t = time.perf_counter() - t0
        spent += t
        out["dbf"] = {"B": 512, "s": round(t, 3), "TFLOP/s": round(2.0 * 512 * 2 * 4096 ** 2 / t / 1e12, 5)}
    else:
        out["skipped"].append("dbf B=512")
    return out


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _pci_bus_id(torch, dev):
    """NVML-style PCI bus id string of a torch CUDA device."""
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


def pin_gemv_choices(ops, path: str):
    """Pin each sweep pair's kernel to the choice a previous bench line recorded
    (its rows.gemv[*].choice), so that a profiled run launches the same kernels
    as the plain run whose numbers it explains."""
    with open(path) as f:
        line = [ln for ln in f.read().splitlines() if ln.strip().startswith("{")][-1]
    for r in json.loads(line)["rows"]["gemv"]:
        if r.get("choice"):
            ops.gemv_set_choice(r["N"], r["K"], r["B"], r["choice"])


def run_gpu(args):
    import torch
    from pack_sign_g128_b200 import ops, synth

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    peaks, peaks_kind = load_peaks()
    props = torch.cuda.get_device_properties(local)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20)

    if args.choices:
        pin_gemv_choices(ops, args.choices)
    if args.section != "all":
        rows = {}
        if args.section == "gemm":
            rows["gemm"] = gemm_rows(torch, ops, synth, peaks)
        elif args.section == "moe":
            rows["moe"] = moe_rows(torch, ops, synth, peaks, only_t=args.moe_t)
        elif args.section == "dbf":
            rows["dbf"] = dbf_rows(torch, ops, synth, peaks, l2, only_b=args.dbf_b)
        elif args.section == "gemv1":
            rows["gemv1"] = gemv_one(torch, ops, synth, args.shape)
        elif args.section == "measure":
            rows["measure"] = measure_rows(torch, ops, synth, peaks)
        elif args.section == "okt":
            combos, stream = build_gemv_sweep(torch, ops, synth, l2)
            rows["okt"] = okt_rows(torch, ops, synth, combos, stream)
        if rank == 0:
            print(json.dumps({"section": args.section, "rows": rows}), flush=True)
        return
    combos, stream = build_gemv_sweep(torch, ops, synth, l2, eager=args.eager)
    launches_per_step = sum(cb["R"] for cb in combos)
    bytes_per_step = sum(cb["bytes"] * cb["R"] for cb in combos)

    with ClockSampler(_pci_bus_id(torch, local)) as clk:
        total_ms, per_pair_ms = time_gemv_steps_detailed(torch, combos, stream, args.steps, args.warmup, world)
    t_max = max_over_ranks(world, total_ms)
    all_bytes = sum_over_ranks(world, float(bytes_per_step * args.steps))
    value = all_bytes / (t_max * 1e-3) / 1e9

    static_us = time_gemv_static(torch, combos, stream)
    floor_us = time_gemv_floor(torch, ops, combos, stream)
    gemv_rows = []
    for cb, ms, st_us, fl in zip(combos, per_pair_ms, static_us, floor_us):
        per_launch_us = ms * 1e3 / (cb["R"] * args.steps)
        gbs = cb["bytes"] / (per_launch_us * 1e-6) / 1e9
        gemv_rows.append({"N": cb["N"], "K": cb["K"], "B": cb["B"], "launches": cb["R"],
                          "choice": ops.gemv_choice(cb["N"], cb["K"], cb["B"]),
                          "kernel": KERNEL_OF_CHOICE.get(ops.gemv_choice(cb["N"], cb["K"], cb["B"]).split("/")[0], "?"),
                          "us_per_launch": round(per_launch_us, 3), "GB/s": round(gbs, 1),
                          "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                          "static_weights_us_per_launch": round(st_us, 3),
                          "static_weights_GB/s": round(cb["bytes"] / (st_us * 1e-6) / 1e9, 1),
                          # the launch floor (w1_stream_probe over the same bytes, same launch form)
                          "floor_us": round(fl["plain"], 3), "x_floor": round(per_launch_us / fl["plain"], 2),
                          "floor_static_us": round(fl["static"], 3),
                          "x_floor_static": round(st_us / fl["static"], 2)})
    # roofline of the dominant kernel (largest share of the step's device time)
    per_kernel = {}
    for cb, ms, row in zip(combos, per_pair_ms, gemv_rows):
        k = per_kernel.setdefault(row["kernel"], {"ms": 0.0, "bytes": 0.0, "launches": 0})
        k["ms"] += ms
        k["bytes"] += cb["bytes"] * cb["R"] * args.steps
        k["launches"] += cb["R"] * args.steps
    dom = max(per_kernel, key=lambda k: per_kernel[k]["ms"])
    dk = per_kernel[dom]
    achieved = dk["bytes"] / (dk["ms"] * 1e-3) / 1e9
    # DRAM traffic per launch: each pair's own capture (none scaled from another
    # pair); the line's figure is the launch-weighted mean over the pairs whose
    # first-call choice has a capture, with the share of launches it covers
    cap_bytes = 0.0
    cap_launches = 0
    for cb, row in zip(combos, gemv_rows):
        if row["kernel"] != dom:
            continue
        t = CAPTURED_TRAFFIC.get((cb["N"], cb["K"], cb["B"], row["choice"]))
        row["traffic_bytes_per_launch"] = t
        if t is not None:
            cap_bytes += t * cb["R"] * args.steps
            cap_launches += cb["R"] * args.steps
    traffic = round(cap_bytes / cap_launches) if cap_launches else None
    cap_alg = sum(cb["bytes"] * cb["R"] * args.steps for cb, row in zip(combos, gemv_rows)
                  if row["kernel"] == dom and row.get("traffic_bytes_per_launch") is not None)
    traffic_vs_alg = round(cap_bytes / cap_alg, 4) if cap_alg else None
    dom_share = dk["ms"] / sum(per_pair_ms)

    e2e = gemv_e2e(torch, ops, combos, max(1, min(args.steps, 3)))
    rows = {"gemv": gemv_rows}
    if not args.skip_extra:
        rows["gemm"] = gemm_rows(torch, ops, synth, peaks)
        rows["moe"] = moe_rows(torch, ops, synth, peaks)
        rows["dbf"] = dbf_rows(torch, ops, synth, peaks, l2)
        rows["okt"] = okt_rows(torch, ops, synth, combos, stream)
        rows["measure"] = measure_rows(torch, ops, synth, peaks)
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        nb, phases, cpu_pairs = cpu_oracle_sweep()
        secs = phases["matmul_ref_s"]
        cpu = {"value": nb / secs / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "sample": "fp64 numpy oracle on the whole sweep: every (shape, batch) pair once at full size "
                         "(weights packed by the oracle, pack time reported apart); value = packed bytes / "
                         "seconds of matmul_ref (dequantise + fp64 BLAS product + tolerance scale)",
               "phases": phases, "pairs": cpu_pairs}
        if not args.skip_extra:
            rows["cpu"] = cpu_oracle_rows()

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "s8 x s8 -> s32 (B <= 2) or bf16 x +-1 bf16 -> f32 (B >= 3) mma.sync, kernel chosen per shape by timing, + f32 scale fold; x bf16, 1-bit weights, fp16 scales",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "launches_per_step": launches_per_step,
                   "packed_bytes_per_step": bytes_per_step,
                   "l2": "inputs larger than L2: each pair cycles R weight copies totalling > 4x L2",
                   "timing": ("eager launches (profiling form)" if args.eager else
                              "CUDA graphs of back-to-back launches") + ", CUDA events on the launch stream",
                   "parallelism": f"replicas x{world} (independent sweeps, no collective)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "kernel": dom, "time_share": round(dom_share, 4),
                     "algorithmic_bytes_per_launch": round(dk["bytes"] / dk["launches"]),
                     "traffic_note": ("launch-weighted mean of each pair's own ncu capture (DRAM read + write "
                                      "bytes of one launch) over the pairs whose kernel choice was captured; "
                                      "per-pair figures in rows.gemv[*].traffic_bytes_per_launch"),
                     "traffic_launch_coverage": round(cap_launches / dk["launches"], 4),
                     "traffic_vs_algorithmic": traffic_vs_alg,
                     "peak_kind": peaks_kind},
        "cpu_baseline": cpu,
        "e2e": {k: e2e[k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step")},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "rows": rows,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The CPU oracle as the reference arm (rank 0 only under torchrun)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import w1_oracle as O
    from pack_sign_g128_b200 import synth
    # each step: the whole sweep, every (shape, batch) pair once at full size;
    # the oracle packs each shape's weights once, before the timed steps
    packed = {}
    for (N, K) in GEMV_SHAPES:
        W, _ = synth.gemv_case(N, K, 1)
        packed[(N, K)] = O.pack_ref_fast(W)
        del W
    spec = [(N, K, B) for (N, K) in GEMV_SHAPES for B in GEMV_BATCHES]
    xs = {(K, B): O.bf16_bits_to_f64(synth.activations_bf16(synth.rng(100 + B), B, K)) for (_, K, B) in spec}

    def one_step():
        t = 0.0
        nbytes = 0
        for (N, K, B) in spec:
            s, c = packed[(N, K)]
            t0 = time.perf_counter()
            O.matmul_ref(xs[(K, B)], s, c, K)
            t += time.perf_counter() - t0
            nbytes += packed_bytes(N, K)
        return nbytes, t

    for _ in range(args.warmup):
        one_step()
    nb = 0
    secs = 0.0
    for _ in range(args.steps):
        b, t = one_step()
        nb += b
        secs += t
    value = nb / secs / 1e9
    sample = ("fp64 numpy oracle (matmul_ref: dequantise + BLAS product + tolerance scale), every sweep pair "
              "once per step at full size; weights packed by the oracle before the timed steps")
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(secs * 1e3 / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="w1", choices=["w1", "reference"])
    ap.add_argument("--skip-extra", action="store_true", help="only the headline sweep")
    ap.add_argument("--skip-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--eager", action="store_true",
                    help="issue the sweep's launches one by one instead of CUDA graphs (for ncu launch lists)")
    ap.add_argument("--shape", default="4096,4096,1",
                    help="N,K,B of the single GEMV that --section gemv1 launches (for ncu captures)")
    ap.add_argument("--dbf-b", type=int, default=None, help="--section dbf: that batch only (profiling)")
    ap.add_argument("--moe-t", type=int, default=None, help="--section moe: that decode batch only (profiling)")
    ap.add_argument("--choices", default=None,
                    help="JSON line of an earlier run: pin each GEMV pair to the kernel it chose (profiling)")
    ap.add_argument("--section", default="all", choices=["all", "gemm", "moe", "dbf", "gemv1", "okt", "measure"],
                    help="run one row only (for profiling); prints a rows-only JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
