#!/usr/bin/env python
"""Benchmark of the quantized-KV attention hot path on B200.

One step = one decode call (qsdpa_decode) of the workload named by --workload
(default: B=1, Hq=32, Hkv=8, D=128, L=65536, affine 4-bit groups of 64,
uniform fp16 inputs, scale 1.0 -- the MLX quantized-SDPA benchmark shape).
The primary number is HBM throughput in GB/s of ALGORITHMIC bytes (packed K/V
codes, scales, biases, q and out) per call; microseconds per call are reported
beside it.  Inputs are synthetic (seeded SplitMix64), quantized on the GPU by
qkv_quantize_update; the timed calls rotate over enough cache copies that the
data read in one call is no longer in the 126 MB L2 when it is read again.

The line's `rows` object times the other rows of the path the same way
(--no-rows leaves them out): bulk and one-token quantize, the 8-bit decode
and the fused update + decode, the Q8_0 D=256 decodes, the 512-query prefill,
the materialize-then-library-attention A/B rows, the attention extensions
(softcap, sinks, ALiBi) on decode and prefill, and the llama.cpp block
conversions.

--impl reference runs the CPU oracle (the only reference this repository has)
on a bounded sample of the same workload and reports the same metric.

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run, one process per GPU (independent replicas: the path
has no cross-GPU exchange), rank 0 prints one JSON line.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "quant-KV decode attention µs/call and HBM GB/s (% of peak) at L=64K, 1 B200"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.lines = []
        self.proc = None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        inside = []
        for t, line in self.lines:
            if any(a <= t <= b for a, b in self.windows):
                inside.append(line)
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in inside:
            parts = [p.strip() for p in line.split(",")]
            try:
                sm.append(float(parts[2]))
                smax.append(float(parts[3]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def dev16(bits, dtype, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16).to(device)


def build_caches(w, inp, ncopies, device):
    """Quantize the workload's K/V on the GPU into `ncopies` cache copies."""
    import torch
    from quantized_kv_attention_split_b200 import qkv
    fmt = qkv.Q8_0 if w.fmt == "q8_0" else qkv.AFFINE
    kd_src = dev16(inp.k, w.kv_dtype, device)
    vd_src = dev16(inp.v, w.kv_dtype, device)
    caches = []
    for _ in range(ncopies):
        kc = qkv.QuantCache.empty(w.B, w.Hkv, w.Lcap, w.D, fmt, w.bits, w.gs, device)
        vc = qkv.QuantCache.empty(w.B, w.Hkv, w.Lcap, w.D, fmt, w.bits, w.gs, device)
        qkv.qkv_quantize_update(kd_src, vd_src, kc, vc, 0)
        caches.append((kc, vc))
    del kd_src, vd_src
    torch.cuda.synchronize()
    return caches


def graph_kernel_nodes(g):
    """Kernel nodes of a captured CUDA graph (None if it cannot be read)."""
    try:
        from cuda.bindings import runtime as rt
        h = g.raw_cuda_graph()
        graph = h if isinstance(h, rt.cudaGraph_t) else rt.cudaGraph_t(init_value=int(h))
        err, _, n = rt.cudaGraphGetNodes(graph, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kern = 0
        for nd in nodes[:n]:
            err, t = rt.cudaGraphNodeGetType(nd)
            if err == rt.cudaError_t.cudaSuccess and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


LAUNCHES = {}


def new_graph():
    """A CUDA graph whose captured graph stays readable (for counting launches)."""
    import torch
    try:
        return torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        return torch.cuda.CUDAGraph()


def graph_time(step, K, W, sampler=None, min_window_s=0.3, tag=None, sync_ranks=False):
    """Device time of exactly K calls of step(i): W eager warm-up calls, then
    K calls captured in CUDA graphs and replayed between events.  With a tag,
    the kernel launches of the K calls (counted from the captured graphs) are
    recorded in LAUNCHES[tag].  sync_ranks: a barrier over all ranks right
    before the timed region (only for calls that every rank makes; the
    secondary rows run on rank 0 alone)."""
    import torch
    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    chunk = min(K, 256)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graphs = []
    with torch.cuda.stream(s):
        g1 = new_graph()
        with torch.cuda.graph(g1, stream=s):
            for i in range(chunk):
                step(i)
        graphs.append(g1)
        rem = K % chunk
        g2 = None
        if rem:
            g2 = new_graph()
            with torch.cuda.graph(g2, stream=s):
                for i in range(rem):
                    step(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    if tag is not None:
        n1 = graph_kernel_nodes(g1)
        n2 = graph_kernel_nodes(g2) if g2 is not None else 0
        LAUNCHES[tag] = None if n1 is None or n2 is None else n1 * (K // chunk) + n2
    for g in (g1, g2):
        if g is not None and hasattr(g, "instantiate"):
            try:
                g.instantiate()
            except RuntimeError:
                pass                              # already instantiated
    g1.replay()                                   # one untimed replay
    torch.cuda.synchronize()
    reps = K // chunk
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sync_ranks and torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record()
    for _ in range(reps):
        g1.replay()
    if g2 is not None:
        g2.replay()
    end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    ms = start.elapsed_time(end)
    extra = False
    if sampler is not None:
        sampler.mark(t0, t1)
        if t1 - t0 < min_window_s:
            # too short for the 50 ms clock sampler: replay the same graph
            # (untimed) for a while and sample the clocks there as well
            extra = True
            n = max(1, int(min_window_s / max(1e-6, ms / 1e3 / max(1, reps))))
            t2 = time.time()
            for _ in range(n):
                g1.replay()
            torch.cuda.synchronize()
            sampler.mark(t2, time.time())
    del graphs
    return ms / K, extra


def isolated_time(step, n=20, flush_bytes=512 << 20):
    """Median device time of single calls that overlap nothing: before each
    call the L2 is flushed by reading flush_bytes (more than the 126 MB L2;
    a read leaves clean lines, so the call pays no write-backs) and the
    stream drains, so the call neither starts early nor finds its data in
    L2; events bracket the call alone."""
    import torch
    buf = torch.ones(flush_bytes // 8, dtype=torch.int64, device="cuda")
    times = []
    for i in range(n + 2):
        buf.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step(i)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1) / 1e3)
    del buf
    return statistics.median(times)


def oracle_rows_time(w, host_k, host_v, q_bits, nrows_target_s=15.0, max_rows=None):
    """Time the CPU oracle on a sample of query rows of the workload."""
    import oracle
    total_rows = w.B * w.Hq * w.Lq
    t0 = time.time()
    oracle.attention(q_bits, w.q_dtype, host_k, host_v, w.L, w.scale,
                     mask=oracle.Mask("causal") if w.mask == "causal" else None,
                     rows=np.array([0]), nthreads=1)
    t_row = max(1e-4, time.time() - t0)
    threads = oracle.default_threads()
    nrows = int(min(total_rows, max(threads, nrows_target_s * threads / t_row)))
    if max_rows:
        nrows = min(nrows, max_rows)
    rows = np.linspace(0, total_rows - 1, nrows).astype(np.int64)
    t0 = time.time()
    out = oracle.attention(q_bits, w.q_dtype, host_k, host_v, w.L, w.scale,
                           mask=oracle.Mask("causal") if w.mask == "causal" else None,
                           rows=rows, nthreads=threads)
    dt = time.time() - t0
    return dt, nrows, total_rows, threads, rows, out


def host_cache(dc, fmt):
    import oracle
    codes = dc.codes.cpu().numpy().view(np.uint32)
    scales = dc.scales.cpu().numpy().view(np.uint16)
    biases = None if dc.biases is None else dc.biases.cpu().numpy().view(np.uint16)
    return oracle.QCache(fmt, dc.bits, dc.group_size, codes, scales, biases)


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------
def max_over_ranks(x: float, device, world: int) -> float:
    """Max of a per-rank value over all ranks (times: the slowest replica sets
    the job's time).  NCCL on the GPU ranks; any backend works on its device."""
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_rate(units_per_rank: float, max_sec: float, world: int) -> float:
    """Whole-job throughput of `world` independent replicas that each process
    `units_per_rank` units: all units over the slowest rank's time."""
    return units_per_rank * world / max_sec


def run_ours(args, rank, world, device):
    import torch
    from quantized_kv_attention_split_b200 import qkv, synthetic as S

    qkv.lib()
    w = S.WORKLOADS[args.workload]
    hbm_peak, _, peak_kind = peaks()
    inp = S.make_inputs(w)
    cache_bytes = w.cache_bytes()
    io_bytes = 2 * w.B * w.Hq * w.Lq * w.D * 2
    alg_bytes = cache_bytes + io_bytes
    ncopies = max(2, math.ceil(3 * 126e6 / cache_bytes))
    caches = build_caches(w, inp, ncopies, device)
    qd = dev16(inp.q, w.q_dtype, device)
    out = torch.empty(w.B, w.Hq, w.Lq, w.D, dtype=torch.float16, device=device)
    ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, w.Lq, w.D, w.L, device)

    # correctness gate on sampled rows before timing anything
    qkv.qsdpa_decode(qd, caches[0][0], caches[0][1], w.L, w.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    hk, hv = host_cache(caches[0][0], w.fmt), host_cache(caches[0][1], w.fmt)
    if rank == 0:
        import oracle
        rows = np.array([0, w.Hq // 2, w.Hq - 1])
        ref = oracle.attention(inp.q, w.q_dtype, hk, hv, w.L, w.scale, rows=rows)
        got = out.float().cpu().numpy().reshape(-1, w.D)
        err = float(np.abs(got[rows] - ref.reshape(-1, w.D)[rows]).max())
        if not err <= 2e-3:
            print(json.dumps({"error": f"decode output differs from the oracle: {err}"}))
            sys.exit(1)

    def step(i):
        kc, vc = caches[i % ncopies]
        qkv.qsdpa_decode(qd, kc, vc, w.L, w.scale, out=out, workspace=ws)

    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    sec, extra = graph_time(step, args.steps, args.warmup, sampler, tag="main", sync_ranks=True)
    sec /= 1e3
    if sampler:
        time.sleep(0.1)
        sampler.stop()

    sec = max_over_ranks(sec, device, world)
    gbs = alg_bytes / sec / 1e9
    # one call alone (cold L2, no overlap with a previous call)
    iso_sec = max_over_ranks(isolated_time(step), device, world)

    # e2e through the public API with host buffers: q in pinned host memory,
    # the output back in pinned host memory.  The library takes such buffers
    # directly (its kernels read q and write out over the host link), so a
    # step is one call; the variant with explicit copies (H2D of q into a
    # device buffer, decode, D2H of the output) is timed beside it.
    q_host = torch.from_numpy(inp.q.view(np.int16)).view(torch.float16).pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    qe = torch.empty_like(qd)
    ke = max(20, min(args.steps, 2000))

    def e2e_step(i):
        kc, vc = caches[i % ncopies]
        qkv.qsdpa_decode(q_host, kc, vc, w.L, w.scale, out=out_host, workspace=ws)

    def copy_step(i):
        qe.copy_(q_host, non_blocking=True)
        kc, vc = caches[i % ncopies]
        qkv.qsdpa_decode(qe, kc, vc, w.L, w.scale, out=out, workspace=ws)
        out_host.copy_(out, non_blocking=True)

    for i in range(5):
        e2e_step(i)
        copy_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record()
    for i in range(ke):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    eager_sec = max_over_ranks(e0.elapsed_time(e1) / 1e3 / ke, device, world)
    # the same steps recorded once in a CUDA graph and replayed (what a serving
    # loop does to take the host's per-call cost out)
    e2e_ms, _ = graph_time(e2e_step, ke, 5, sync_ranks=True)
    e2e_sec = max_over_ranks(e2e_ms / 1e3, device, world)
    copy_ms, _ = graph_time(copy_step, ke, 5, sync_ranks=True)
    copy_sec = max_over_ranks(copy_ms / 1e3, device, world)
    # the host buffers hold the same result as the device-buffer call
    ref_out = out.clone()
    qkv.qsdpa_decode(qd, caches[0][0], caches[0][1], w.L, w.scale, out=ref_out, workspace=ws)
    e2e_step(0)
    torch.cuda.synchronize()
    e2e_diff = (out_host.float() - ref_out.float().cpu()).abs().max().item()
    if not e2e_diff <= 2e-3:
        raise SystemExit(f"e2e: host-buffer result differs from the device-buffer call by {e2e_diff}")

    result = None
    if rank == 0:
        clocks = sampler.summary() if sampler else {}
        # CPU baseline: the oracle on the host cores, bounded sample of rows
        dt, nrows, total_rows, threads, _, _ = oracle_rows_time(w, hk, hv, inp.q, 12.0)
        cpu_gbs = (nrows / total_rows) * alg_bytes / dt / 1e9
        result = {
            "metric": METRIC,
            "value": round(replica_rate(alg_bytes, sec, world) / 1e9, 2),
            "unit": "GB/s",
            "us_per_call": round(sec * 1e6, 3),
            "us_per_call_isolated": round(iso_sec * 1e6, 3),
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "data": "synthetic (seeded SplitMix64, uniform fp16 q/k/v, K/V quantized on the GPU)",
            "config": workload_config(w, world),
            "l2": f"inputs larger than L2: {ncopies} rotating cache copies "
                  f"({ncopies * cache_bytes / 1e6:.0f} MB)",
            "timing": "CUDA events around CUDA-graph replays of exactly K back-to-back calls "
                      "(a call's set-up overlaps the previous kernel's tail); "
                      "us_per_call_isolated: median of single calls after an L2 flush",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(gbs / hbm_peak, 4),
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "traffic": read_traffic(w.name)},
            "cpu_baseline": {"value": round(cpu_gbs, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"{nrows} of {total_rows} query rows over all {w.L} keys "
                                       f"(fp64 dequantize + attention), scaled to the workload"},
            "e2e": {"value": round(replica_rate(alg_bytes, e2e_sec, world) / 1e9, 2), "unit": "GB/s",
                    "us_per_call": round(e2e_sec * 1e6, 3),
                    "eager_us_per_call": round(eager_sec * 1e6, 3),
                    "copy_engine_us_per_call": round(copy_sec * 1e6, 3),
                    "h2d_bytes_per_step": int(qd.numel() * 2),
                    "d2h_bytes_per_step": int(out.numel() * 2),
                    "note": "each step: qsdpa_decode through the Python binding and C ABI with q "
                            "in pinned host memory and the output written to pinned host memory "
                            "(the kernels move both over the host link); the steps recorded in "
                            "CUDA graphs and replayed (device time of exactly K steps); "
                            "eager_us_per_call: the same steps issued one by one from Python "
                            "(host-bound); copy_engine_us_per_call: explicit cudaMemcpyAsync of q "
                            "in and of the output out around a call on device buffers, replayed "
                            "the same way"},
            "gpu_launches": LAUNCHES.get("main") if LAUNCHES.get("main") is not None else args.steps,
            "gpu_launches_source": ("kernel nodes of the captured CUDA graphs (decode kernel, plus "
                                    "the merge kernel when a unit is split over CTAs)"
                                    if LAUNCHES.get("main") is not None else "one per call (graph not readable)"),
            "clocks": {"sm_mhz": clocks.get("sm_mhz"), "sm_max_mhz": clocks.get("sm_max_mhz"),
                       "reasons": clocks.get("reasons", []), "samples": clocks.get("samples", 0),
                       "window": "timed region" + (" + untimed replay of the same graph"
                                                   if extra else "")},
        }
        if args.rows:
            result["rows"] = other_rows(device)
    del caches
    return result


def workload_config(w, world):
    """The `config` object of both arms: the workload and its sizes."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.L,
            "Lq": w.Lq, "format": w.fmt, "bits": w.bits, "group_size": w.gs, "scale": w.scale,
            "out_dtype": w.out_dtype,
            "algorithmic_bytes_per_call": w.cache_bytes() + 2 * w.B * w.Hq * w.Lq * w.D * 2,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def read_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel, if
    it was taken on the current kernel source (else null)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"decode_{workload}_traffic.txt")
    if not os.path.exists(path):
        return None
    src = os.path.join(ROOT, "quantized_kv_attention_split_b200", "csrc", "decode_kernel.cuh")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != h:
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def other_rows(device):
    """Secondary rows of the hot path, each timed the same way (device time,
    rotating copies where the data would fit in L2)."""
    import torch
    from quantized_kv_attention_split_b200 import qkv, synthetic as S
    hbm_peak, _, _ = peaks()
    rows = {}

    # bulk quantize-and-append: 65536 tokens x 8 heads of K and V, 8-bit affine
    w = S.WORKLOADS["decode_64k_affine8_update"]
    inp = S.make_inputs(w, L=w.Lcap)
    kd_src, vd_src = dev16(inp.k, "f16", device), dev16(inp.v, "f16", device)
    kc = qkv.QuantCache.empty(w.B, w.Hkv, w.Lcap, w.D, qkv.AFFINE, 8, 64, device)
    vc = qkv.QuantCache.empty(w.B, w.Hkv, w.Lcap, w.D, qkv.AFFINE, 8, 64, device)
    sec, _ = graph_time(lambda i: qkv.qkv_quantize_update(kd_src, vd_src, kc, vc, 0), 50, 5)
    nb = 2 * kd_src.numel() * 2 + w.cache_bytes(w.Lcap)
    rows["quantize_bulk_65536tok_affine8"] = {
        "us_per_call": round(sec * 1e3, 2), "GB/s": round(nb / (sec / 1e3) / 1e9, 1),
        "frac_hbm": round(nb / (sec / 1e3) / 1e9 / hbm_peak, 4), "bytes": nb}
    # single-token update at offset 65535, then the 8-bit decode over 65536 keys
    nk, nv = dev16(inp.k[:, :, :1].copy(), "f16", device), dev16(inp.v[:, :, :1].copy(), "f16", device)
    sec, _ = graph_time(lambda i: qkv.qkv_quantize_update(nk, nv, kc, vc, w.Lcap - 1), 200, 10)
    rows["update_1tok_affine8"] = {"us_per_call": round(sec * 1e3, 3)}
    del kd_src, vd_src
    ncopies = max(2, math.ceil(3 * 126e6 / w.cache_bytes()))
    copies = [(kc, vc)]
    for _ in range(ncopies - 1):
        k2 = qkv.QuantCache(kc.fmt, kc.bits, kc.group_size, kc.codes.clone(), kc.scales.clone(),
                            kc.biases.clone())
        v2 = qkv.QuantCache(vc.fmt, vc.bits, vc.group_size, vc.codes.clone(), vc.scales.clone(),
                            vc.biases.clone())
        copies.append((k2, v2))
    q = dev16(S.make_inputs(w).q, "f16", device)
    out = torch.empty(w.B, w.Hq, 1, w.D, dtype=torch.float16, device=device)
    ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, 1, w.D, w.L, device)

    def dstep(i):
        a, b = copies[i % ncopies]
        qkv.qsdpa_decode(q, a, b, w.L, w.scale, out=out, workspace=ws)
    sec, _ = graph_time(dstep, 400, 20)
    nb = w.cache_bytes() + 2 * w.Hq * w.D * 2
    rows["decode_64k_affine8"] = {"us_per_call": round(sec * 1e3, 3),
                                  "GB/s": round(nb / (sec / 1e3) / 1e9, 1),
                                  "frac_hbm": round(nb / (sec / 1e3) / 1e9 / hbm_peak, 4)}
    # the decode step with its cache update: the separate calls (update of the
    # token at row 65535, then decode over 65536 keys) and the fused call
    def sstep(i):
        a, b = copies[i % ncopies]
        qkv.qkv_quantize_update(nk, nv, a, b, w.Lcap - 1)
        qkv.qsdpa_decode(q, a, b, w.L, w.scale, out=out, workspace=ws)

    def fstep(i):
        a, b = copies[i % ncopies]
        qkv.qsdpa_decode_update(q, nk, nv, a, b, w.Lcap - 1, w.scale, out=out, workspace=ws)
    sec_s, _ = graph_time(sstep, 400, 20)
    sec_f, _ = graph_time(fstep, 400, 20)
    rows["update_decode_64k_affine8"] = {
        "separate_us_per_call": round(sec_s * 1e3, 3), "fused_us_per_call": round(sec_f * 1e3, 3),
        "fused_GB/s": round(nb / (sec_f / 1e3) / 1e9, 1),
        "fused_frac_hbm": round(nb / (sec_f / 1e3) / 1e9 / hbm_peak, 4),
        "note": "update of one token per kv head at row 65535 plus decode over 65536 keys: "
                "qkv_quantize_update + qsdpa_decode vs qsdpa_decode_update (one decode launch)"}
    del copies, kc, vc
    torch.cuda.empty_cache()

    for name in ("decode_q8_0_10k", "decode_q8_0_20k"):
        w = S.WORKLOADS[name]
        inp = S.make_inputs(w)
        ncopies = max(2, math.ceil(3 * 126e6 / w.cache_bytes()))
        caches = build_caches(w, inp, ncopies, device)
        q = dev16(inp.q, "f16", device)
        out = torch.empty(w.B, w.Hq, 1, w.D, dtype=torch.float16, device=device)
        ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, 1, w.D, w.L, device)

        def qstep(i, caches=caches, q=q, out=out, ws=ws, w=w, n=ncopies):
            a, b = caches[i % n]
            qkv.qsdpa_decode(q, a, b, w.L, w.scale, out=out, workspace=ws)
        sec, _ = graph_time(qstep, 400, 20)
        nb = w.cache_bytes() + 2 * w.Hq * w.D * 2
        rows[name] = {"us_per_call": round(sec * 1e3, 3), "GB/s": round(nb / (sec / 1e3) / 1e9, 1),
                      "frac_hbm": round(nb / (sec / 1e3) / 1e9 / hbm_peak, 4)}
        if name == "decode_q8_0_20k":
            # llama.cpp-style interleaved blocks <-> planes for this cache (K and V)
            a, b = caches[0]
            bk = qkv.qkv_q8_0_to_blocks(a, w.L)
            bv = qkv.qkv_q8_0_to_blocks(b, w.L)
            sec_f, _ = graph_time(lambda i: (qkv.qkv_q8_0_from_blocks(bk, a),
                                             qkv.qkv_q8_0_from_blocks(bv, b)), 200, 10)
            sec_t, _ = graph_time(lambda i: (qkv.qkv_q8_0_to_blocks(a, w.L, out=bk),
                                             qkv.qkv_q8_0_to_blocks(b, w.L, out=bv)), 200, 10)
            moved = 2 * (bk.numel() + w.cache_bytes() // 2)     # read one form, write the other
            rows["q8_0_blocks_20k"] = {
                "from_blocks_us": round(sec_f * 1e3, 3), "to_blocks_us": round(sec_t * 1e3, 3),
                "from_GB/s": round(moved / (sec_f / 1e3) / 1e9, 1),
                "to_GB/s": round(moved / (sec_t / 1e3) / 1e9, 1),
                "frac_hbm_from": round(moved / (sec_f / 1e3) / 1e9 / hbm_peak, 4),
                "note": "K and V of decode_q8_0_20k (2 x 11.1 MB of planes, 2 x 11.1 MB of "
                        "34-byte blocks): qkv_q8_0_from_blocks / qkv_q8_0_to_blocks; the data "
                        "fit in L2"}
            del bk, bv
        del caches
        torch.cuda.empty_cache()

    # prefill: 512 causal queries at depth 20480 over a Q8_0 cache (tcgen05 kernel)
    w = S.WORKLOADS["prefill_q8_0_512_at_20k"]
    inp = S.make_inputs(w)
    caches = build_caches(w, inp, 1, device)
    q = dev16(inp.q, w.q_dtype, device)
    out = torch.empty(w.B, w.Hq, w.Lq, w.D, dtype=torch.bfloat16, device=device)
    ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, w.Lq, w.D, w.L, device)
    kc, vc = caches[0]
    sec, _ = graph_time(lambda i: qkv.qsdpa_prefill(q, kc, vc, w.L, w.scale, causal=True, out=out,
                                                    workspace=ws), 20, 3)
    flop = prefill_flops(w)
    _, bf16_peak, _ = peaks()
    rows[w.name] = {"us_per_call": round(sec * 1e3, 2),
                    "TFLOP/s": round(flop / (sec / 1e3) / 1e12, 1),
                    "frac_tensor_peak": round(flop / (sec / 1e3) / 1e12 / bf16_peak, 4),
                    "flop": flop,
                    "peak_note": "fp16 operands; measured bf16 dense peak x nominal fp16:bf16 ratio 1"}
    # A/B: materialize the cache as fp16 (qkv_dequantize), then dense attention
    # through torch's scaled_dot_product_attention (a library kernel), against
    # the fused prefill above
    try:
        from torch.nn.attention.bias import causal_lower_right
        kd = torch.empty(w.B, w.Hkv, w.L, w.D, dtype=torch.float16, device=device)
        vd = torch.empty_like(kd)
        qh = q.to(torch.float16)
        cmask = causal_lower_right(w.Lq, w.L)

        def mstep(i):
            qkv.qkv_dequantize(kc, w.L, out=kd)
            qkv.qkv_dequantize(vc, w.L, out=vd)
            torch.nn.functional.scaled_dot_product_attention(qh, kd, vd, attn_mask=cmask,
                                                             scale=w.scale, enable_gqa=True)
        sec_m, _ = graph_time(mstep, 20, 3)
        sec_d, _ = graph_time(lambda i: (qkv.qkv_dequantize(kc, w.L, out=kd),
                                         qkv.qkv_dequantize(vc, w.L, out=vd)), 20, 3)
        rows["materialize_" + w.name] = {
            "us_per_call": round(sec_m * 1e3, 2), "dequantize_us": round(sec_d * 1e3, 2),
            "TFLOP/s": round(flop / (sec_m / 1e3) / 1e12, 1),
            "note": "qkv_dequantize of K and V to fp16, then torch scaled_dot_product_attention "
                    "(causal, lower-right aligned, GQA); compare prefill_q8_0_512_at_20k"}
        del kd, vd
    except Exception as e:                       # the library attention may be unavailable
        rows["materialize_" + w.name] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    del caches
    torch.cuda.empty_cache()

    # A/B for the main decode workload: materialize K and V (65536 keys), then
    # dense attention for the one query, against the fused decode (bench value)
    try:
        w = S.WORKLOADS["decode_64k_affine4"]
        inp = S.make_inputs(w)
        kc, vc = build_caches(w, inp, 1, device)[0]
        q = dev16(inp.q, "f16", device)
        kd = torch.empty(w.B, w.Hkv, w.L, w.D, dtype=torch.float16, device=device)
        vd = torch.empty_like(kd)

        def dstep2(i):
            qkv.qkv_dequantize(kc, w.L, out=kd)
            qkv.qkv_dequantize(vc, w.L, out=vd)
            torch.nn.functional.scaled_dot_product_attention(q, kd, vd, scale=w.scale,
                                                             enable_gqa=True)
        sec_m, _ = graph_time(dstep2, 200, 10)
        nb = w.cache_bytes() + 2 * w.Hq * w.D * 2
        rows["materialize_" + w.name] = {
            "us_per_call": round(sec_m * 1e3, 3), "GB/s": round(nb / (sec_m / 1e3) / 1e9, 1),
            "note": "qkv_dequantize of K and V to fp16 (268 MB written), then torch "
                    "scaled_dot_product_attention (GQA); compare the bench value"}
        del kd, vd, kc, vc
    except Exception as e:
        rows["materialize_decode_64k_affine4"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    torch.cuda.empty_cache()

    # llama.cpp Q4_0 blocks of the main decode shape (K and V, 65536 tokens,
    # token-major) into 4-bit affine caches with groups of 32
    try:
        w = S.WORKLOADS["decode_64k_affine4"]
        nbk = w.D // 32
        blk = torch.randint(0, 256, (w.B, w.L, w.Hkv * nbk * 18), dtype=torch.uint8, device=device)
        blk.view(w.B, w.L, w.Hkv, nbk, 18)[..., 1] = 0x2C        # finite fp16 scales
        st = (w.L * w.Hkv * nbk * 18, nbk * 18, w.Hkv * nbk * 18)
        dk = qkv.QuantCache.empty(w.B, w.Hkv, w.L, w.D, qkv.AFFINE, 4, 32, device)
        dv = qkv.QuantCache.empty(w.B, w.Hkv, w.L, w.D, qkv.AFFINE, 4, 32, device)
        sec, _ = graph_time(lambda i: (qkv.qkv_llama_blocks_to_cache("q4_0", blk, dk, L=w.L, strides=st),
                                       qkv.qkv_llama_blocks_to_cache("q4_0", blk, dv, L=w.L, strides=st)),
                            100, 5)
        moved = 2 * (blk.numel() + w.B * w.Hkv * w.L * nbk * 20)
        rows["llama_q4_0_blocks_64k"] = {
            "us_per_call": round(sec * 1e3, 3), "GB/s": round(moved / (sec / 1e3) / 1e9, 1),
            "frac_hbm": round(moved / (sec / 1e3) / 1e9 / hbm_peak, 4),
            "note": "qkv_llama_blocks_to_cache, Q4_0 blocks (token-major, 2 x 37.7 MB) into K "
                    "and V 4-bit affine caches with groups of 32 (2 x 41.9 MB)"}
        del blk, dk, dv
    except Exception as e:
        rows["llama_q4_0_blocks_64k"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    torch.cuda.empty_cache()

    # values as a view of the keys (MLA 576/512): one Q8_0 cache of 576-wide
    # K rows, 128 query heads over one KV head, 32768 keys, bf16 q and out
    try:
        B, Hq, L = 1, 128, 32768
        xk = torch.randn(B, 1, L, 576, device=device, dtype=torch.float16)
        per_cache = B * L * (576 + 36)
        ncopies = max(3, math.ceil(3 * 126e6 / per_cache))
        caches = []
        for _ in range(ncopies):
            kc = qkv.QuantCache.empty(B, 1, L, 576, qkv.Q8_0, 8, 32, device)
            qkv.qkv_quantize_update(xk, xk, kc, kc, 0)
            caches.append(kc)
        del xk
        qm = torch.randn(B, Hq, 1, 576, device=device, dtype=torch.bfloat16)
        om = torch.empty(B, Hq, 1, 512, device=device, dtype=torch.bfloat16)
        wsm = torch.zeros(qkv.lib().qsdpa_kview_workspace_size(B, Hq, 1, 1, 576, 512, L),
                          dtype=torch.uint8, device=device)
        sec, _ = graph_time(lambda i: qkv.qsdpa_attention_kview(qm, caches[i % ncopies], L,
                                                                576 ** -0.5, out=om, workspace=wsm),
                            400, 20)
        nb = per_cache + B * Hq * (576 + 512) * 2
        flops = 2 * B * Hq * L * (576 + 512)
        rows["kview_mla_q8_0_32k"] = {
            "us_per_call": round(sec * 1e3, 3), "GB/s": round(nb / (sec / 1e3) / 1e9, 1),
            "frac_hbm": round(nb / (sec / 1e3) / 1e9 / hbm_peak, 4),
            "TFLOP/s": round(flops / (sec / 1e3) / 1e12, 1), "bytes": nb,
            "note": "qsdpa_attention_kview: Q8_0 K rows of 576, V = their first 512, 128 query "
                    "heads over 1 KV head, L = 32768 (decode)"}
        del caches
    except Exception as e:
        rows["kview_mla_q8_0_32k"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    torch.cuda.empty_cache()

    # affine codes stored 2, 3, 5 and 6 bits wide: decode of the main shape
    # (L = 65536, 32 query heads over 8 KV heads, D = 128, groups of 64)
    try:
        w = S.WORKLOADS["decode_64k_affine4"]
        inp = S.make_inputs(w)
        kx, vx = dev16(inp.k, "f16", device), dev16(inp.v, "f16", device)
        q = dev16(inp.q, "f16", device)
        out = torch.empty(w.B, w.Hq, 1, w.D, dtype=torch.float16, device=device)
        ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, 1, w.D, w.L, device)
        for bits in (2, 3, 5, 6):
            per_cache = w.B * w.Hkv * w.L * (w.D * bits // 8 + 2 * 2 * (w.D // w.gs))
            ncopies = max(3, math.ceil(3 * 126e6 / (2 * per_cache)))
            caches = []
            for _ in range(ncopies):
                kc = qkv.QuantCache.empty(w.B, w.Hkv, w.L, w.D, qkv.AFFINE, bits, w.gs, device)
                vc = qkv.QuantCache.empty(w.B, w.Hkv, w.L, w.D, qkv.AFFINE, bits, w.gs, device)
                qkv.qkv_quantize_update(kx, vx, kc, vc, 0)
                caches.append((kc, vc))

            def xstep(i):
                a, b = caches[i % ncopies]
                qkv.qsdpa_decode(q, a, b, w.L, w.scale, out=out, workspace=ws)
            sec, _ = graph_time(xstep, 400, 20)
            nb = 2 * per_cache + 2 * w.Hq * w.D * 2
            rows[f"decode_64k_affine{bits}"] = {
                "us_per_call": round(sec * 1e3, 3), "GB/s": round(nb / (sec / 1e3) / 1e9, 1),
                "frac_hbm": round(nb / (sec / 1e3) / 1e9 / hbm_peak, 4), "bytes": nb,
                "note": f"{bits}-bit codes (one bit stream per row), transcoded per block to "
                        f"{4 if bits < 4 else 8}-bit codes by the decode kernel; caches written "
                        f"by qkv_quantize_update"}
            del caches
        del kx, vx
    except Exception as e:
        rows["decode_64k_affine3"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    torch.cuda.empty_cache()

    # llama.cpp's reference Q4_0 / Q5_1 quantizers on the GPU: 65536 tokens of
    # K and V (the main decode shape) into token-major blocks, and one new
    # token of every head written straight into the affine caches
    try:
        w = S.WORKLOADS["decode_64k_affine4"]
        nbk = w.D // 32
        inp = S.make_inputs(w)
        kx, vx = dev16(inp.k, "f16", device), dev16(inp.v, "f16", device)
        for kind, nbytes, bits in (("q4_0", 18, 4), ("q5_1", 24, 8)):
            ob = torch.empty(w.B, w.L, w.Hkv * nbk * nbytes, dtype=torch.uint8, device=device)
            st = (w.L * w.Hkv * nbk * nbytes, nbk * nbytes, w.Hkv * nbk * nbytes)
            sec, _ = graph_time(lambda i: (qkv.qkv_llama_quantize_blocks(kind, kx, out=ob, strides=st),
                                           qkv.qkv_llama_quantize_blocks(kind, vx, out=ob, strides=st)),
                                50, 5)
            moved = 2 * (kx.numel() * 2 + ob.numel())
            dk = qkv.QuantCache.empty(w.B, w.Hkv, 64, w.D, qkv.AFFINE, bits, 32, device)
            dv = qkv.QuantCache.empty(w.B, w.Hkv, 64, w.D, qkv.AFFINE, bits, 32, device)
            nk, nv = kx[:, :, :1].contiguous(), vx[:, :, :1].contiguous()
            sec1, _ = graph_time(lambda i: qkv.qkv_llama_quantize_update(kind, nk, nv, dk, dv, 63),
                                 200, 10)
            rows[f"llama_{kind}_quantize_64k"] = {
                "us_per_call": round(sec * 1e3, 3), "GB/s": round(moved / (sec / 1e3) / 1e9, 1),
                "frac_hbm": round(moved / (sec / 1e3) / 1e9 / hbm_peak, 4),
                "update_1tok_us": round(sec1 * 1e3, 3),
                "note": f"qkv_llama_quantize_blocks, K and V of 65536 tokens x 8 heads (2 x 16.8 MB "
                        f"fp16 in) to token-major {kind} blocks; update_1tok: "
                        f"qkv_llama_quantize_update of one token per head into the affine caches"}
            del ob, dk, dv
        del kx, vx
    except Exception as e:
        rows["llama_q4_0_quantize_64k"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    torch.cuda.empty_cache()

    # the attention extensions on the main decode workload (the extension
    # variant of the decode kernel): logit softcap 30 with per-head sinks, and
    # ALiBi (a broadcast fp32 distance mask with per-head slopes)
    w = S.WORKLOADS["decode_64k_affine4"]
    inp = S.make_inputs(w)
    ncopies = max(3, math.ceil(3 * 126e6 / w.cache_bytes()))
    caches = build_caches(w, inp, ncopies, device)
    q = dev16(inp.q, "f16", device)
    out = torch.empty(w.B, w.Hq, 1, w.D, dtype=torch.float16, device=device)
    ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, 1, w.D, w.L, device)
    sinks = torch.linspace(8.0, 12.0, w.Hq, device=device)
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / w.Hq) for h in range(w.Hq)], device=device)
    dist = -torch.arange(w.L - 1, -1, -1, dtype=torch.float32, device=device)
    nb = w.cache_bytes() + 2 * w.Hq * w.D * 2

    def estep(i, **kw):
        a, b = caches[i % ncopies]
        qkv.qsdpa_decode(q, a, b, w.L, w.scale, out=out, workspace=ws, **kw)
    sec_c, _ = graph_time(lambda i: estep(i, softcap=30.0, sinks=sinks), 400, 20)
    sec_a, _ = graph_time(lambda i: estep(i, mask=(dist, (0, 0, 0)), mask_slopes=slopes), 400, 20)
    rows["extensions_decode_64k_affine4"] = {
        "softcap_sinks_us_per_call": round(sec_c * 1e3, 3),
        "softcap_sinks_frac_hbm": round(nb / (sec_c / 1e3) / 1e9 / hbm_peak, 4),
        "alibi_us_per_call": round(sec_a * 1e3, 3),
        "alibi_frac_hbm": round(nb / (sec_a / 1e3) / 1e9 / hbm_peak, 4),
        "note": "qsdpa_decode_ext on decode_64k_affine4: softcap 30 + per-head sinks; ALiBi as "
                "a broadcast fp32 distance mask (256 KB) with per-head slopes; compare the "
                "bench value"}
    del caches
    torch.cuda.empty_cache()

    # the same for the prefill workload: softcap 30 + sinks on the tcgen05 kernel
    w = S.WORKLOADS["prefill_q8_0_512_at_20k"]
    inp = S.make_inputs(w)
    kc, vc = build_caches(w, inp, 1, device)[0]
    q = dev16(inp.q, w.q_dtype, device)
    out = torch.empty(w.B, w.Hq, w.Lq, w.D, dtype=torch.bfloat16, device=device)
    ws = qkv.make_workspace(w.B, w.Hq, w.Hkv, w.Lq, w.D, w.L, device)
    sinks = torch.linspace(8.0, 12.0, w.Hq, device=device)
    sec, _ = graph_time(lambda i: qkv.qsdpa_prefill(q, kc, vc, w.L, w.scale, causal=True, out=out,
                                                    workspace=ws, softcap=30.0, sinks=sinks),
                        20, 3)
    # ALiBi: per-query distances (fp32 [Lq, L], -inf above the causal
    # diagonal, broadcast over heads) with per-head slopes
    qpos = torch.arange(w.L - w.Lq, w.L, device=device).view(-1, 1)
    dist = (torch.arange(w.L, device=device).view(1, -1) - qpos).float()
    alibi = torch.where(dist <= 0, dist, torch.full_like(dist, -float("inf"))).contiguous()
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / w.Hq) for h in range(w.Hq)], device=device)
    sec_m, _ = graph_time(lambda i: qkv.qsdpa_prefill(q, kc, vc, w.L, w.scale, mask=(alibi, (0, 0, w.L)),
                                                      out=out, workspace=ws, mask_slopes=slopes),
                          10, 3)
    flop = prefill_flops(w)
    _, bf16_peak, _ = peaks()
    rows["extensions_" + w.name] = {
        "softcap_sinks_us_per_call": round(sec * 1e3, 2),
        "TFLOP/s": round(flop / (sec / 1e3) / 1e12, 1),
        "frac_tensor_peak": round(flop / (sec / 1e3) / 1e12 / bf16_peak, 4),
        "alibi_mask_us_per_call": round(sec_m * 1e3, 2),
        "alibi_mask_frac_tensor_peak": round(flop / (sec_m / 1e3) / 1e12 / bf16_peak, 4),
        "note": "qsdpa_prefill_ext, softcap 30 + per-head sinks; and an ALiBi additive mask (fp32 "
                "[Lq, L] distances, -inf above the causal diagonal, broadcast over heads) with "
                "per-head slopes; compare prefill_q8_0_512_at_20k"}
    del alibi, dist
    del kc, vc
    torch.cuda.empty_cache()
    return rows


def prefill_flops(w):
    """Multiply-adds of Q K^T and P V actually required (causal keys only):
    4 * D * Hq * sum over queries of visible keys."""
    vis = sum(min(w.L, w.L - w.Lq + i + 1) for i in range(w.Lq))
    return 4 * w.D * w.Hq * w.B * vis


def run_reference(args, rank, world):
    """CPU oracle on a bounded sample of the workload, same metric."""
    import oracle
    from quantized_kv_attention_split_b200 import synthetic as S
    if rank != 0:
        return None
    w = S.WORKLOADS[args.workload]
    inp = S.make_inputs(w)
    kc = oracle.quantize(inp.k, w.kv_dtype, w.fmt, w.gs, w.bits)
    vc = oracle.quantize(inp.v, w.kv_dtype, w.fmt, w.gs, w.bits)
    alg_bytes = w.cache_bytes() + 2 * w.B * w.Hq * w.Lq * w.D * 2
    total_rows = w.B * w.Hq * w.Lq
    threads = oracle.default_threads()
    # size each step so the whole run stays within --ref-seconds (two minutes by default)
    t0 = time.time()
    oracle.attention(inp.q, w.q_dtype, kc, vc, w.L, w.scale, rows=np.array([0]), nthreads=1)
    t_row = max(1e-4, time.time() - t0)
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    nrows = int(min(total_rows, max(1, per_step * threads / t_row)))
    rows = np.linspace(0, total_rows - 1, nrows).astype(np.int64)
    for _ in range(args.warmup):
        oracle.attention(inp.q, w.q_dtype, kc, vc, w.L, w.scale, rows=rows, nthreads=threads)
    t0 = time.time()
    for _ in range(args.steps):
        oracle.attention(inp.q, w.q_dtype, kc, vc, w.L, w.scale, rows=rows, nthreads=threads)
    dt = (time.time() - t0) / max(1, args.steps)
    gbs = (nrows / total_rows) * alg_bytes / dt / 1e9
    sample = f"{nrows} of {total_rows} query rows over all {w.L} keys per step"
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_64k_affine4")
    ap.add_argument("--rows", dest="rows", action="store_true", default=True)
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="CPU time budget of the --impl reference run (oracle on a sample)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import datetime
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        res = run_ours(args, rank, world, device)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
