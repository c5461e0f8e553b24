#!/usr/bin/env python
"""Benchmark of the hybrid compressed attention decode step (CSA + HCA) on B200.

Default workload: 1M-context decode, B=4 sequences of N=2^20 raw tokens (262,144 CSA entries and
8,192 HCA entries each), production widths (d=512 latent, 64 heads, indexer 4 x 64, top-k 1024,
window 128, m'=128).  A step = one decode step of all B sequences through ``hybrid_attn_decode``:
append one token per sequence (compressing the entries it completes), indexer scan + exact top-k,
sparse attention over the selected entries + window, dense HCA attention, log-sum-exp merge.

Prints one JSON line (rank 0).  Inputs are synthetic (seeded counter-based generator), resident in
HBM before the timed region; the per-step working set (about 172 MB) exceeds the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config ctx1m|...]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA+HCA decode queries/s at 1M ctx; achieved HBM GB/s vs ~8 TB/s peak"

# DRAM bytes (read + write) of one index_scan_kernel launch at the 1M-context workload (B=4), from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel source it
# was taken on: the key is the SHA-256 prefix of csrc/index_topk.cu at that capture.  Any other
# source reports null traffic until it is captured again.
SCAN_TRAFFIC = {"source_sha256": "0c71bf725604b67a", "bytes": 134291712 + 5024512}


def _source_sha(name):
    import hashlib
    path = os.path.join(ROOT, "compressed_sparse_kv_overlapped_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def scan_traffic():
    """The captured DRAM bytes of one scan launch if they belong to the current scan source, else None."""
    try:
        if SCAN_TRAFFIC["source_sha256"] and _source_sha("index_topk.cu") == SCAN_TRAFFIC["source_sha256"]:
            return SCAN_TRAFFIC["bytes"]
    except OSError:
        pass
    return None


def graph_kernel_nodes(graph):
    """Kernel nodes of a captured CUDA graph (torch.cuda.CUDAGraph(keep_graph=True)): the number of
    kernel launches one replay makes."""
    from cuda.bindings import runtime as rt
    err, _, n = rt.cudaGraphGetNodes(graph.raw_cuda_graph(), 0)
    if err != rt.cudaError_t.cudaSuccess:
        return None
    err, nodes, n = rt.cudaGraphGetNodes(graph.raw_cuda_graph(), n)
    if err != rt.cudaError_t.cudaSuccess:
        return None
    count = 0
    for node in nodes[:n]:
        err, typ = rt.cudaGraphNodeGetType(node)
        if err == rt.cudaError_t.cudaSuccess and typ == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
            count += 1
    return count


def max_over_ranks(values, dev, world):
    """Element-wise maximum of `values` over the ranks (the slowest rank sets the job's time);
    the values themselves on one rank."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="ctx1m", choices=["ctx1m", "long", "ragged", "tiny", "prefill"],
                    help="decode workloads (the default ctx1m is the headline), or the causal prefill of "
                         "131,072 queries, reported as tensor-pipe throughput")
    ap.add_argument("--keys", default="bf16", choices=["bf16", "mx8"],
                    help="indexer keys of the decode workloads: bf16 (the workload as stated) or 8-bit block-scaled")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp4"],
                    help="compressed entries the decode attention reads: bf16 (the workload as stated) or FP4 "
                         "with 32-channel block scales")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--stage", default=None, choices=["index", "attn", "compress"],
                    help="time one stage alone on a compact case of the workload's geometry (profiling aid); "
                         "compress: the full compressor pass at the prefill geometry")
    ap.add_argument("--prefill-n", type=int, default=None,
                    help="sequence length of the prefill workload (default 131,072; a smaller one for profiling)")
    return ap.parse_args()


def peaks(sustained=False):
    """(copy GB/s, bf16 TFLOP/s, source): the measured figures of MEASURED_PEAKS.json, else the
    fallback measurement on this hardware (6,650 GB/s; 1,590 TFLOP/s burst, 1,400 sustained)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        tf = p.get("bf16_tflops_sustained" if sustained else "bf16_tflops", 1590.0)
        return float(p["hbm_gbs"]), float(tf), "measured (MEASURED_PEAKS.json)"
    except Exception:
        return 6650.0, 1400.0 if sustained else 1590.0, "fallback (MEASURED_PEAKS.json absent)"


# ------------------------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls NVML (SM clock, max SM clock, clock-event reasons) every 2 ms in a thread."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                self.samples.append((t, mhz, int(self._reasons())))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside if inside else self.samples[-5:]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = sorted(s[1] for s in use)
        bits = 0
        for s in use:
            bits |= s[2]
        names = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(inside), "window": "timed region" if inside else "right after the timed region"}


# ------------------------------------------------------------------------------------ workloads

def workload(name):
    from synth import workloads
    return {"ctx1m": workloads.ctx1m_decode, "long": workloads.long_decode, "ragged": workloads.ragged_decode,
            "tiny": workloads.tiny}[name]()


def dims_of(wd):
    import compressed_sparse_kv_overlapped_b200 as csa
    return csa.make_dims(d=wd.d, H=wd.H, d_I=wd.d_I, H_I=wd.H_I, m=wd.m, m_hca=wd.m_hca, k=wd.k, W=wd.W)


def step_bytes(wd, lens, keys="bf16", kv="bf16"):
    """Algorithmic HBM bytes of one decode step: indexer-key scan, gathered top-k entries, raw window,
    HCA entries (queries and outputs not counted), the block-scale bytes of 8-bit keys (one per 32 key
    channels; 0 for bf16 keys) and of FP4 entries (one per 32 channels of every gathered or HCA entry;
    0 for bf16 entries, whose rows are then 2 bytes per channel instead of half a byte)."""
    kb = wd.d_I if keys == "mx8" else wd.d_I * 2
    eb = wd.d // 2 if kv == "fp4" else wd.d * 2
    idx = sum((L // wd.m) * kb for L in lens)
    scales = sum((L // wd.m) * (wd.d_I // 32) for L in lens) if keys == "mx8" else 0
    gather = sum(min(wd.k, L // wd.m) * eb for L in lens)
    window = sum(min(wd.W, L) * wd.d * 2 for L in lens)
    hca = sum((L // wd.m_hca) * eb for L in lens)
    escales = sum((min(wd.k, L // wd.m) + L // wd.m_hca) * (wd.d // 32) for L in lens) if kv == "fp4" else 0
    return idx, gather, window, hca, scales, escales


# ------------------------------------------------------------------------------------ our arm

def run_ours(args, rank, world):
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    from synth import device as sdev

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = workload(args.config)
    wd = wl.dims
    B = wl.B
    K, W = args.steps, args.warmup
    extra = W + K + (0 if args.no_e2e else W + K) + 1
    layer = csa.HybridLayer(dims_of(wd), [n + extra for n in wl.n0], device=dev, key_format=args.keys,
                            kv_format=args.kv)
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths(list(wl.n0))
    layer.compress()
    steps_total = W + K
    q_all = torch.empty(steps_total, B, wd.H, wd.d, dtype=torch.bfloat16, device=dev)
    qi_all = torch.empty(steps_total, B, wd.H_I, wd.d_I, dtype=torch.bfloat16, device=dev)
    w_all = torch.empty(steps_total, B, wd.H_I, dtype=torch.float32, device=dev)
    tq = torch.empty(steps_total, wd.H, wd.d, dtype=torch.bfloat16, device=dev)
    tqi = torch.empty(steps_total, wd.H_I, wd.d_I, dtype=torch.bfloat16, device=dev)
    tw = torch.empty(steps_total, wd.H_I, dtype=torch.float32, device=dev)
    for b in range(B):  # generate each sequence's rows contiguously, then scatter into [step, b]
        sdev.fill_queries(wl, b, 0, steps_total, tq, tqi, tw)
        q_all[:, b].copy_(tq)
        qi_all[:, b].copy_(tqi)
        w_all[:, b].copy_(tw)
    del tq, tqi, tw
    out = torch.empty(B, wd.H, wd.d, dtype=torch.float32, device=dev)
    max_len = max(layer.capacity)
    ws = layer.decode_workspace(max_len)
    torch.cuda.synchronize()

    def args_for(s):
        return layer.decode_args(q_all[s], qi_all[s], w_all[s], out, max_len=max_len)

    # warm-up (eager)
    for s in range(W):
        layer.decode(args_for(s), ws)
    st = csa.csa_sync_status()
    if st != csa.CSA_OK:
        raise RuntimeError(f"device status {st} during warm-up")

    # Two graphs of K decode steps each: the timed one (the product path as a caller runs it) and
    # an identical one with per-stage CUDA events recorded between the kernels (events between
    # kernels disable programmatic dependent launch there, so it is timed separately).
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(csa.CSA_DECODE_MARKS * K)]
    for e in marks:  # torch creates the CUDA event on first record
        e.record()
    torch.cuda.synchronize()
    lens_before = list(layer.lens)
    stream = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream):
        for s in range(K):
            csa.hybrid_attn_decode(args_for(W + s), ws, torch.cuda.current_stream())
    launches = graph_kernel_nodes(graph)
    graph.instantiate()
    graph_ev = torch.cuda.CUDAGraph()
    csa.csa_set_stage_events(marks)
    with torch.cuda.graph(graph_ev, stream=stream):
        for s in range(K):
            csa.hybrid_attn_decode(args_for(W + s), ws, torch.cuda.current_stream())
    csa.csa_set_stage_events(None)

    def reset_lengths():
        layer.set_lengths(lens_before)
        torch.cuda.synchronize()

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.05)
    # one untimed replay of the same K steps first, so the timed one starts on a busy GPU (clocks up,
    # caches in their steady state) rather than after the idle wait above
    reset_lengths()
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()  # (the reset below is a copy on another stream)
    reset_lengths()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        e0.record()
        graph.replay()
        e1.record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
    clocks.stop()
    st = csa.csa_sync_status()
    if st != csa.CSA_OK:
        raise RuntimeError(f"device status {st} in the timed region")
    ms, = max_over_ranks([e0.elapsed_time(e1)], dev, world)
    # the same K steps again, with the stage events
    reset_lengths()
    with torch.cuda.stream(stream):
        graph_ev.replay()
    torch.cuda.synchronize()
    st = csa.csa_sync_status()
    if st != csa.CSA_OK:
        raise RuntimeError(f"device status {st} in the stage-timed region")
    layer.lens = [n + K for n in lens_before]

    # per-stage durations inside the timed region
    M = csa.CSA_DECODE_MARKS
    stage = {"append": 0.0, "index_scan": 0.0, "topk_select": 0.0, "attention": 0.0}
    for s in range(K):
        ev = marks[M * s:M * (s + 1)]
        stage["append"] += ev[0].elapsed_time(ev[1])
        stage["index_scan"] += ev[1].elapsed_time(ev[2])
        stage["topk_select"] += ev[2].elapsed_time(ev[3])
        stage["attention"] += ev[3].elapsed_time(ev[4])
    stage = {k: v / K for k, v in stage.items()}
    # per-step durations (first mark to last) in the stage-event graph, whose events keep the kernels
    # of a step from overlapping; the timed graph has no per-step events
    steps_sorted = sorted(marks[M * s].elapsed_time(marks[M * s + M - 1]) for s in range(K))

    def pct(q):
        return steps_sorted[min(K - 1, int(round(q * (K - 1))))]

    # algorithmic bytes per step (lengths after each step's append)
    tot = [0, 0, 0, 0, 0, 0]
    for s in range(K):
        lens = [n + s + 1 for n in lens_before]
        for i, v in enumerate(step_bytes(wd, lens, args.keys, args.kv)):
            tot[i] += v
    per_step = [v / K for v in tot]
    bytes_step = sum(per_step)
    hbm_peak, tf_peak, peak_src = peaks()
    ms_step = ms / K
    achieved_step_gbs = bytes_step / (ms_step * 1e-3) / 1e9
    scan_ms = stage["index_scan"]
    scan_bytes = per_step[0] + per_step[4]  # keys and, for 8-bit keys, their scale bytes
    scan_gbs = scan_bytes / (scan_ms * 1e-3) / 1e9 if scan_ms > 0 else None
    result = {
        "metric": METRIC, "value": B * world * K / (ms * 1e-3), "unit": "queries/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": wl.name + ("_mx8keys" if args.keys == "mx8" else "") + ("_fp4kv" if args.kv == "fp4" else ""),
                   "B": B, "N": wl.n0[0] if len(set(wl.n0)) == 1 else "ragged", "indexer_keys": args.keys,
                   "entries": args.kv,
                   "d": wd.d, "heads": wd.H, "d_I": wd.d_I, "H_I": wd.H_I, "k": wd.k, "W": wd.W, "m": wd.m,
                   "m_hca": wd.m_hca, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "per-step working set larger than L2 (no flush)"},
        "hbm": {"algorithmic_bytes_per_step": int(bytes_step),
                "breakdown_bytes": {"index_keys": int(per_step[0]), "scale_bytes": int(per_step[4]),
                                    "gathered_entries": int(per_step[1]), "window": int(per_step[2]),
                                    "hca_entries": int(per_step[3]), "entry_scale_bytes": int(per_step[5])},
                "achieved_gbs": achieved_step_gbs, "peak_gbs": hbm_peak, "frac": achieved_step_gbs / hbm_peak,
                "peak_source": peak_src},
        "stages_ms": stage,
        "stages_note": "per-stage CUDA events recorded on the decode stream in a second, identical K-step graph",
        "stage_graph_step_ms": {"p50": pct(0.50), "p95": pct(0.95), "p99": pct(0.99), "max": steps_sorted[-1],
                                "note": "per-step durations in the stage-event graph (no launch overlap inside a "
                                        "step), not the timed graph"},
        "roofline": {"kernel": "index_scan_kernel", "bound": "hbm", "achieved": scan_gbs, "peak": hbm_peak,
                     "unit": "GB/s", "frac": (scan_gbs / hbm_peak) if scan_gbs else None,
                     "traffic": scan_traffic() if wl.name.startswith("ctx1m") and args.keys == "bf16" else None,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch, "
                                       "taken on the current scan source (null otherwise)",
                     "bytes_per_launch": int(scan_bytes), "peak_source": f"{peak_src}: copy bandwidth"},
        "clocks": clocks.summary(t0, t1),
    }
    # kernel nodes of the timed graph (all of them this library's kernels)
    result["gpu_launches"] = launches

    if not args.no_e2e:
        result["e2e"] = run_e2e(layer, wl, K, W, max_len, ws, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, keys=args.keys, kv=args.kv)
    return result


def run_e2e(layer, wl, K, W, max_len, ws, dev, world):
    """The same decode steps through the C ABI with each step's inputs in pinned HOST memory: per step
    one host->device copy of a packed buffer (queries, indexer queries, head weights and the appended
    token's raw rows, handed to the call as new_rows) and one device->host read of the output, all
    inside the timed region.  Two staging slots: the copy stream moves step s+1's inputs in and step
    s-1's output out while the decode stream computes step s; the copies and events are issued
    through the CUDA runtime directly (no per-copy framework overhead).  W untimed steps through the
    same loop come first, after whole warm-up passes lasting at least 100 ms.  (Replaying each step's call from a CUDA graph was measured slower here
    than the eager calls: the graph launch adds its own latency at every step boundary.)"""
    import numpy as np
    import torch
    from cuda.bindings import runtime as rt

    import compressed_sparse_kv_overlapped_b200 as csa
    from synth import workloads

    wd = wl.dims
    B = wl.B
    base = W + K  # query rows already used
    n_steps = W + K
    sizes = [B * wd.H * wd.d * 2, B * wd.H_I * wd.d_I * 2, B * wd.H_I * 4, B * (3 * wd.d + wd.d_I) * 2]
    offs = [0]
    for n in sizes:
        offs.append(offs[-1] + ((n + 255) // 256) * 256)
    step_bytes = offs[-1]
    host = torch.empty(n_steps, step_bytes, dtype=torch.uint8).pin_memory()
    lens0 = list(layer.lens)
    for s in range(n_steps):
        qs = [workloads.queries(wl, b, base + s, base + s + 1) for b in range(B)]
        rows = np.stack([np.concatenate([workloads.raw_tokens(wl, b, lens0[b] + s, lens0[b] + s + 1, name)[0]
                                         for name in ("x", "a", "b", "kI")]) for b in range(B)])
        for i, arr in enumerate([np.stack([t[j][0] for t in qs]) for j in range(3)] + [rows]):
            raw = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
            host[s, offs[i]:offs[i] + raw.size] = torch.from_numpy(raw)
    stages, outs, argv = [], [], []
    for i in range(2):
        st = torch.empty(step_bytes, dtype=torch.uint8, device=dev)
        dq = st[offs[0]:offs[0] + sizes[0]].view(torch.bfloat16).view(B, wd.H, wd.d)
        dqi = st[offs[1]:offs[1] + sizes[1]].view(torch.bfloat16).view(B, wd.H_I, wd.d_I)
        dw = st[offs[2]:offs[2] + sizes[2]].view(torch.float32).view(B, wd.H_I)
        drows = st[offs[3]:offs[3] + sizes[3]].view(torch.bfloat16).view(B, 3 * wd.d + wd.d_I)
        o = torch.empty(B, wd.H, wd.d, dtype=torch.float32, device=dev)
        stages.append(st)
        outs.append(o)
        argv.append(layer.decode_args(dq, dqi, dw, o, max_len=max_len, new_rows=drows))
    out_bytes = outs[0].numel() * 4
    hout = torch.empty(n_steps, B, wd.H, wd.d, dtype=torch.float32).pin_memory()
    h2d = sum(sizes)
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream(device=dev)
    ok = rt.cudaError_t.cudaSuccess

    def ck(r):
        if r[0] != ok:
            raise RuntimeError(f"CUDA runtime call failed in the e2e loop: {r[0]}")
        return r[1] if len(r) > 1 else None

    def event():
        return ck(rt.cudaEventCreateWithFlags(rt.cudaEventDisableTiming))

    h2d_done, comp_done, d2h_done = [event() for _ in range(2)], [event() for _ in range(2)], [event() for _ in range(2)]
    ds, cs = rt.cudaStream_t(stream.cuda_stream), rt.cudaStream_t(copy_stream.cuda_stream)
    H2D, D2H = rt.cudaMemcpyKind.cudaMemcpyHostToDevice, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost
    host_ptr, hout_ptr = host.data_ptr(), hout.data_ptr()
    stage_ptr, out_ptr = [t.data_ptr() for t in stages], [t.data_ptr() for t in outs]

    def loop(s0, s1):
        def h2d_step(s):
            i = s % 2
            if s - s0 >= 2:
                ck(rt.cudaStreamWaitEvent(cs, comp_done[i], 0))  # step s-2 has finished reading slot i
            ck(rt.cudaMemcpyAsync(stage_ptr[i], host_ptr + s * step_bytes, step_bytes, H2D, cs))
            ck(rt.cudaEventRecord(h2d_done[i], cs))

        h2d_step(s0)
        for s in range(s0, s1):
            i = s % 2
            if s + 1 < s1:
                h2d_step(s + 1)
            ck(rt.cudaStreamWaitEvent(ds, h2d_done[i], 0))
            if s - s0 >= 2:
                ck(rt.cudaStreamWaitEvent(ds, d2h_done[i], 0))  # step s-2's output has left slot i
            csa.hybrid_attn_decode(argv[i], ws, stream)
            ck(rt.cudaEventRecord(comp_done[i], ds))
            ck(rt.cudaStreamWaitEvent(cs, comp_done[i], 0))
            ck(rt.cudaMemcpyAsync(hout_ptr + s * out_bytes, out_ptr[i], out_bytes, D2H, cs))
            ck(rt.cudaEventRecord(d2h_done[i], cs))
        ck(rt.cudaStreamWaitEvent(ds, d2h_done[(s1 - 1) % 2], 0))

    # untimed warm-up through the same path: whole passes over the step rows (lengths reset before
    # each) until at least 100 ms have gone by (the host side of a cold eager loop runs slower for its
    # first milliseconds), then the W warm-up steps that precede the timed ones
    t_warm = time.perf_counter()
    while True:
        layer.set_lengths(lens0)
        loop(0, n_steps)
        torch.cuda.synchronize()
        if time.perf_counter() - t_warm >= 0.1:
            break
    layer.set_lengths(lens0)
    loop(0, W)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    ck(rt.cudaStreamWaitEvent(cs, rt.cudaEvent_t(e0.cuda_event), 0))
    loop(W, W + K)
    e1.record(stream)
    torch.cuda.synchronize()
    st = csa.csa_sync_status()
    if st != csa.CSA_OK:
        raise RuntimeError(f"device status {st} in the e2e region")
    ms, = max_over_ranks([e0.elapsed_time(e1)], dev, world)
    layer.lens = [n + n_steps for n in lens0]
    for e in h2d_done + comp_done + d2h_done:
        rt.cudaEventDestroy(e)
    return {"value": B * world * K / (ms * 1e-3), "unit": "queries/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(out_bytes), "ms_per_step": ms / K,
            "how": "eager hybrid_attn_decode calls; per step one H2D copy of a packed pinned buffer (q, q_idx, w "
                   "and the appended token rows, passed as new_rows) and one D2H copy of the output, on a copy "
                   "stream double-buffered against the decode stream; untimed warm-up of the same loop (at "
                   "least 100 ms, then W steps) first"}


# ------------------------------------------------------------------------------------ oracle arm

class OracleDecode:
    """The fp64 oracle's decode query at the workload's geometry, for one prepared sequence: caches
    (indexer keys, HCA entries) are built untimed; CSA entries are built for the entries each sample
    query selects (also untimed).  A timed query runs the oracle's indexer scores, top-k, sparse
    attention with the window, HCA attention and LSE merge."""

    def __init__(self, wl, b=0, rows=(0,), keys="bf16", kv="bf16"):
        import numpy as np

        import oracle
        from synth import workloads
        self.wl, self.b = wl, b
        wd = wl.dims
        L = wl.n0[b] + 1
        self.L = L
        self.shape = oracle.Shape(d=wd.d, H=wd.H, d_I=wd.d_I, H_I=wd.H_I, m=wd.m, m_hca=wd.m_hca, k=wd.k, W=wd.W)
        x = workloads.raw_tokens(wl, b, 0, L, "x")
        a_idx = workloads.raw_tokens_cols(wl, b, 0, L, "a", 0, wd.d_I)
        kI = workloads.raw_tokens(wl, b, 0, L, "kI")
        bias_c = workloads.bias_c(wl)
        n_c, n_h = L // wd.m, L // wd.m_hca
        # indexer keys: the compressor on channels 0..d_I-1 with the raw indexer keys as values
        KI, _ = oracle.compress_parallel(kI, a_idx, np.ascontiguousarray(bias_c[:, :wd.d_I]), None, L, wd.m,
                                         2 * wd.m, np.arange(n_c))
        self.KI = oracle.round_bf16(KI)
        self.keys_mx8 = oracle.quantize_keys_mx8(self.KI) if keys == "mx8" else None
        del a_idx, kI
        bl = workloads.raw_tokens(wl, b, 0, L, "b")
        H, _ = oracle.compress_parallel(x, bl, workloads.bias_h(wl), None, L, wd.m_hca, wd.m_hca, np.arange(n_h))
        self.H = oracle.round_bf16(H)
        if kv == "fp4" and n_h:
            self.H = oracle.mx4_entries_as_bf16(self.H)
        del bl
        self.x = x
        self.E = np.zeros((n_c, wd.d), np.uint16)
        self.queries = [tuple(t[0] for t in workloads.queries(wl, b, r, r + 1)) for r in rows]

        def selection(qv):  # the entries a sample query selects (untimed preparation)
            _, qi, w = qv
            sc = (oracle.index_scores_mx8(qi, w, *self.keys_mx8) if self.keys_mx8 is not None
                  else oracle.index_scores(qi, w, self.KI))
            return oracle.topk(sc, wd.k)

        sel = oracle.parallel_map(selection, self.queries)
        need = np.unique(np.concatenate([i[i >= 0] for i in sel])).astype(np.int64)
        a = workloads.raw_tokens(wl, b, 0, L, "a")
        E, _ = oracle.compress_parallel(x, a, bias_c, None, L, wd.m, 2 * wd.m, need)
        self.E[need] = oracle.mx4_entries_as_bf16(oracle.round_bf16(E)) if kv == "fp4" else oracle.round_bf16(E)

    def run(self, i):
        import oracle
        q, qi, w = self.queries[i]
        return oracle.hybrid_query(self.shape, self.L, q, qi, w, self.x, self.E, self.KI, self.H,
                                   keys_mx8=self.keys_mx8)


def cpu_baseline(wl, samples=None, keys="bf16", kv="bf16"):
    """The oracle on a bounded sample of the workload: one decode query per host core (at least 4) on
    one prepared sequence, in parallel threads (the oracle's C code releases the GIL)."""
    from concurrent.futures import ThreadPoolExecutor
    host = os.cpu_count() or 1
    samples = samples or max(4, host)
    threads = min(samples, host)
    od = OracleDecode(wl, 0, rows=tuple(range(samples)), keys=keys, kv=kv)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(od.run, range(samples)))
    dt = time.perf_counter() - t0
    return {"value": samples / dt, "unit": "queries/s", "cores": threads, "host_cores": host, "kind": "oracle",
            "sample": f"{samples} decode queries of one sequence at L={od.L} (the workload's geometry, {keys} "
                      f"indexer keys, {kv} entries), caches prepared untimed (FP4 entries dequantized), one query "
                      f"per thread"}


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores, on this arm's config / metric / unit.  A step is one
    decode query per sequence slot (B of them), evaluated on one prepared sequence in parallel."""
    if rank != 0:
        return None
    from concurrent.futures import ThreadPoolExecutor
    wl = workload(args.config)
    B = wl.B
    K, W = args.steps, args.warmup
    od = OracleDecode(wl, 0, rows=tuple(range(B)), keys=args.keys, kv=args.kv)
    threads = min(B, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        for _ in range(W):
            list(ex.map(od.run, range(B)))
        t0 = time.perf_counter()
        for _ in range(K):
            list(ex.map(od.run, range(B)))
        dt = time.perf_counter() - t0
    v = B * K / dt
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "queries/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": dt * 1e3 / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded counter-based generator)",
            "config": {"workload": wl.name + ("_mx8keys" if args.keys == "mx8" else "") +
                                   ("_fp4kv" if args.kv == "fp4" else ""), "B": B},
            "cpu_baseline": {"value": v, "unit": "queries/s", "cores": threads, "kind": "oracle",
                             "sample": f"each step: {B} decode queries at L={od.L} on one prepared sequence"},
            "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_stage_index(args):
    """csa_index_topk alone at the workload's indexer geometry (B queries over B sequences of
    floor(N/4) entries of d_I-wide keys, keys N(0, 0.5^2)); no raw-token arrays, so the device holds
    only the key cache (128 MiB at ctx1m) and the scratch.  Times K launches with CUDA events."""
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    import synth
    wl = workload(args.config)
    wd = wl.dims
    B = wl.B
    E = [n // wd.m for n in wl.n0]
    keys = torch.empty(sum(E), wd.d_I, dtype=torch.bfloat16, device="cuda")
    off = 0
    rows = []
    for b in range(B):
        synth.dev_fill("bf16_normal", wl.seed, synth.KI, b, wd.d_I, 0, E[b], keys[off].data_ptr(), scale=0.5)
        rows.append([0, off, 0, wl.n0[b]])
        off += E[b]
    seqs = torch.tensor(rows, dtype=torch.int64, device="cuda")
    qt = torch.tensor([[b, wl.n0[b]] for b in range(B)], dtype=torch.int64, device="cuda")
    qi = torch.empty(B, wd.H_I, wd.d_I, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(B, wd.H_I, dtype=torch.float32, device="cuda")
    for b in range(B):
        synth.dev_fill("bf16_normal", wl.seed, synth.QI, b, wd.H_I * wd.d_I, 0, 1, qi[b].data_ptr())
        synth.dev_fill("f32_uniform", wl.seed, synth.W, b, wd.H_I, 0, 1, w[b].data_ptr())
    idx = torch.empty(B, wd.k, dtype=torch.int32, device="cuda")
    dims = dims_of(wd)
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, B, max(wl.n0)
    ws = torch.empty(csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, wq), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        csa.csa_index_topk(dims, seqs, qt, B, max(wl.n0), qi, w, keys, idx, None, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        csa.csa_index_topk(dims, seqs, qt, B, max(wl.n0), qi, w, keys, idx, None, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    nbytes = sum(E) * wd.d_I * 2
    hbm, _, src = peaks()
    assert csa.csa_sync_status() == csa.CSA_OK
    return {"stage": "index_topk (memset + scan + select)", "workload": wl.name, "ms_per_call": ms,
            "key_bytes": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9, "peak_gbs": hbm, "peak_source": src}


def prefill_flops(wd, N):
    """Algorithmic FLOPs of a causal prefill of N queries (query i sees L = i + 1 tokens): indexer
    scores 2*H_I*d_I per (query, causal entry); attention 4*H*d per (query, key) over the valid top-k
    entries, the window and the HCA entries (two products of 2*H*d each)."""
    import numpy as np
    L = np.arange(1, N + 1, dtype=np.float64)
    e_c = np.floor(L / wd.m)
    index = float((e_c * 2 * wd.H_I * wd.d_I).sum())
    keys = np.minimum(e_c, wd.k) + np.minimum(L, wd.W) + np.floor(L / wd.m_hca)
    attn = float((keys * 4 * wd.H * wd.d).sum())
    return index, attn


def prefill_workload(args):
    import dataclasses

    from synth import workloads
    wl = workloads.prefill()
    if args.prefill_n:
        wl = dataclasses.replace(wl, name=f"prefill_N{args.prefill_n}", n0=(int(args.prefill_n),))
    return wl


def compress_bytes(wd, N):
    """Algorithmic bytes of the full compressor pass over N tokens: the token rows (x, both logit
    arrays, raw indexer keys) read once; CSA entries with their indexer keys and HCA entries written."""
    return N * (3 * wd.d + wd.d_I) * 2 + (N // wd.m) * (wd.d + wd.d_I) * 2 + (N // wd.m_hca) * wd.d * 2


def run_stage_compress(args):
    """csa_compress_all alone (one pass for the CSA entries, their indexer keys and the HCA entries)
    at the prefill geometry; K calls timed with CUDA events."""
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    from synth import device as sdev
    wl = prefill_workload(args)
    wd = wl.dims
    N = wl.n0[0]
    layer = csa.HybridLayer(dims_of(wd), [N])
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    for _ in range(args.warmup):
        layer.compress()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        layer.compress()
    e1.record()
    torch.cuda.synchronize()
    assert csa.csa_sync_status() == csa.CSA_OK
    ms = e0.elapsed_time(e1) / args.steps
    nb = compress_bytes(wd, N)
    hbm, _, src = peaks()
    return {"stage": "compress (csa_compress_all, CSA + keys + HCA in one pass)", "workload": wl.name,
            "us_per_call": ms * 1e3, "bytes": nb, "achieved_gbs": nb / (ms * 1e-3) / 1e9, "peak_gbs": hbm,
            "frac": nb / (ms * 1e-3) / 1e9 / hbm, "peak_source": src}


def run_prefill(args, rank, world):
    """Causal prefill of one sequence (hybrid_attn_prefill over all N queries; the compressor pass
    is timed on its own, then each step runs the indexer, top-k and attention for every query).
    Reported as queries/s and as tensor-pipe TFLOP/s against the measured sustained bf16 peak."""
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    from synth import device as sdev
    from synth import workloads
    wl = prefill_workload(args)
    wd = wl.dims
    N = wl.n0[0]
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    layer = csa.HybridLayer(dims_of(wd), [N], device=dev)
    sdev.fill_layer_inputs(layer, wl)
    layer.set_lengths([N])
    q = torch.empty(N, wd.H, wd.d, dtype=torch.bfloat16, device=dev)
    qi = torch.empty(N, wd.H_I, wd.d_I, dtype=torch.bfloat16, device=dev)
    w = torch.empty(N, wd.H_I, dtype=torch.float32, device=dev)
    sdev.fill_queries(wl, 0, 0, N, q, qi, w)
    out = torch.empty(N, wd.H, wd.d, dtype=torch.float32, device=dev)
    ws = layer.prefill_workspace(N)
    args_c = layer.prefill_args(q, qi, w, out, 0, N, compress=False)
    layer.compress()
    K, W = args.steps, args.warmup
    for _ in range(W):
        layer.prefill(args_c, ws)
    torch.cuda.synchronize()
    if csa.csa_sync_status() != csa.CSA_OK:
        raise RuntimeError("device status during warm-up")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.05)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev[0].record()
    for _ in range(K):
        layer.compress()
    ev[1].record()
    ev[2].record()
    for _ in range(K):
        layer.prefill(args_c, ws)
    ev[3].record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    clocks.stop()
    if csa.csa_sync_status() != csa.CSA_OK:
        raise RuntimeError("device status in the timed region")
    ms_comp = ev[0].elapsed_time(ev[1]) / K
    ms = ev[2].elapsed_time(ev[3]) / K
    ms, ms_comp = max_over_ranks([ms, ms_comp], dev, world)
    f_index, f_attn = prefill_flops(wd, N)
    hbm, tf_peak, src = peaks(sustained=True)
    tflops = (f_index + f_attn) / (ms * 1e-3) / 1e12
    comp_bytes = compress_bytes(wd, N)
    res = {
        "metric": "causal prefill queries/s (indexer + top-k + sparse/HCA attention); tensor TFLOP/s",
        "value": N * world / (ms * 1e-3), "unit": "queries/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": wl.name, "N": N, "d": wd.d, "heads": wd.H, "d_I": wd.d_I, "H_I": wd.H_I, "k": wd.k,
                   "W": wd.W, "m": wd.m, "m_hca": wd.m_hca, "prefill_chunk": int(os.environ.get("CSA_PREFILL_CHUNK", 0)) or 64 * torch.cuda.get_device_properties(dev).multi_processor_count,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "flops": {"index": f_index, "attention": f_attn, "total": f_index + f_attn},
        "roofline": {"kernel": "whole prefill (index + select + attention)", "bound": "tensor", "achieved": tflops,
                     "peak": tf_peak, "unit": "TFLOP/s", "frac": tflops / tf_peak, "traffic": None,
                     "peak_source": f"{src}: sustained bf16 tensor throughput"},
        "compress": {"ms": ms_comp, "bytes": comp_bytes, "achieved_gbs": comp_bytes / (ms_comp * 1e-3) / 1e9,
                     "peak_gbs": hbm, "frac": comp_bytes / (ms_comp * 1e-3) / 1e9 / hbm,
                     "note": "csa_compress_all: CSA entries, indexer keys and HCA entries over all N tokens, one pass"},
        "clocks": clocks.summary(t0, t1),
    }
    del q, qi, w, out, ws, args_c
    torch.cuda.empty_cache()
    if not args.no_e2e:
        res["e2e"] = prefill_e2e(layer, wl, K, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = prefill_cpu_baseline(wl)
    return res


def prefill_e2e(layer, wl, K, dev, world, chunk=8192):
    """The prefill through the public call with every input in pinned HOST memory: per step the raw
    rows (x, both logit arrays, indexer keys) and all queries go host -> device, the outputs device ->
    host, inside the timed region.  hybrid_attn_prefill runs over query chunks (compressing in the
    first), and a copy stream moves chunk i+1's queries in and chunk i-1's outputs out while chunk i
    computes."""
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    from synth import device as sdev
    wd = wl.dims
    N = wl.n0[0]
    try:
        h_raw = [torch.empty_like(t, device="cpu").pin_memory() for t in (layer.x, layer.logit_c, layer.logit_h,
                                                                          layer.idx_key)]
        h_q = torch.empty(N, wd.H, wd.d, dtype=torch.bfloat16).pin_memory()
        h_qi = torch.empty(N, wd.H_I, wd.d_I, dtype=torch.bfloat16).pin_memory()
        h_w = torch.empty(N, wd.H_I, dtype=torch.float32).pin_memory()
        h_out = torch.empty(N, wd.H, wd.d, dtype=torch.float32).pin_memory()
    except RuntimeError as e:
        return {"unavailable": f"pinned host buffers of {N} queries could not be allocated: {e}"[:200]}
    for h, t in zip(h_raw, (layer.x, layer.logit_c, layer.logit_h, layer.idx_key)):
        h.copy_(t)
    # the queries, generated on the device chunk by chunk and parked in host memory (untimed)
    tq = torch.empty(chunk, wd.H, wd.d, dtype=torch.bfloat16, device=dev)
    tqi = torch.empty(chunk, wd.H_I, wd.d_I, dtype=torch.bfloat16, device=dev)
    tw = torch.empty(chunk, wd.H_I, dtype=torch.float32, device=dev)
    for c0 in range(0, N, chunk):
        n = min(chunk, N - c0)
        sdev.fill_queries(wl, 0, c0, c0 + n, tq[:n], tqi[:n], tw[:n])
        h_q[c0:c0 + n].copy_(tq[:n])
        h_qi[c0:c0 + n].copy_(tqi[:n])
        h_w[c0:c0 + n].copy_(tw[:n])
    del tq, tqi, tw
    dq = [torch.empty(chunk, wd.H, wd.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dqi = [torch.empty(chunk, wd.H_I, wd.d_I, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dw = [torch.empty(chunk, wd.H_I, dtype=torch.float32, device=dev) for _ in range(2)]
    do = [torch.empty(chunk, wd.H, wd.d, dtype=torch.float32, device=dev) for _ in range(2)]
    ws = layer.prefill_workspace(N)
    stream = torch.cuda.current_stream()
    cs = torch.cuda.Stream(device=dev)
    nch = (N + chunk - 1) // chunk

    def one_step():
        raw_done = torch.cuda.Event()
        with torch.cuda.stream(cs):
            for h, t in zip(h_raw, (layer.x, layer.logit_c, layer.logit_h, layer.idx_key)):
                t.copy_(h, non_blocking=True)
            raw_done.record(cs)
        in_done = [torch.cuda.Event() for _ in range(nch)]
        comp_done = [torch.cuda.Event() for _ in range(nch)]
        out_done = [torch.cuda.Event() for _ in range(nch)]

        def h2d(i):
            c0, n, b = i * chunk, min(chunk, N - i * chunk), i % 2
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(comp_done[i - 2])
                dq[b][:n].copy_(h_q[c0:c0 + n], non_blocking=True)
                dqi[b][:n].copy_(h_qi[c0:c0 + n], non_blocking=True)
                dw[b][:n].copy_(h_w[c0:c0 + n], non_blocking=True)
                in_done[i].record(cs)

        h2d(0)
        stream.wait_event(raw_done)
        for i in range(nch):
            c0, n, b = i * chunk, min(chunk, N - i * chunk), i % 2
            if i + 1 < nch:
                h2d(i + 1)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])
            a = layer.prefill_args(dq[b], dqi[b], dw[b], do[b], c0, c0 + n, compress=(i == 0))
            csa.hybrid_attn_prefill(a, ws, stream)
            comp_done[i].record(stream)
            with torch.cuda.stream(cs):
                cs.wait_event(comp_done[i])
                h_out[c0:c0 + n].copy_(do[b][:n], non_blocking=True)
                out_done[i].record(cs)
        for i in range(max(0, nch - 2), nch):
            stream.wait_event(out_done[i])

    one_step()  # warm-up
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cs.wait_event(e0)
    for _ in range(K):
        one_step()
    e1.record(stream)
    torch.cuda.synchronize()
    if csa.csa_sync_status() != csa.CSA_OK:
        raise RuntimeError("device status in the prefill e2e region")
    ms, = max_over_ranks([e0.elapsed_time(e1) / K], dev, world)
    h2d_b = sum(t.numel() * t.element_size() for t in h_raw) + sum(t.numel() * t.element_size()
                                                                   for t in (h_q, h_qi, h_w))
    return {"value": N * world / (ms * 1e-3), "unit": "queries/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d_b), "d2h_bytes_per_step": int(h_out.numel() * 4),
            "how": f"hybrid_attn_prefill over chunks of {chunk} queries (compress in the first); raw rows and "
                   f"queries from pinned host memory, outputs back to pinned host memory, on a copy stream "
                   f"double-buffered against the compute stream"}


def prefill_cpu_baseline(wl, n_rows=512):
    """The oracle on 512 seeded query rows of the prefill (positions 0-4, 127, 128, 4095, 4096 and N-1
    among them), all host cores: caches (indexer keys and HCA entries for the whole sequence, CSA
    entries where a sampled row selects them) are prepared untimed; a timed row runs the oracle's
    indexer scores, top-k, sparse attention with the window, HCA attention and LSE merge."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle
    from synth import workloads
    wd = wl.dims
    N = wl.n0[0]
    rng = np.random.default_rng(wl.seed)
    fixed = [0, 1, 2, 3, 4, 127, 128, 4095, 4096, N - 1]
    rest = [int(r) for r in rng.choice(N, size=4 * n_rows, replace=False) if int(r) not in fixed]
    rows = sorted(fixed + rest[:n_rows - len(fixed)])
    shape = oracle.Shape(d=wd.d, H=wd.H, d_I=wd.d_I, H_I=wd.H_I, m=wd.m, m_hca=wd.m_hca, k=wd.k, W=wd.W)
    x = workloads.raw_tokens(wl, 0, 0, N, "x")
    a = workloads.raw_tokens(wl, 0, 0, N, "a")
    kI = workloads.raw_tokens(wl, 0, 0, N, "kI")
    bias_c = workloads.bias_c(wl)
    n_c, n_h = N // wd.m, N // wd.m_hca
    KI, _ = oracle.compress_parallel(kI, np.ascontiguousarray(a[:, :wd.d_I]), np.ascontiguousarray(bias_c[:, :wd.d_I]),
                                     None, N, wd.m, 2 * wd.m, np.arange(n_c))
    KI = oracle.round_bf16(KI)
    bl = workloads.raw_tokens(wl, 0, 0, N, "b")
    H, _ = oracle.compress_parallel(x, bl, workloads.bias_h(wl), None, N, wd.m_hca, wd.m_hca, np.arange(n_h))
    H = oracle.round_bf16(H)
    del bl, kI
    qs = [workloads.queries(wl, 0, r, r + 1) for r in rows]
    host = os.cpu_count() or 1
    with ThreadPoolExecutor(host) as ex:
        sel = list(ex.map(lambda i: oracle.topk(oracle.index_scores(qs[i][1][0], qs[i][2][0],
                                                                    KI[:(rows[i] + 1) // wd.m]), wd.k),
                          range(len(rows))))
    need = np.unique(np.concatenate([s[s >= 0] for s in sel] + [np.zeros(0, np.int32)]))
    E = np.zeros((max(n_c, 1), wd.d), np.uint16)
    if len(need):
        Ev, _ = oracle.compress_parallel(x, a, bias_c, None, N, wd.m, 2 * wd.m, need.astype(np.int64))
        E[need] = oracle.round_bf16(Ev)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(host) as ex:
        list(ex.map(lambda i: oracle.hybrid_query(shape, rows[i] + 1, qs[i][0][0], qs[i][1][0], qs[i][2][0], x, E, KI,
                                                  H), range(len(rows))))
    dt = time.perf_counter() - t0
    return {"value": len(rows) / dt, "unit": "queries/s", "cores": min(host, len(rows)), "host_cores": host,
            "kind": "oracle",
            "sample": f"{len(rows)} seeded query rows of the N={N} prefill (positions 0-4, 127, 128, 4095, 4096, "
                      f"N-1 among them), caches prepared untimed, one row per thread"}


def run_stage_attn(args):
    """The decode attention alone at the workload's geometry: for each of the B queries, the sparse
    CSA part (k selected entries + W window tokens) through csa_sparse_attn and the HCA part
    (floor(N/m') entries) through hca_dense_attn, on caches filled directly with N(0, 0.5^2) values
    (no raw-token arrays beyond the window rows).  Times K launches of each with CUDA events."""
    import numpy as np
    import torch

    import compressed_sparse_kv_overlapped_b200 as csa
    import synth
    wl = workload(args.config)
    wd = wl.dims
    B = wl.B
    n_c = [n // wd.m for n in wl.n0]
    n_h = [n // wd.m_hca for n in wl.n0]
    ent = torch.empty(sum(n_c), wd.d, dtype=torch.bfloat16, device="cuda")
    hca = torch.empty(sum(n_h), wd.d, dtype=torch.bfloat16, device="cuda")
    raw = torch.empty(B * wd.W, wd.d, dtype=torch.bfloat16, device="cuda")
    rows = []
    oc = oh = 0
    for b in range(B):
        synth.dev_fill("bf16_normal", wl.seed, synth.X, b, wd.d, 0, n_c[b], ent[oc].data_ptr(), scale=0.5)
        synth.dev_fill("bf16_normal", wl.seed, synth.B, b, wd.d, 0, n_h[b], hca[oh].data_ptr(), scale=0.5)
        synth.dev_fill("bf16_normal", wl.seed, synth.A, b, wd.d, 0, wd.W, raw[b * wd.W].data_ptr())
        # raw rows of sequence b are stored so that its last W tokens land at raw[b*W : (b+1)*W]
        rows.append([b * wd.W - (wl.n0[b] - wd.W), oc, oh, wl.n0[b]])
        oc += n_c[b]
        oh += n_h[b]
    seqs = torch.tensor(rows, dtype=torch.int64, device="cuda")
    qt = torch.tensor([[b, wl.n0[b]] for b in range(B)], dtype=torch.int64, device="cuda")
    q = torch.empty(B, wd.H, wd.d, dtype=torch.bfloat16, device="cuda")
    synth.dev_fill("bf16_normal", wl.seed, synth.Q, 0, wd.H * wd.d, 0, B, q.data_ptr())
    rng = np.random.default_rng(0)
    idx = np.stack([np.sort(rng.choice(n_c[b], size=min(wd.k, n_c[b]), replace=False)) for b in range(B)])
    idx = torch.from_numpy(idx.astype(np.int32)).cuda()
    out = torch.empty(B, wd.H, wd.d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, wd.H, dtype=torch.float32, device="cuda")
    dims = dims_of(wd)
    wq = csa.csa_ws_query()
    wq.dims, wq.Q, wq.max_len = dims, B, max(wl.n0)
    wq0 = csa.csa_ws_query()  # the HCA call below runs without the window
    wq0.dims, wq0.Q, wq0.max_len = dims_of(wd), B, max(wl.n0)
    wq0.dims.W = 0
    ws = torch.empty(max(csa.csa_workspace_size(csa.CSA_OP_SPARSE_ATTN, wq),
                         csa.csa_workspace_size(csa.CSA_OP_HCA_ATTN, wq0)), dtype=torch.uint8, device="cuda")
    scale = wd.d ** -0.5
    res = {"stage": "attention", "workload": wl.name}
    for name, fn, nbytes in (
            ("sparse", lambda: csa.csa_sparse_attn(dims, seqs, qt, B, q, ent, idx, raw, scale, out, lse, ws),
             B * (wd.k + wd.W) * wd.d * 2),
            ("hca", lambda: csa.hca_dense_attn(dims, seqs, qt, B, max(wl.n0), q, hca, raw, 0, scale, out, lse, ws),
             sum(n_h) * wd.d * 2)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms_per_call": ms, "key_bytes": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9}
    assert csa.csa_sync_status() == csa.CSA_OK
    return res


def main():
    args = parse()
    if args.stage == "attn":
        print(json.dumps(run_stage_attn(args)), flush=True)
        return
    if args.stage == "index":
        print(json.dumps(run_stage_index(args)), flush=True)
        return
    if args.stage == "compress":
        print(json.dumps(run_stage_compress(args)), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_prefill(args, rank, world) if args.config == "prefill" else run_ours(args, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
