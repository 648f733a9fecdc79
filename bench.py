"""Benchmark of the QLoRA NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one forward + backward of the seven projections of a
Llama-3.1-8B-shaped block (q, k, v, o: 4096<-4096 / 1024<-4096; gate, up:
14336<-4096; down: 4096<-14336), T = 4096 tokens, LoRA rank 16, s = 2, NF4
weights with double quantization: per projection one qlora_linear_fwd and one
qlora_linear_bwd.  Metric: fwd+bwd TFLOP/s with 4 T N K + 6 T r (N + K) FLOPs
per projection.  Inputs are synthetic (seeded normal draws of the workload's
distributions) and resident in HBM; the step's working set (~0.8 GB) is far
larger than the 126 MB L2, so no flush is needed between steps.

The JSON line also carries: `e2e` (same metric with the step's X and dY copied
from pinned host memory and dA, dB read back, inside the timed region; the
copies run on two copy streams that overlap the projections' compute),
`roofline` of the dominant kernel (CUDA-event durations of every launch in the
timed region, through the library's trace hook), `cpu_baseline` (the CPU
oracle timed on a bounded token sample), `clocks` sampled with nvidia-smi
during the timed region, and `secondary` figures for the decode-sized forward
(T = 1, 4, 16, rank 64) and for quantize/dequantize.

With --gpus N (launched under torchrun) every rank runs an independent replica
of the step (the layer has no cross-GPU exchange); the time is the maximum over
ranks and the value the work of all ranks divided by it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

T_TOKENS, RANK, SCALE = 4096, 16, 2.0
METRIC = "QLoRA NF4 linear fwd+bwd TFLOP/s (8B shapes); decode GB/s; % of roofline"


def proj_shapes():
    from bit_nf4_quantized_20_b200.inputs import LLAMA8B_PROJ
    return LLAMA8B_PROJ


def step_flops(T=T_TOKENS, r=RANK):
    return sum(4.0 * T * n * k + 6.0 * T * r * (n + k) for (_, n, k) in proj_shapes())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi every 10 ms; summary() keeps the samples taken inside the
    window mark_start() .. mark_stop() (all samples if none fell inside)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "10",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        import datetime
        rows = []
        for line in (self.out or "").splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((float(parts[2]), float(parts[3]), float(parts[4]), parts[5:], ts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        window = "timed region"
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if self.t0 <= r[4] <= self.t1]
            if inside:
                rows = inside
            else:
                window = "whole run (no sample fell inside the timed region)"
        sm = [r[0] for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[3][1:]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "window": window,
                "power_w_max": max(r[2] for r in rows)}


def max_over_ranks(ms, dist, device):
    """The slowest rank's time per step (every rank gets it); `ms` unchanged
    on one process.  Works on any backend: the tensor lives on `device`."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_rank_step, ms):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world * flops_per_rank_step / (ms * 1e-3) / 1e12


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def build_layers(device, T, r, config=1):
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    layers = []
    for i, (name, N, K) in enumerate(proj_shapes()):
        W, X, A, B, dY = inputs.layer_inputs(config, 0, i, T, N, K, r, device=device)
        qw = q.quantize_nf4(W)
        del W
        layers.append(dict(name=name, N=N, K=K, qw=qw, X=X, A=A, B=B, dY=dY,
                           U=torch.empty(q.saved_u_bytes(T, r), dtype=torch.uint8, device=device),
                           Y=torch.empty(T, N, dtype=torch.bfloat16, device=device),
                           dX=torch.empty(T, K, dtype=torch.bfloat16, device=device),
                           dA=torch.empty(r, K, dtype=torch.bfloat16, device=device),
                           dB=torch.empty(N, r, dtype=torch.bfloat16, device=device)))
    torch.cuda.synchronize()
    return layers


def run_projection(L, s, saved=True):
    """One projection's forward and backward: the forward saves U = s X A^T for
    the backward (the training path), or the plain pair recomputes it."""
    import bit_nf4_quantized_20_b200 as q
    if saved:
        q.linear_fwd_save(L["X"], L["qw"], L["A"], L["B"], s, out=L["Y"], u_save=L["U"])
        q.linear_bwd_saved(L["dY"], L["X"], L["qw"], L["A"], L["B"], s, L["U"], outs=(L["dX"], L["dA"], L["dB"]))
    else:
        q.linear_fwd(L["X"], L["qw"], L["A"], L["B"], s, out=L["Y"])
        q.linear_bwd(L["dY"], L["X"], L["qw"], L["A"], L["B"], s, outs=(L["dX"], L["dA"], L["dB"]))


def run_step(layers, s, saved=True):
    for L in layers:
        run_projection(L, s, saved)


class Tracer:
    """Per-launch CUDA events through qlora_trace_attach."""

    def __init__(self, capacity):
        import ctypes as C
        import torch
        from bit_nf4_quantized_20_b200 import _lib
        self.C, self.torch, self._lib = C, torch, _lib
        self.recs = (_lib.TraceRec * capacity)()
        self.count = C.c_int32(0)
        self.events = []
        for i in range(capacity):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()      # torch creates the CUDA event on first record
            b.record()
            self.events.append((a, b))
            self.recs[i].start = C.c_void_p(a.cuda_event)
            self.recs[i].stop = C.c_void_p(b.cuda_event)
        self.capacity = capacity

    def __enter__(self):
        self._lib.check("qlora_trace_attach", self._lib.lib().qlora_trace_attach(
            self.recs, self.capacity, self.C.byref(self.count)))
        return self

    def __exit__(self, *a):
        self._lib.lib().qlora_trace_attach(None, 0, None)

    def per_kernel(self):
        lib = self._lib.lib()
        n = min(self.count.value, self.capacity)
        out = {}
        for i in range(n):
            rec = self.recs[i]
            a, b = self.events[i]
            ms = a.elapsed_time(b)
            name = lib.qlora_kernel_name(rec.kernel).decode()
            d = out.setdefault(name, {"launches": 0, "ms": 0.0, "flops": 0.0, "bytes": 0.0})
            d["launches"] += 1
            d["ms"] += ms
            d["flops"] += rec.flops
            d["bytes"] += rec.bytes
        return out


def bench_ours(args, rank, world, local_rank):
    import torch
    import bit_nf4_quantized_20_b200 as q
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    T, r, s = T_TOKENS, RANK, SCALE
    layers = build_layers(dev, T, r)
    launches_per_step = 7 * 7
    tracer = Tracer(args.steps * launches_per_step + 64)
    # clocks are sampled from the start of the warm-up through the timed region
    with ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0) as clk:
        for _ in range(args.warmup):
            run_step(layers, s, args.path == "saved")
        q.get_error(dev)
        torch.cuda.synchronize()
        # ---- device-resident timed region ----
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clk.mark_start()
        start.record()
        for _ in range(args.steps):
            run_step(layers, s, args.path == "saved")
        stop.record()
        torch.cuda.synchronize()
        clk.mark_stop()
    q.get_error(dev)
    ms = start.elapsed_time(stop) / args.steps
    # per-kernel breakdown: the same steps again with an event pair around every
    # launch (outside the timed region: the events serialise the launches, so
    # no kernel starts early and the backward's dB/dA grid runs after the dX
    # GEMM instead of in its last round; every pair of events times one launch)
    with tracer:
        for _ in range(args.steps):
            run_step(layers, s, args.path == "saved")
    torch.cuda.synchronize()
    q.get_error(dev)
    ms = max_over_ranks(ms, dist, dev)
    if dist:
        dist.barrier()
    flops = step_flops(T, r)
    value = aggregate_tflops(world, flops, ms)
    kern = tracer.per_kernel()
    gpu_launches = int(tracer.count.value)

    # ---- end-to-end: host inputs in, adapter gradients out ----
    e2e = bench_e2e(args, layers, dev, s, world, dist)
    clocks = clk.summary()

    result = None
    if rank == 0:
        peaks, peak_src = measured_peaks()
        # a kernel timed alone, or a short timed region at full clock without the
        # power cap, is compared with the burst GEMM figure; a long run that hit
        # the power cap with the sustained one
        timed_s = ms * args.steps * 1e-3
        capped = "sw_power_cap" in (clocks.get("reasons") or [])
        step_key = "bf16_tflops_sustained" if (capped or timed_s > 1.0) else "bf16_tflops"
        step_peak = float(peaks.get(step_key, peaks.get("bf16_tflops")))
        dom_name = max(kern, key=lambda k: kern[k]["ms"]) if kern else None
        roof = None
        if dom_name:
            d = kern[dom_name]
            avg_ms = d["ms"] / d["launches"]
            if d["flops"] > 0:
                ach = (d["flops"] / d["launches"]) / (avg_ms * 1e-3) / 1e12
                peak = float(peaks["bf16_tflops"])
                roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s",
                        "frac": round(ach / peak, 4), "traffic": profile_traffic(dom_name),
                        "kernel": dom_name, "peak_source": f"{peak_src} bf16_tflops (burst: the kernel is "
                        "timed alone, launch by launch)",
                        "launches": d["launches"], "avg_launch_ms": round(avg_ms, 4),
                        "step_achieved": round(value / world, 1), "step_peak": step_peak,
                        "step_frac": round(value / world / step_peak, 4),
                        "step_peak_source": f"{peak_src} {step_key} (timed region {timed_s:.2f} s, "
                                            f"median SM clock {clocks.get('sm_mhz')} MHz)"}
            else:
                ach = (d["bytes"] / d["launches"]) / (avg_ms * 1e-3) / 1e9
                peak = float(peaks["hbm_gbs"])
                roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                        "frac": round(ach / peak, 4), "traffic": profile_traffic(dom_name), "kernel": dom_name,
                        "peak_source": f"{peak_src} hbm_gbs"}
        kernels = {k: {"launches": v["launches"], "ms_per_step": round(v["ms"] / args.steps, 4),
                       "share": round(v["ms"] / sum(x["ms"] for x in kern.values()), 4),
                       "tflops": round(v["flops"] / (v["ms"] * 1e-3) / 1e12, 1) if v["flops"] else None}
                   for k, v in sorted(kern.items(), key=lambda kv: -kv[1]["ms"])}
        secondary = None
        if not args.no_secondary:
            secondary = bench_secondary(dev, peaks)
            secondary["stack_8b_32_layers"] = bench_stack_8b(dev, peaks)
            secondary["codebook_tables"] = bench_tables(dev)
            secondary["adam_step"] = bench_adam(dev, peaks)
            if not args.no_65b:
                secondary["stack_65b_80_layers"] = bench_stack_65b(dev, peaks)
        cpu = None if args.no_cpu else cpu_baseline(args)
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal draws: W~N(0,0.02^2), X,dY~N(0,1), A~N(0,1/K), B~N(0,0.01^2))",
            "config": {"workload": "llama3.1-8b block, 7 NF4+DQ projections, fwd+bwd", "global_batch": world * T,
                       "path": ("forward saves U = s X A^T, backward reuses it" if args.path == "saved"
                                else "plain forward and backward (U recomputed)"),
                       "seq_len": T, "tokens_per_gpu": T, "lora_rank": r, "lora_scale": s,
                       "flops_per_step_per_gpu": flops, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (0.8 GB working set per step), no flush"},
            "e2e": e2e, "gpu_launches": gpu_launches, "roofline": roof, "kernels": kernels,
            "cpu_baseline": cpu, "clocks": clocks, "secondary": secondary,
        }
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return result


def bench_e2e(args, layers, dev, s, world, dist):
    import torch
    import bit_nf4_quantized_20_b200 as q
    host = []
    for L in layers:
        host.append((L["X"].cpu().pin_memory(), L["dY"].cpu().pin_memory(),
                     torch.empty_like(L["dA"], device="cpu").pin_memory(),
                     torch.empty_like(L["dB"], device="cpu").pin_memory()))
    h2d = sum(h[0].numel() * 2 + h[1].numel() * 2 for h in host)
    d2h = sum(h[2].numel() * 2 + h[3].numel() * 2 for h in host)

    # The copies run on their own streams so that they overlap the projections'
    # compute: the inputs of projection p+1 cross PCIe while p computes, and dA,
    # dB go back on a second copy stream.  Every copy of the step is still
    # inside the timed region: both copy streams join the compute stream at the
    # end of the step, and a projection's buffers are refilled for the next
    # step only after that projection's compute has consumed them.
    compute = torch.cuda.current_stream(dev)
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(layers)
    ev_in = [torch.cuda.Event() for _ in range(n)]     # inputs of p landed
    ev_done = [torch.cuda.Event() for _ in range(n)]   # p's compute finished
    for e in ev_done:
        e.record(compute)

    def e2e_step():
        with torch.cuda.stream(h2d_s):
            for i, (L, (hx, hdy, _, _)) in enumerate(zip(layers, host)):
                h2d_s.wait_event(ev_done[i])
                L["X"].copy_(hx, non_blocking=True)
                L["dY"].copy_(hdy, non_blocking=True)
                ev_in[i].record(h2d_s)
        for i, (L, (_, _, hda, hdb)) in enumerate(zip(layers, host)):
            compute.wait_event(ev_in[i])
            run_projection(L, s, args.path == "saved")
            ev_done[i].record(compute)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[i])
                hda.copy_(L["dA"], non_blocking=True)
                hdb.copy_(L["dB"], non_blocking=True)
        compute.wait_stream(h2d_s)
        compute.wait_stream(d2h_s)

    steps = max(1, min(args.steps, 5))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    h2d_s.wait_stream(compute)   # no copy of the timed steps starts before `a`
    for _ in range(steps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, dist, dev)
    v = aggregate_tflops(world, step_flops(), ms)
    return {"value": round(v, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms, 3), "steps": steps}


def profile_traffic(kernel_name):
    """DRAM bytes per launch from a committed ncu summary of this exact kernel
    source (profiles/traffic.json), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        ent = d.get(kernel_name)
        if not ent:
            return None
        import hashlib
        src = os.path.join(ROOT, "bit_nf4_quantized_20_b200", "csrc", ent["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return ent["bytes_per_launch"] if h == ent["source_sha"] else None
    except Exception:
        return None


def bench_secondary(dev, peaks):
    """Decode-sized forward sweep (T = 1, 4, 16; rank 64; s = 1) over the seven
    8B shapes, and quantize/dequantize of the 14336 x 4096 gate weight."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    out = {}
    r = 64
    shapes = proj_shapes()
    qws, adapters = [], []
    for i, (_, N, K) in enumerate(shapes):
        W = inputs.normal_bf16((N, K), 0.02, inputs.seed_of(2, 0, i, "W"), dev)
        qws.append(q.quantize_nf4(W))
        del W
        adapters.append((inputs.normal_bf16((r, K), (1.0 / K) ** 0.5, inputs.seed_of(2, 0, i, "A"), dev),
                         inputs.normal_bf16((N, r), 0.01, inputs.seed_of(2, 0, i, "B"), dev)))
    # L2 flush between timed replays: a 256 MB read (a write would leave the
    # 126 MB L2 full of dirty lines that the timed kernels then write back)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        torch.sum(flush, dim=0, dtype=torch.float32, out=flush_sink)

    for T in (1, 4, 16):
        xs = [inputs.normal_bf16((T, K), 1.0, inputs.seed_of(2, T, i, "X"), dev)
              for i, (_, N, K) in enumerate(shapes)]
        ys = [torch.empty(T, N, dtype=torch.bfloat16, device=dev) for (_, N, K) in shapes]
        nbytes = sum(N * K * (0.5 + 1 / 64) + 4 * ((N * K // 64 + 255) // 256) + 2 * r * (N + K) + 2 * T * (N + K)
                     for (_, N, K) in shapes)

        def sweep():
            for i in range(len(shapes)):
                q.linear_fwd(xs[i], qws[i], adapters[i][0], adapters[i][1], 1.0, out=ys[i])

        # the seven-projection sweep is replayed as one CUDA graph (no host launch gaps);
        # the L2 is flushed (256 MB read) before every replay
        sweep()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream(dev)
        s_cap.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s_cap):
            sweep()       # warm the capture stream
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s_cap, capture_error_mode="relaxed"):
                sweep()
        torch.cuda.current_stream(dev).wait_stream(s_cap)
        times = []
        for rep in range(13):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            if rep >= 3:
                times.append(a.elapsed_time(b))
        del g
        ms = statistics.median(times)
        out[f"decode_T{T}_per_call"] = {"us_per_sweep": round(ms * 1e3, 2),
                                        "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                                        "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                        "bytes_per_sweep": int(nbytes), "timing": "CUDA graph of the "
                                        "7-projection sweep as 7 qlora_linear_fwd calls, L2 flushed (256 MB "
                                        "read) before each replay, median of 10"}
        # the same sweep as one grouped call (all seven projections in one U' launch
        # and one GEMV launch)
        batch = q.DecodeBatch([(xs[i], qws[i], adapters[i][0], adapters[i][1], 1.0, ys[i])
                               for i in range(len(shapes))])
        batch()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s_cap):
            batch()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s_cap, capture_error_mode="relaxed"):
                batch()
        torch.cuda.current_stream(dev).wait_stream(s_cap)
        times = []
        for rep in range(13):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            if rep >= 3:
                times.append(a.elapsed_time(b))
        del g
        ms = statistics.median(times)
        out[f"decode_T{T}"] = {"us_per_sweep": round(ms * 1e3, 2),
                                       "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                                       "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                       "bytes_per_sweep": int(nbytes),
                                       "timing": "CUDA graph of one qlora_linear_fwd_decode_batch call over the 7 "
                                                 "projections (one U' launch, one GEMV launch), L2 flushed "
                                                 "(256 MB read) before each replay, median of 10"}
    # quantize / dequantize / rank-16 adapter merge of one gate-shaped weight (58.7 M weights)
    N, K = 14336, 4096
    W = inputs.normal_bf16((N, K), 0.02, 7, dev)
    qw = q.quantize_nf4(W)
    wd = torch.empty_like(W)
    per = 2.0 + 0.5 + 1 / 64
    A = inputs.normal_bf16((16, K), (1.0 / K) ** 0.5, 8, dev)
    B = inputs.normal_bf16((N, 16), 0.01, 9, dev)
    for name, fn in (("quantize", lambda: q.quantize_nf4(W)), ("dequantize", lambda: q.dequantize(qw)),
                     ("merge_adapter", lambda: q.merge_adapter(qw, A, B, 2.0))):
        times = []
        for rep in range(6):
            flush_l2()
            # a ~0.1 ms spin on the GPU, so that the call below is already queued
            # when the start event fires: the events then time device work only
            torch.cuda._sleep(200000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        gbs = N * K * per / (ms * 1e-3) / 1e9
        out[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                     "weights": N * K, "timing": "CUDA events around one call (queued behind a GPU spin, "
                     "so host-side argument handling is not timed), L2 flushed before, median of 4"}
    q.get_error(dev)
    return out


def _timed(fn, stream=None):
    """CUDA-event time of fn() on the current stream, in ms."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def bench_stack_8b(dev, peaks):
    """Every linear weight of a 32-layer Llama-3.1-8B-shaped stack (6.98e9
    parameters, 14 GB of BF16, generated on the device), quantized to NF4 + DQ
    and dequantized back, each as one back-to-back pass over the 224 matrices
    between two CUDA events (the dequantize pass writes over the BF16 input)."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    Ws = [inputs.normal_bf16((N, K), 0.02, inputs.seed_of(3, layer, i, "W"), dev)
          for layer in range(32) for i, (_, N, K) in enumerate(proj_shapes())]
    qws = [q.quantize_nf4(W) for W in Ws]        # warm-up, and the buffers the timed pass refills
    torch.cuda.synchronize()
    n_w = sum(W.numel() for W in Ws)
    n_b = sum(qw.nbytes() for qw in qws)
    tq = _timed(lambda: [q.quantize_nf4_into(W, qw) for W, qw in zip(Ws, qws)])
    td = _timed(lambda: [q.dequantize(qw, out=W) for W, qw in zip(Ws, qws)])
    q.get_error(dev)
    per = 2.0 + 0.5 + 1.0 / 64
    res = {"weights": n_w, "stored_bytes": n_b, "bits_per_param": n_b * 8 / n_w}
    for name, ms in (("quantize", tq), ("dequantize", td)):
        gbs = n_w * per / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    res["timing"] = ("one pass of 224 back-to-back calls between CUDA events, for quantize and for "
                     "dequantize; the stack is resident in HBM (14 GB BF16 + 3.6 GB NF4), far larger than L2")
    del Ws, qws
    torch.cuda.empty_cache()
    return res


def bench_stack_65b(dev, peaks, clocks_fn=None):
    """The 65B-shaped stack layer by layer: 80 layers x 7 projections (hidden
    8192, ffn 22016), NF4 + DQ weights generated and quantized per layer (BF16
    weights never all resident: 33.4 GB of NF4 are), rank-64 adapters, s =
    0.25, fwd+bwd of every projection on 4 x 512 tokens (the saved-U path)."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    T, r, s = 2048, 64, 0.25
    shapes = inputs.LLAMA65B_PROJ
    per_proj = []
    for i, (_, N, K) in enumerate(shapes):
        _, X, _, _, dY = inputs.layer_inputs(4, 0, i, T, N, K, r, device=dev)
        per_proj.append(dict(X=X, dY=dY, U=torch.empty(q.saved_u_bytes(T, r), dtype=torch.uint8, device=dev),
                             Y=torch.empty(T, N, dtype=torch.bfloat16, device=dev),
                             dX=torch.empty(T, K, dtype=torch.bfloat16, device=dev),
                             dA=torch.empty(r, K, dtype=torch.bfloat16, device=dev),
                             dB=torch.empty(N, r, dtype=torch.bfloat16, device=dev)))
    layers = []
    nf4_bytes = 0
    t0 = time.perf_counter()
    for layer in range(80):
        row = []
        for i, (_, N, K) in enumerate(shapes):
            W = inputs.normal_bf16((N, K), 0.02, inputs.seed_of(4, layer, i, "W"), dev)
            qw = q.quantize_nf4(W)
            del W
            A = inputs.normal_bf16((r, K), (1.0 / K) ** 0.5, inputs.seed_of(4, layer, i, "A"), dev)
            B = inputs.normal_bf16((N, r), 0.01, inputs.seed_of(4, layer, i, "B"), dev)
            nf4_bytes += qw.nbytes()
            row.append((qw, A, B))
        layers.append(row)
    torch.cuda.synchronize()
    setup_s = time.perf_counter() - t0

    def run(n_layers):
        for row in layers[:n_layers]:
            for (qw, A, B), P in zip(row, per_proj):
                q.linear_fwd_save(P["X"], qw, A, B, s, out=P["Y"], u_save=P["U"])
                q.linear_bwd_saved(P["dY"], P["X"], qw, A, B, s, P["U"], outs=(P["dX"], P["dA"], P["dB"]))

    run(3)   # warm-up
    torch.cuda.synchronize()
    ms = _timed(lambda: run(80))
    q.get_error(dev)
    flops = 80 * sum(4.0 * T * N * K + 6.0 * T * r * (N + K) for (_, N, K) in shapes)
    tf = flops / (ms * 1e-3) / 1e12
    return {"layers": 80, "tokens": T, "lora_rank": r, "lora_scale": s, "flops": flops, "ms": round(ms, 2),
            "TFLOP/s": round(tf, 1), "frac_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
            "frac_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
            "nf4_bytes_resident": nf4_bytes, "setup_s": round(setup_s, 1),
            "timing": "CUDA events around one pass of the 80 layers after a 3-layer warm-up; weights "
                      "generated and quantized layer by layer before it (not timed)"}


def bench_tables(dev):
    """Round-trip error of each 4-bit table through the GPU path: quantize and
    dequantize a 4096 x 4096 N(0, 0.02^2) weight, RMS of W' - W relative to
    the weights' RMS, with codes snapped against c1 or against the
    double-quantized scale."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    cb = q.nf4_codebook()
    zero = list(cb)
    zero[7] = 0.0
    tables = {"nf4_eq2": cb, "nf4_eq2_zero_level": zero, "int4_uniform": [(i - 8) / 8.0 for i in range(16)],
              "uniform_16": [(2 * i - 15) / 15.0 for i in range(16)]}
    W = inputs.normal_bf16((4096, 4096), 0.02, 12345, dev)
    wf = W.float()
    ref = wf.pow(2).mean().sqrt().item()
    out = {}
    for name, table in tables.items():
        row = {}
        for snap in (False, True):
            wd = q.dequantize(q.quantize_nf4(W, codebook=table, snap_to_dq_scale=snap)).float()
            row["snap_dq_scale" if snap else "snap_c1"] = round((wd - wf).pow(2).mean().sqrt().item() / ref, 5)
        out[name] = row
    q.get_error(dev)
    return {"relative_rms_error": out, "weights": "4096 x 4096 N(0, 0.02^2) BF16, blocks of 64, DQ groups of 256"}


def bench_adam(dev, peaks):
    """The adapters' optimizer step over the 8B stack's 41.9 M rank-16 adapter
    parameters (32 layers x 1,310,720), FP32 state in device memory and in
    unified (paged) memory prefetched to the GPU."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    n = 32 * 1_310_720
    g = inputs.normal_bf16((n,), 0.02, 777, dev)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    res = {"params": n, "bytes_per_param": 28}
    dev_state = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(3)]
    paged = [q.PagedBuffer(n, device=dev) for _ in range(3)]
    for b in paged:
        b.prefetch()
    for name, (p, m, v) in (("device", dev_state), ("paged", paged)):
        for t in range(1, 4):
            q.adam_step(p, m, v, g, out, step=t, lr=1e-4)
        times = [_timed(lambda: q.adam_step(p, m, v, g, out, step=4, lr=1e-4)) for _ in range(5)]
        ms = statistics.median(times)
        gbs = 28.0 * n / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    q.get_error(dev)
    del paged
    return res


# --------------------------------------------------------------------------
# the CPU oracle (reference arm and cpu_baseline)
# --------------------------------------------------------------------------
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def oracle_sample_step(T_sample, r=RANK, s=SCALE, prepared=None):
    """One pass of the CPU oracle over the 8B block at T_sample tokens:
    dequantize each projection's NF4 weight, then fp64 forward and backward."""
    from oracle import oracle as O
    from bit_nf4_quantized_20_b200 import inputs
    if prepared is None:
        prepared = []
        for i, (_, N, K) in enumerate(proj_shapes()):
            W, X, A, B, dY = inputs.layer_inputs(1, 0, i, T_sample, N, K, r, device="cpu")
            codes, scales, c2 = O.quantize_nf4(inputs.bf16_bits(W))
            prepared.append((N, K, codes, scales, c2, inputs.bf16_bits(X), inputs.bf16_bits(A),
                             inputs.bf16_bits(B), inputs.bf16_bits(dY)))
        return prepared
    t0 = time.perf_counter()
    for (N, K, codes, scales, c2, xb, ab, bb, dyb) in prepared:
        wd = O.dequantize_nf4(codes, scales, c2, N, K)
        O.linear_fwd(xb, wd, ab, bb, s)
        O.linear_bwd(dyb, xb, wd, ab, bb, s)
    return time.perf_counter() - t0


def cpu_baseline(args, T_sample=256):
    prepared = oracle_sample_step(T_sample)
    sec = oracle_sample_step(T_sample, prepared=prepared)
    v = step_flops(T_sample) / sec / 1e12
    res = {"value": round(v, 6), "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
           "sample": f"one fwd+bwd pass of all 7 projections at T={T_sample} tokens (of 4096), "
                     f"including the per-step NF4 dequantization; {sec:.1f} s"}
    res["other_legs"] = cpu_other_legs()
    return res


def cpu_other_legs():
    """The oracle on bounded samples of the quantize and decode workloads."""
    from oracle import oracle as O
    from bit_nf4_quantized_20_b200 import inputs
    out = {}
    # quantize + dequantize of one 4096 x 4096 matrix of the 32-layer stack
    N, K = 4096, 4096
    wb = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, inputs.seed_of(3, 0, 0, "W")))
    t0 = time.perf_counter()
    codes, scales, c2 = O.quantize_nf4(wb)
    tq = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.dequantize_nf4(codes, scales, c2, N, K)
    td = time.perf_counter() - t0
    per = 2.0 + 0.5 + 1.0 / 64
    out["quantize"] = {"GB/s": round(N * K * per / tq / 1e9, 3), "s": round(tq, 2),
                       "sample": "one 4096 x 4096 matrix of the 32-layer 8B stack"}
    out["dequantize"] = {"GB/s": round(N * K * per / td / 1e9, 3), "s": round(td, 2), "sample": "same matrix"}
    # decode forward of the q projection at T = 1, rank 64 (dequantization included)
    r = 64
    W, X, A, B, _ = inputs.layer_inputs(2, 0, 0, 1, N, K, r)
    codes, scales, c2 = O.quantize_nf4(inputs.bf16_bits(W))
    xb, ab, bb = inputs.bf16_bits(X), inputs.bf16_bits(A), inputs.bf16_bits(B)
    t0 = time.perf_counter()
    O.linear_fwd(xb, O.dequantize_nf4(codes, scales, c2, N, K), ab, bb, 1.0)
    tf = time.perf_counter() - t0
    nbytes = N * K * (0.5 + 1 / 64) + 4 * ((N * K // 64 + 255) // 256) + 2 * r * (N + K) + 2 * (N + K)
    out["decode_T1"] = {"GB/s": round(nbytes / tf / 1e9, 3), "s": round(tf, 2),
                        "sample": "the q projection (4096 x 4096) at T = 1, rank 64"}
    out["cores"] = oracle_threads()
    return out


def bench_reference(args, rank, world):
    if rank != 0:
        return None
    T_sample = 128
    prepared = oracle_sample_step(T_sample)
    for _ in range(args.warmup):
        pass   # the oracle has no warm-up state; warm-up steps are not repeated
    secs = []
    for _ in range(args.steps):
        secs.append(oracle_sample_step(T_sample, prepared=prepared))
    sec = sum(secs) / len(secs)
    v = step_flops(T_sample) / sec / 1e12
    cores = oracle_threads()
    sample = f"each step: fwd+bwd of all 7 projections at T={T_sample} tokens (of 4096) with NF4 dequantization"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "llama3.1-8b block, 7 NF4+DQ projections, fwd+bwd",
                                            "seq_len": T_TOKENS, "lora_rank": RANK, "lora_scale": SCALE,
                                            "token_sample": T_sample},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_case(a):
    """A small case for profilers: the seeded inputs of one Llama-3.1-8B
    projection (or all seven), quantized once, then `reps` rounds of the
    forward and/or backward (the path --path selects), each timed with CUDA
    events and printed."""
    import torch
    import bit_nf4_quantized_20_b200 as q
    from bit_nf4_quantized_20_b200 import inputs
    names = [p[0] for p in inputs.LLAMA8B_PROJ]
    dev = torch.device("cuda", 0)
    cases = []
    for i in (range(len(names)) if a.proj == "all" else [names.index(a.proj)]):
        _, N, K = inputs.LLAMA8B_PROJ[i]
        W, X, A, B, dY = inputs.layer_inputs(1, 0, i, a.T, N, K, a.r, device=dev)
        qw = q.quantize_nf4(W)
        del W
        L = dict(name=names[i], N=N, K=K, qw=qw, X=X, A=A, B=B, dY=dY,
                 U=torch.empty(q.saved_u_bytes(a.T, a.r), dtype=torch.uint8, device=dev),
                 Y=torch.empty(a.T, N, dtype=torch.bfloat16, device=dev),
                 dX=torch.empty(a.T, K, dtype=torch.bfloat16, device=dev),
                 dA=torch.empty(a.r, K, dtype=torch.bfloat16, device=dev),
                 dB=torch.empty(N, a.r, dtype=torch.bfloat16, device=dev))
        cases.append(L)
    saved = a.path == "saved"
    for rep in range(a.reps):
        for L in cases:
            N, K = L["N"], L["K"]
            for op in (["fwd", "bwd"] if a.op == "both" else [a.op]):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                if op == "fwd":
                    if saved:
                        q.linear_fwd_save(L["X"], L["qw"], L["A"], L["B"], a.s, out=L["Y"], u_save=L["U"])
                    else:
                        q.linear_fwd(L["X"], L["qw"], L["A"], L["B"], a.s, out=L["Y"])
                    fl = 2.0 * a.T * N * K + 2.0 * a.T * a.r * (N + K)
                else:
                    outs = (L["dX"], L["dA"], L["dB"])
                    if saved:
                        q.linear_bwd_saved(L["dY"], L["X"], L["qw"], L["A"], L["B"], a.s, L["U"], outs=outs)
                    else:
                        q.linear_bwd(L["dY"], L["X"], L["qw"], L["A"], L["B"], a.s, outs=outs)
                    fl = 2.0 * a.T * N * K + 4.0 * a.T * a.r * (N + K)
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1)
                print(f"{L['name']} T={a.T} {op} rep {rep}: {ms:.4f} ms  {fl / ms / 1e9:.1f} TFLOP/s", flush=True)
    q.get_error(dev)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-secondary", action="store_true", help="skip the decode and quantize figures")
    ap.add_argument("--no-65b", action="store_true", help="skip the 80-layer 65B-shaped stack")
    ap.add_argument("--path", default="saved", choices=["saved", "plain"],
                    help="saved: the forward saves U for the backward (default); plain: U recomputed")
    ap.add_argument("--profile-case", action="store_true",
                    help="instead of the bench: run one projection (or all) a few times, for profilers")
    ap.add_argument("--proj", default="gate", help="--profile-case: q, k, v, o, gate, up, down or all")
    ap.add_argument("--T", type=int, default=T_TOKENS, help="--profile-case: tokens")
    ap.add_argument("--r", type=int, default=RANK, help="--profile-case: LoRA rank")
    ap.add_argument("--s", type=float, default=SCALE, help="--profile-case: LoRA scale")
    ap.add_argument("--op", default="both", choices=["fwd", "bwd", "both"], help="--profile-case: calls")
    ap.add_argument("--reps", type=int, default=3, help="--profile-case: repetitions")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.profile_case:
        profile_case(args)
        return
    if args.impl == "reference":
        res = bench_reference(args, rank, world)
    else:
        res = bench_ours(args, rank, world, local_rank)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
