#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = one forward pass (fa_fwd) over one batch of synthetic input of the
chosen workload (default: LLM prefill B=4 H=32 N=8192 d=128, bf16, causal).
Prints one JSON line (rank 0).  Timing: CUDA events on the launching stream
around exactly K steps after W warm-up steps, inputs resident in HBM and larger
than L2, SM clocks sampled during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Multi-GPU (launched by torch.distributed.run): every rank runs its own copy of
the workload (weak scaling, no data-path collective); the step time is the max
over ranks of the CUDA-event time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_85_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM traffic per launch of the dominant kernel, from one-pass ncu captures of
# that kernel (dram__bytes_read.sum + dram__bytes_write.sum); reported only while
# the kernel sources still hash to the values they were measured with.
TRAFFIC = {
    "prefill": {"bytes": 807555328 + 253336832, "src": ("fwd.cuh", "sm100.cuh"),
                "sha1": "d17a89c792c0f38b6388ce3907e811ffde3c2927"},
    "decode": {"bytes": 1073828608 + 3488256, "src": ("decode.cuh", "sm100.cuh"),
               "sha1": "725bc8cae726ee0b4c4ac46b4da2a68672b5a5e5"},
}


def _src_hash(files) -> str:
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "exact_io_aware_85_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [s for s in sm if mx is None or s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank scalar (the device step time) over all ranks."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, step_ms_max: float, ws: int) -> float:
    """Whole-job TFLOP/s under weak scaling: every rank does flops_per_rank per
    step and the job's step takes the slowest rank's time."""
    return ws * flops_per_rank / (step_ms_max * 1e-3) / 1e12


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def device_inputs(w: synth.Workload, seed: int):
    """Seeded synthetic inputs generated on the device (N(0,1), bf16)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    q = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(dt)
    k = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(dt)
    v = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(dt)
    return q, k, v


def measure_fp8_peak(n: int = 8192, reps: int = 10):
    """Dense E4M3 GEMM throughput of this GPU: torch._scaled_mm (cuBLASLt) on
    n x n x n E4M3 operands with bf16 output, the best of `reps` CUDA-event
    timed launches after warm-up, the way the bf16 peak is measured (a burst)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(12345)
    a = torch.randn((n, n), generator=g, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn((n, n), generator=g, device="cuda").to(torch.float8_e4m3fn).t()  # column-major operand
    one = torch.ones((), dtype=torch.float32, device="cuda")
    for _ in range(3):
        torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def cpu_baseline(w: synth.Workload, target_s: float = 14.0):
    """The fp64 oracle on the host cores over a bounded sample of query rows of
    the same workload; TFLOP/s of useful attention work."""
    import oracle
    oracle.build()
    x = synth.make_inputs(1, 1, w.N, w.d, w.dtype, seed=synth.workload_seed(w.name))
    rng = np.random.default_rng(0)

    def flops(rows):
        nk = (rows[:, 1] + 1) if w.causal else np.full(len(rows), w.N)
        return float((4.0 * w.d * nk).sum())

    n, dt = 256, 0.0
    while True:  # grow the sample until it takes about target_s of host time
        rows = np.stack([np.zeros(n, dtype=np.int64), rng.integers(0, w.N, n)], axis=1)
        t0 = time.perf_counter()
        oracle.attn_fwd_rows(x["q"], x["k"], x["v"], rows, w.causal, w.scale)
        dt = time.perf_counter() - t0
        if dt >= 0.7 * target_s or n >= 1000000:
            break
        n = int(min(1000000, n * max(2.0, 0.9 * target_s / max(dt, 1e-3))))
    rate = flops(rows) / dt
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} random query rows of one head of the {w.name} workload (N={w.N}, d={w.d}, "
                      f"{'causal' if w.causal else 'full'}), fp64, {dt:.1f} s",
            "seconds": dt}


def run_reference(args, w):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps = []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(w, target_s=max(2.0, 60.0 / (args.warmup + args.steps)))
        if i >= args.warmup:
            steps.append(cb["value"])
    v = statistics.median(steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, ws),
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "attention fwd/bwd TFLOP/s at 1 B200 and % of dense BF16/FP8 tensor peak"


def config_of(w, ws):
    what = ("forward + backward (dQ, dK, dV from the saved LSE)" if w.backward else
            "bf16 forward without the cast (the sink workload's reference cost), sink Delta=8"
            if w.sink and w.variant == "bf16" else
            "FP8 P-cast forward, S=256, forward key order, sink Delta=8, no flush counting"
            if w.sink and w.variant == "nostats" else
            "FP8 P-cast forward, S=256, forward key order, sink Delta=8" if w.sink else
            "E4M3 forward (Hadamard-rotated block-quantised Q/K, per-head V, P-cast S=256)" if w.dtype == "fp8"
            else "forward (O + LSE)")
    hk = f" H_kv={w.hkv}" if w.hkv else ""
    return {"workload": f"{w.name}: B={w.B} H={w.H}{hk} N={w.N} d={w.d} {w.dtype} "
                        f"{'causal' if w.causal else 'non-causal'} {what}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "parallelism": f"replicas x{ws}",
            "l2": "inputs larger than L2 (no flush needed)" if 3 * w.B * w.H * w.N * w.d * 2 > 126e6
            else "L2 flushed between steps"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=list(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    from exact_io_aware_85_b200 import fa

    peaks, peak_src = load_peaks()
    q, k, v = device_inputs(w, seed=synth.workload_seed(w.name) + rank)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    launches_per_step = 1
    # A step is a function of a buffer set (the tensors its copies touch), so that
    # the end-to-end leg can alternate two sets; everything else is shared.
    if w.backward:
        # training step: forward, then backward from the saved LSE (4 launches)
        g = torch.Generator(device="cuda")
        g.manual_seed(synth.workload_seed(w.name) + 7919 + rank)
        do = torch.randn(q.shape, generator=g, device="cuda", dtype=torch.float32).to(q.dtype)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws_buf = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device="cuda")
        launches_per_step = 4
        inputs, outputs = ("q", "k", "v", "do"), ("dq", "dk", "dv", "lse")

        def step(b):
            fa.fa_fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale)
            fa.fa_bwd(b["q"], b["k"], b["v"], b["o"], b["do"], b["lse"], b["dq"], b["dk"], b["dv"], w.causal, w.scale,
                      ws_buf)
    elif w.sink:
        # FP8 P-cast, forward key order, S = 256, on sink inputs with Delta = 8
        k[..., :4, 0] = 8.0 * math.sqrt(w.d)
        k[..., 4:, 0] = 0.0
        q[..., 0] = 1.0
        stats = torch.zeros(4, dtype=torch.int64, device="cuda") if not w.variant else None
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        if w.variant == "bf16":
            def step(b):
                fa.fa_fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale)
        else:
            def step(b):
                fa.fa_fwd_fp8p(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale, 256.0, 0, stats, 4)
    elif w.dtype == "fp8":
        # E4M3 operands prepared once (quantisation with the random-sign Hadamard
        # rotation, outside the timed step); the step is the FP8 attention kernel
        nb = (w.N + 127) // 128
        q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device="cuda") for _ in range(3))
        sq = torch.empty((w.B, w.H, nb), dtype=torch.float32, device="cuda")
        sk = torch.empty_like(sq)
        sv = torch.empty((w.B, w.H), dtype=torch.float32, device="cuda")
        signs = torch.from_numpy(synth.random_signs(w.d, seed=synth.workload_seed(w.name))).cuda()
        fa.fa_fp8_quantize(q, k, v, signs, q8, k8, v8, sq, sk, sv)
        qz0 = torch.cuda.Event(enable_timing=True)
        qz1 = torch.cuda.Event(enable_timing=True)
        qz0.record()
        fa.fa_fp8_quantize(q, k, v, signs, q8, k8, v8, sq, sk, sv)
        qz1.record()
        torch.cuda.synchronize()
        quant_ms = qz0.elapsed_time(qz1)
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        def step(b):
            fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, b["o"], b["lse"], w.causal, w.scale, 256.0, 0)

        def quantize(b):  # end to end: the fresh inputs are quantised inside the step
            fa.fa_fp8_quantize(b["q"], b["k"], b["v"], signs, q8, k8, v8, sq, sk, sv)
    elif w.decode:
        # q, o: one row per head; k, v: the cache of H_kv heads
        q = q[:, :, 0].contiguous()
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H), dtype=torch.float32, device="cuda")
        k = k[:, : w.hkv].contiguous()
        v = v[:, : w.hkv].contiguous()
        ws_dec = torch.empty(fa.fa_decode_workspace_bytes(w.B, w.H, w.hkv, w.N, w.d), dtype=torch.uint8,
                             device="cuda")
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        def step(b):
            fa.fa_decode(b["q"], b["k"], b["v"], b["o"], b["lse"], w.scale, ws_dec)
    elif w.hkv:
        k = k[:, : w.hkv].contiguous()
        v = v[:, : w.hkv].contiguous()
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        def step(b):
            fa.fa_fwd_gqa(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale)
    elif w.dtype == "bf16":
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        def step(b):
            fa.fa_fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale)
    else:
        inputs, outputs = ("q", "k", "v"), ("o", "lse")

        def step(b):
            fa.fa_fwd_f32(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.scale)
    bufs = {"q": q, "k": k, "v": v, "o": o, "lse": lse}
    if w.backward:
        bufs.update(do=do, dq=dq, dk=dk, dv=dv)

    def run():
        step(bufs)
    small = 3 * q.numel() * q.element_size() < 126e6
    flush = torch.empty(int(256e6), dtype=torch.uint8, device="cuda") if small else None

    nvtx = torch.cuda.nvtx  # ranges for an external profiler's timeline: warm-up, timed steps, end-to-end steps
    nvtx.range_push(f"fa_bench:{w.name}:warmup")
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize()
    nvtx.range_pop()
    assert fa.fa_check_status() == 0

    # ---- device-resident timing: per-launch CUDA events on the launch stream ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        nvtx.range_push(f"fa_bench:{w.name}:timed x{args.steps}")
        t_all0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            run()
            ends[i].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
        nvtx.range_pop()
    barrier(ws)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    step_ms_local = sum(launch_ms) / len(launch_ms)
    step_ms = max_over_ranks(step_ms_local, ws)
    assert fa.fa_check_status() == 0
    flops = w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)
    value = job_throughput(flops, step_ms, ws)

    # ---- end to end through the C ABI with pinned host buffers -----------------
    # Every step copies its inputs from pinned host memory, runs, and copies its
    # results back.  Consecutive steps are pipelined over two device buffer sets
    # and three streams (copies in, compute, copies out), so step i+1's inputs
    # travel while step i computes and step i-1's results return; the same steps
    # run back to back on one stream are reported too.
    host_in = {n: bufs[n].cpu().pin_memory() for n in inputs}
    host_out = [{n: torch.empty(bufs[n].shape, dtype=bufs[n].dtype, pin_memory=True) for n in outputs}
                for _ in range(2)]
    sets = [bufs, {n: (torch.empty_like(t) if n in inputs or n in outputs or n == "o" else t) for n, t in bufs.items()}]
    e2e_steps = max(4, min(args.steps, 10))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(n_steps, e_first=None, e_last=None):
        if e_first is not None:
            e_first.record(s_in)
        for i in range(n_steps):
            j = i % 2
            b = sets[j]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_out[j])  # step i-2's results have left this set
                for n in inputs:
                    b[n].copy_(host_in[n], non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if w.dtype == "fp8":
                quantize(b)
            step(b)
            ev_comp[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                for n in outputs:
                    host_out[j][n].copy_(b[n], non_blocking=True)
                ev_out[j].record(s_out)
        if e_last is not None:
            e_last.record(s_out)

    def e2e_sequential_step():
        for n in inputs:
            bufs[n].copy_(host_in[n], non_blocking=True)
        if w.dtype == "fp8":
            quantize(bufs)
        step(bufs)
        for n in outputs:
            host_out[0][n].copy_(bufs[n], non_blocking=True)

    e2e_pipelined(2)
    e2e_sequential_step()
    torch.cuda.synchronize()
    barrier(ws)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    nvtx.range_push(f"fa_bench:{w.name}:e2e x{e2e_steps}")
    e2e_pipelined(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    nvtx.range_pop()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        e2e_sequential_step()
    s1.record(stream)
    torch.cuda.synchronize()
    seq_ms = max_over_ranks(s0.elapsed_time(s1) / e2e_steps, ws)
    h2d = sum(bufs[n].numel() * bufs[n].element_size() for n in inputs)
    d2h = sum(bufs[n].numel() * bufs[n].element_size() for n in outputs)

    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_note = f"{peak_src} bf16 burst (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback 1590 TFLOP/s"
    fp8_peak = None
    if w.dtype == "fp8":
        # the E4M3 contraction is held against an E4M3 GEMM measured here, now
        fp8_peak = measure_fp8_peak()
        peak = fp8_peak
        peak_note = "E4M3 GEMM burst measured in this run (torch._scaled_mm 8192^3, best of 10)"
    bound, unit, peak_val = "tensor", "TFLOP/s", peak
    if w.decode:
        # bound by reading the key/value cache: roofline in bytes against measured HBM
        bound, unit = "hbm", "GB/s"
        peak_val = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        peak_note = f"{peak_src} HBM copy bandwidth (MEASURED_PEAKS.json)"
    if w.backward:
        kernel_name = "training step: %s + fa_bwd (pre, main, post)" % (
            "fa_fwd256_kernel" if w.d == 256 else "fa_fwd_kernel<bf16,%d>" % w.d)
    elif w.sink:
        kernel_name = ("fa_fwd_kernel<bf16,%d> (no cast)" % w.d if w.variant == "bf16" else
                       "fa_fwd_kernel<bf16,%d,FP8P%s>" % (w.d, "" if w.variant else ",COUNT"))
    elif w.dtype == "fp8":
        kernel_name = "fa_fwd_kernel<e4m3,%d> (kind::f8f6f4)" % w.d
    elif w.decode:
        kernel_name = "fa_decode_split_kernel<%d> + fa_decode_combine_kernel<%d>" % (w.d, w.d)
    elif w.hkv:
        kernel_name = "fa_fwd_kernel<bf16,%d> grouped-query (%d query heads per key/value head)" % (w.d, w.H // w.hkv)
    elif w.d == 256:
        kernel_name = "fa_fwd256_kernel (one Q tile per CTA, double-buffered S)"
    else:
        kernel_name = "fa_fwd_kernel<%s,%d>" % ("bf16" if w.dtype == "bf16" else "f32/tf32", w.d)
    achieved = flops / (step_ms_local * 1e-3) / 1e12
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    hbm = None
    if w.name == "tiny":
        # short sequence: the algorithmic bytes (Q, K, V read, O and LSE written once) over the launch time
        nbytes = 4 * q.numel() * q.element_size() + lse.numel() * 4
        hbm = {"what": "fa_fwd_f32 launch", "algorithmic_bytes": nbytes,
               "achieved_gbs": nbytes / (step_ms_local * 1e-3) / 1e9,
               "frac_of_measured": nbytes / (step_ms_local * 1e-3) / 1e9 / hbm_peak}
    elif w.backward:
        # the backward alone (pre, main, post), timed after the step: Q, K, V, O, dO read and dQ, dK, dV
        # written once in bf16, LSE read, plus the fp32 dQ accumulator zeroed once and read once
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.steps):
            fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, w.causal, w.scale, ws_buf)
        b1.record(stream)
        torch.cuda.synchronize()
        bwd_ms = b0.elapsed_time(b1) / args.steps
        nbytes = 8 * q.numel() * 2 + lse.numel() * 4 + 2 * q.numel() * 4
        hbm = {"what": "fa_bwd (pre + main + post) alone", "ms": bwd_ms, "algorithmic_bytes": nbytes,
               "achieved_gbs": nbytes / (bwd_ms * 1e-3) / 1e9,
               "frac_of_measured": nbytes / (bwd_ms * 1e-3) / 1e9 / hbm_peak,
               "tflops": w.bwd_flops() / (bwd_ms * 1e-3) / 1e12}
    if w.decode:
        achieved_bytes = (sum(t.numel() * t.element_size() for t in (q, k, v, o)) + lse.numel() * 4) / (
            step_ms_local * 1e-3) / 1e9
    tr = TRAFFIC.get(w.name)
    traffic = tr["bytes"] if tr and tr["sha1"] == _src_hash(tr["src"]) else None
    clocks = clk.summary()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": {"bf16": "bf16", "f32": "f32", "fp8": "e4m3"}[w.dtype], "data": "synthetic",
            "config": config_of(w, ws),
            "tokens_per_s": ws * w.B * w.N / (step_ms * 1e-3),
            "pct_of_peak": {"measured_bf16_burst": achieved / peak,
                            "measured_bf16_sustained": achieved / float(peaks.get("bf16_tflops_sustained", 1390.0)),
                            "datasheet_bf16_2250": achieved / 2250.0},
            "roofline": {"bound": bound, "achieved": achieved_bytes if w.decode else achieved,
                         "peak": peak_val, "unit": unit,
                         "frac": (achieved_bytes if w.decode else achieved) / peak_val, "peak_source": peak_note,
                         "traffic": traffic, "kernel": kernel_name,
                         "launch_ms": {"median": statistics.median(launch_ms), "min": min(launch_ms),
                                       "mean": step_ms_local}},
            "clocks": clocks,
            "e2e": {"value": job_throughput(flops, e2e_ms, ws), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "how": "each step's inputs copied from pinned host memory and its results copied back; "
                           "consecutive steps pipelined over two device buffer sets",
                    "sequential": {"value": job_throughput(flops, seq_ms, ws), "ms_per_step": seq_ms}},
            "gpu_launches": args.steps * launches_per_step,
        }
        if w.dtype == "fp8":
            line["fp8_quantize_ms"] = quant_ms
            line["fp8_peak_tflops"] = fp8_peak
            line["pct_of_peak"]["measured_e4m3_burst"] = achieved / fp8_peak
        if hbm is not None:
            line["hbm"] = hbm
        if ws == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(w)
            cb.pop("seconds", None)
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
