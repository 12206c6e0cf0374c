#!/usr/bin/env python
"""Fused vs materialised attention across sequence lengths on one B200.

"flash-attention-trading-models", section "Cuando alcanzarlo": above roughly 2K
steps the fused kernel always wins, below roughly 512 it does not matter, and
those thresholds are folklore -- the crossover on one's own model and card is a
short benchmark to run.  This is that benchmark, for the page's trading-model
head shape (d = 64, 12 heads, batch 1, causal) by default:

  fused         fa_fwd (this library): S never leaves the chip
  materialised  S = Q K^T / sqrt(d) written to HBM (cuBLAS through torch), masked
                softmax, then P V: the N x N path the page replaces

Both run in bf16 on the same device-resident inputs; time is the median of
CUDA-event timings over repeats; memory is the peak extra device memory of one
call.  Prints one JSON line per N and a summary line with the crossover.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)


def _time(fn, reps):
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ts.sort()
    return ts[len(ts) // 2]


def _peak_extra(fn):
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    fn()
    torch.cuda.synchronize()
    return torch.cuda.max_memory_allocated() - base


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--lengths", default="128,256,512,1024,2048,4096,8192,16384,23400")
    ap.add_argument("--reps", type=int, default=20)
    args = ap.parse_args()
    from exact_io_aware_85_b200 import fa

    B, H, d, causal = args.B, args.H, args.d, bool(args.causal)
    scale = 1.0 / math.sqrt(d)
    rows = []
    for N in (int(x) for x in args.lengths.split(",")):
        g = torch.Generator(device="cuda")
        g.manual_seed(N)
        q, k, v = (torch.randn((B, H, N, d), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        mask = torch.ones((N, N), dtype=torch.bool, device="cuda").triu(1) if causal else None

        def fused():
            fa.fa_fwd(q, k, v, o, lse, causal, scale)

        def materialised():
            s = torch.matmul(q, k.transpose(-2, -1)) * scale
            if mask is not None:
                s = s.masked_fill(mask, float("-inf"))
            return torch.matmul(torch.softmax(s.float(), dim=-1).to(torch.bfloat16), v)

        t_f = _time(fused, args.reps)
        m_f = _peak_extra(fused)
        s_bytes = B * H * N * N * 2
        try:
            t_m = _time(materialised, max(3, args.reps // 4))
            m_m = _peak_extra(materialised)
        except torch.cuda.OutOfMemoryError:
            t_m, m_m = None, None
        torch.cuda.empty_cache()
        row = {"N": N, "fused_ms": t_f, "materialised_ms": t_m, "speedup": (t_m / t_f) if t_m else None,
               "fused_extra_bytes": m_f, "materialised_extra_bytes": m_m, "score_matrix_bytes_bf16": s_bytes}
        rows.append(row)
        print(json.dumps(row), flush=True)
    cross = next((r["N"] for r in rows if r["speedup"] and r["speedup"] >= 1.0), None)
    print(json.dumps({"summary": "fused vs materialised attention", "B": B, "H": H, "d": d, "causal": causal,
                      "first_N_where_fused_is_faster": cross,
                      "speedup_at_largest_N": rows[-1]["speedup"]}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
