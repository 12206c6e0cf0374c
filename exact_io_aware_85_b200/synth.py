"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and rounds them to the storage type; it holds
none of the attention arithmetic, and both the CUDA path and the CPU oracle are
fed from it.  Workload shapes follow the pages' workloads:

* ``tiny``     B=1  H=2  N=256   d=64  fp32, non-causal
* ``day``      B=1  H=12 N=23400 d=64  bf16, causal  (one trading day at 1 s)
* ``prefill``  B=4  H=32 N=8192  d=128 bf16, causal  (LLM prefill)
* ``train``    B=2  H=16 N=4096  d=128 bf16, causal, forward + backward
* ``sink``     B=1  H=32 N=16384 d=128 bf16, non-causal, attention sinks for the
  E4M3 P-cast study (4 sink keys whose logit exceeds the others by Delta)

Values are i.i.d. N(0,1) float32 from numpy's PCG64 with a fixed seed, then
rounded to bfloat16 (round to nearest even) for the bf16 workloads, so the
oracle sees exactly the values the GPU sees.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str  # "bf16", "f32", or "fp8" (bf16 inputs quantised to E4M3)
    causal: bool
    backward: bool = False
    sink: bool = False
    hkv: int = 0  # key/value heads for grouped-query attention (0: same as H)
    decode: bool = False  # one query row per head against an N-key cache
    variant: str = ""  # sink workload: "" (P-cast with flush counts), "nostats", "bf16" (no cast)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """4 B H N^2 d for the two matmuls, halved when causal (N^2/2 convention);
        4 B H N d for a decoding step (one query row per head)."""
        if self.decode:
            return 4.0 * self.B * self.H * self.N * self.d
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    def bwd_flops(self) -> float:
        """Five matmuls of the same size: 2.5x the forward count."""
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, "f32", False),
    "day": Workload("day", 1, 12, 23400, 64, "bf16", True),
    "prefill": Workload("prefill", 4, 32, 8192, 128, "bf16", True),
    "train": Workload("train", 2, 16, 4096, 128, "bf16", True, backward=True),
    "sink": Workload("sink", 1, 32, 16384, 128, "bf16", False, sink=True),
    # the prefill shape on E4M3 operands (full FP8 forward with incoherent processing)
    "prefill_fp8": Workload("prefill_fp8", 4, 32, 8192, 128, "fp8", True),
    # the prefill shape with 8 key/value heads shared by groups of 4 query heads
    "prefill_gqa": Workload("prefill_gqa", 4, 32, 8192, 128, "bf16", True, hkv=8),
    # head dim 256 at the prefill scale (the same FLOPs as the d=128 prefill)
    "prefill_d256": Workload("prefill_d256", 4, 16, 8192, 256, "bf16", True),
    # one decoding step of 8 sequences against a 32K-token key/value cache, 8 KV heads
    "decode": Workload("decode", 8, 32, 32768, 128, "bf16", False, hkv=8, decode=True),
    # a training step at head dim 256 (forward + backward), 8192 tokens
    "train_d256": Workload("train_d256", 2, 8, 8192, 256, "bf16", True, backward=True),
    # the decoding step of "decode" at head dim 256
    "decode_d256": Workload("decode_d256", 8, 32, 32768, 256, "bf16", False, hkv=8, decode=True),
    # the sink workload's P-cast without the flush counting, and the same inputs through the plain
    # bf16 forward: together they split the P-cast's cost into the cast and the counting
    "sink_nostats": Workload("sink_nostats", 1, 32, 16384, 128, "bf16", False, sink=True, variant="nostats"),
    "sink_bf16": Workload("sink_bf16", 1, 32, 16384, 128, "bf16", False, sink=True, variant="bf16"),
}

SINK_DELTAS = (0.0, 2.0, 4.0, 6.0, 7.0, 8.0, 10.0, 12.0)
N_SINK = 4


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    out = (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    # keep NaN payloads NaN (not produced by the generators, but be safe)
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return bf16_round(x) if dtype == "bf16" else x


def make_inputs(B: int, H: int, N: int, d: int, dtype: str = "bf16", seed: int = 0, with_grad: bool = False):
    """Q, K, V (and dO) as float32 arrays [B,H,N,d], bf16-exact when dtype is bf16.
    Draw order: Q, K, V, dO."""
    rng = np.random.default_rng(seed)
    q = normal(rng, (B, H, N, d), dtype)
    k = normal(rng, (B, H, N, d), dtype)
    v = normal(rng, (B, H, N, d), dtype)
    out = {"q": q, "k": k, "v": v}
    if with_grad:
        out["do"] = normal(rng, (B, H, N, d), dtype)
    return out


def make_sink_inputs(B: int, H: int, N: int, d: int, delta: float, seed: int = 0, n_sink: int = N_SINK):
    """Attention-sink inputs for the E4M3 P-cast study.

    Q[..., 0] = 1 and Q[..., 1:] ~ N(0,1); K[..., 1:] ~ N(0,1) * sqrt(d/(d-1));
    K[..., :n_sink, 0] = Delta * sqrt(d) and K[..., n_sink:, 0] = 0, so that with
    scale 1/sqrt(d) the sink logits sit Delta above the others, whose logits are
    approximately N(0,1).  V ~ N(0,1).  All values rounded to bf16.
    """
    rng = np.random.default_rng(seed)
    q = rng.standard_normal(size=(B, H, N, d), dtype=np.float32)
    q[..., 0] = 1.0
    k = rng.standard_normal(size=(B, H, N, d), dtype=np.float32) * np.float32(math.sqrt(d / (d - 1)))
    k[..., 0] = 0.0
    k[..., :n_sink, 0] = np.float32(delta * math.sqrt(d))
    v = rng.standard_normal(size=(B, H, N, d), dtype=np.float32)
    return {"q": bf16_round(q), "k": bf16_round(k), "v": bf16_round(v)}


def make_outlier_inputs(B: int, H: int, N: int, d: int, frac: float = 0.01, mag: float = 10.0, seed: int = 0):
    """Q, K, V ~ N(0,1) with a fraction `frac` of entries replaced by N(0, mag^2)
    outliers (the setting in which block-quantised FP8 attention suffers), bf16."""
    rng = np.random.default_rng(seed)
    out = {}
    for name in ("q", "k", "v"):
        x = rng.standard_normal(size=(B, H, N, d), dtype=np.float32)
        m = rng.random(size=x.shape) < frac
        x[m] = rng.standard_normal(size=int(m.sum()), dtype=np.float32) * np.float32(mag)
        out[name] = bf16_round(x)
    return out


def random_signs(d: int, seed: int = 0) -> np.ndarray:
    """The random +-1 diagonal of the incoherent-processing rotation (float32)."""
    rng = np.random.default_rng(seed)
    return np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)


def workload_seed(name: str) -> int:
    return 1000 + list(WORKLOADS).index(name)
