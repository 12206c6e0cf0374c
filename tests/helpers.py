"""Shared helpers for the GPU parity tests (inputs from synth, references from oracle)."""
from __future__ import annotations

import numpy as np
import torch

from exact_io_aware_85_b200 import synth


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return (t.to(torch.bfloat16) if dtype == "bf16" else t).cuda()


def sample_rows(BH: int, N: int, n: int, seed: int = 0, tile: int = 128) -> np.ndarray:
    """(bh, row) pairs: the first/last rows of the sequence, rows on both sides of
    tile boundaries, and random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, N - 1, min(N - 1, tile - 1), min(N - 1, tile), N // 2, max(0, N - tile)}
    edge = (N - 1) // tile * tile
    rows |= {edge, max(0, edge - 1)}
    rows |= set(int(x) for x in rng.integers(0, N, size=max(0, n - len(rows))))
    bhs = rng.integers(0, BH, size=len(rows))
    out = np.array([[int(b), int(r)] for b, r in zip(bhs, sorted(rows))], dtype=np.int64)
    out[:4, 0] = [0, BH - 1, 0, BH - 1][: min(4, len(out))]
    return out
