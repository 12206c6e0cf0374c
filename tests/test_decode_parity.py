"""Decoding step (fa_decode) against the fp64 oracle: one query row per head
against the whole key/value cache; O max-abs <= 1e-2, LSE <= 1e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Hkv,N,d", [(1, 8, 8, 1000, 128), (2, 32, 8, 4097, 128), (4, 16, 1, 333, 64),
                                         (1, 4, 4, 1, 64), (1, 16, 16, 70000, 128), (3, 12, 4, 65, 64),
                                         (2, 24, 2, 5000, 128), (1, 8, 1, 129, 64),
                                         # head dim 256: the ring holds single K or V tiles
                                         (1, 8, 2, 1000, 256), (2, 16, 1, 4097, 256), (1, 4, 4, 1, 256),
                                         (1, 8, 8, 300, 256), (1, 16, 16, 40000, 256)])
def test_decode_matches_oracle(B, H, Hkv, N, d):
    from exact_io_aware_85_b200 import fa
    rng_seed = 1300 + N + H
    x = synth.make_inputs(B, Hkv, N, d, "bf16", seed=rng_seed)
    qx = synth.make_inputs(B, H, 1, d, "bf16", seed=rng_seed + 1)["q"][:, :, 0]
    q = to_dev(np.ascontiguousarray(qx), "bf16")
    k, v = to_dev(x["k"], "bf16"), to_dev(x["v"], "bf16")
    o = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_workspace_bytes(B, H, Hkv, N, d), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(d)
    fa.fa_decode(q, k, v, o, lse, scale, ws)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o_ref, lse_ref = oracle.attn_decode(qx, x["k"], x["v"], scale)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3


def test_decode_rejects_large_groups():
    from exact_io_aware_85_b200 import fa
    q = torch.zeros((1, 32, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 32), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_decode(q, k, k, o, lse, 0.125, ws)  # 32 query heads per key/value head > 16
