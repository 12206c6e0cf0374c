"""Head dim 256 (fa_fwd / fa_fwd_gqa with d = 256) against the fp64 oracle:
O max-abs <= 1e-2, LSE <= 1e-3, on ragged lengths, causal and not, and at the
prefill scale on sampled rows."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Hkv,N,causal", [(1, 2, 2, 300, True), (2, 1, 1, 129, False), (1, 4, 2, 513, True),
                                             (1, 2, 2, 64, False), (1, 1, 1, 1, True), (1, 2, 1, 1000, False)])
def test_d256_forward(B, H, Hkv, N, causal):
    from exact_io_aware_85_b200 import fa
    d = 256
    x = synth.make_inputs(B, H, N, d, "bf16", seed=2000 + N + H)
    xk, xv = np.ascontiguousarray(x["k"][:, :Hkv]), np.ascontiguousarray(x["v"][:, :Hkv])
    q, k, v = to_dev(x["q"], "bf16"), to_dev(xk, "bf16"), to_dev(xv, "bf16")
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    scale = 1 / math.sqrt(d)
    if Hkv == H:
        fa.fa_fwd(q, k, v, o, lse, causal, scale)
    else:
        fa.fa_fwd_gqa(q, k, v, o, lse, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o_ref, lse_ref = oracle.attn_fwd_gqa(x["q"], xk, xv, causal, scale)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3


def test_d256_large_sampled_rows():
    from exact_io_aware_85_b200 import fa
    B, H, N, d = 2, 8, 8192, 256
    x = synth.make_inputs(B, H, N, d, "bf16", seed=2100)
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd(q, k, v, o, lse, True, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    rows = sample_rows(B * H, N, 48, seed=3)
    o_ref, lse_ref = oracle.attn_fwd_rows(x["q"], x["k"], x["v"], rows, True, 1 / math.sqrt(d))
    of = o.float().cpu().numpy().reshape(B * H, N, d)
    lf = lse.cpu().numpy().reshape(B * H, N)
    assert np.abs(of[rows[:, 0], rows[:, 1]] - o_ref).max() <= 1e-2
    assert np.abs(lf[rows[:, 0], rows[:, 1]] - lse_ref).max() <= 1e-3
