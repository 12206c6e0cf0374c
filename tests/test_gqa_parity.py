"""Grouped-query and multi-query attention (fa_fwd_gqa, fa_bwd_gqa) against the
fp64 oracle: forward O/LSE tolerances as fa_fwd, gradients relative L2 <= 2e-2."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu


def _rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


@pytest.mark.parametrize("B,H,Hkv,N,d,causal", [(1, 4, 1, 300, 128, True), (2, 8, 2, 257, 64, False),
                                                (1, 6, 3, 640, 128, True), (1, 4, 4, 129, 64, True),
                                                (1, 16, 2, 1000, 128, False)])
def test_gqa_forward_and_backward(B, H, Hkv, N, d, causal):
    from exact_io_aware_85_b200 import fa
    x = synth.make_inputs(B, H, N, d, "bf16", seed=900 + H + N, with_grad=True)
    xk, xv = x["k"][:, :Hkv], x["v"][:, :Hkv]
    q, do = to_dev(x["q"], "bf16"), to_dev(x["do"], "bf16")
    k, v = to_dev(np.ascontiguousarray(xk), "bf16"), to_dev(np.ascontiguousarray(xv), "bf16")
    scale = 1 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_gqa(q, k, v, o, lse, causal, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd_gqa(q, k, v, o, do, lse, dq, dk, dv, causal, scale, ws)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o_ref, lse_ref = oracle.attn_fwd_gqa(x["q"], xk, xv, causal, scale)
    assert np.abs(o.float().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - lse_ref).max() <= 1e-3
    g_ref = oracle.attn_bwd_gqa(x["q"], xk, xv, x["do"], causal, scale)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        assert _rel_l2(g.float().cpu().numpy().astype(np.float64), r) <= 2e-2, name


def test_gqa_rejects_bad_group():
    from exact_io_aware_85_b200 import fa
    q = torch.zeros((1, 6, 64, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 4, 64, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 6, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_fwd_gqa(q, k, k, o, lse, False, 0.125)
