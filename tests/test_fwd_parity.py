"""Forward parity: the CUDA path against the fp64 oracle on the same seeded inputs.
Tolerances: O max-abs-error <= 1e-2 and LSE max-abs-error <= 1e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import sample_rows, to_dev

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _run_fwd(x, B, H, N, d, causal, dtype):
    from exact_io_aware_85_b200 import fa
    q, k, v = (to_dev(x[n], dtype) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    if dtype == "bf16":
        fa.fa_fwd(q, k, v, o, lse, causal, 1.0 / math.sqrt(d))
    else:
        fa.fa_fwd_f32(q, k, v, o, lse, causal, 1.0 / math.sqrt(d))
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


CASES = [
    (1, 2, 1, 64, False), (1, 2, 127, 64, True), (2, 3, 129, 128, True), (1, 2, 300, 128, False),
    (1, 4, 1000, 64, True), (2, 2, 777, 128, False), (1, 1, 513, 128, True), (1, 3, 256, 64, False),
    (1, 2, 1280, 128, True), (3, 1, 255, 64, True),
]


@pytest.mark.parametrize("B,H,N,d,causal", CASES)
def test_fwd_bf16_full_parity(B, H, N, d, causal):
    x = synth.make_inputs(B, H, N, d, "bf16", seed=B * 1000 + N + d)
    o, lse = _run_fwd(x, B, H, N, d, causal, "bf16")
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1.0 / math.sqrt(d))
    assert np.abs(o - o_ref).max() <= O_TOL
    assert np.abs(lse - lse_ref).max() <= LSE_TOL


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 256, 64, False), (1, 1, 300, 64, True), (2, 1, 129, 64, False)])
def test_fwd_f32_tf32_parity(B, H, N, d, causal):
    x = synth.make_inputs(B, H, N, d, "f32", seed=7 + N)
    o, lse = _run_fwd(x, B, H, N, d, causal, "f32")
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1.0 / math.sqrt(d))
    assert np.abs(o - o_ref).max() <= O_TOL
    assert np.abs(lse - lse_ref).max() <= LSE_TOL


def test_tiny_workload_exact_config():
    w = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(w.B, w.H, w.N, w.d, w.dtype, seed=synth.workload_seed("tiny"))
    o, lse = _run_fwd(x, w.B, w.H, w.N, w.d, w.causal, w.dtype)
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], w.causal, w.scale)
    assert np.abs(o - o_ref).max() <= O_TOL
    assert np.abs(lse - lse_ref).max() <= LSE_TOL


@pytest.mark.parametrize("name", ["day", "prefill"])
def test_full_size_sampled_rows(name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w.B, w.H, w.N, w.d, w.dtype, seed=synth.workload_seed(name))
    o, lse = _run_fwd(x, w.B, w.H, w.N, w.d, w.causal, w.dtype)
    rows = sample_rows(w.B * w.H, w.N, 96, seed=1)
    o_ref, lse_ref = oracle.attn_fwd_rows(x["q"], x["k"], x["v"], rows, w.causal, w.scale)
    of = o.reshape(w.B * w.H, w.N, w.d)
    lf = lse.reshape(w.B * w.H, w.N)
    got_o = of[rows[:, 0], rows[:, 1]]
    got_l = lf[rows[:, 0], rows[:, 1]]
    assert np.abs(got_o - o_ref).max() <= O_TOL
    assert np.abs(got_l - lse_ref).max() <= LSE_TOL
    # property that holds at any size: every row is a convex combination of V rows
    assert np.isfinite(o).all() and np.isfinite(lse).all()


@pytest.mark.parametrize("N,d,causal", [(131072, 128, True), (65537, 64, False)])
def test_long_sequence_sampled_rows(N, d, causal):
    """Long sequences (the longest 2^17 tokens; a ragged 2^16 + 1 non-causal at
    d = 64): sampled rows, including the last tile's, against the oracle."""
    B, H = 1, 2
    scale = 1.0 / math.sqrt(d)
    x = synth.make_inputs(B, H, N, d, "bf16", seed=N % 1000 + d)
    o, lse = _run_fwd(x, B, H, N, d, causal, "bf16")
    rows = sample_rows(B * H, N, 48, seed=2)
    o_ref, lse_ref = oracle.attn_fwd_rows(x["q"], x["k"], x["v"], rows, causal, scale)
    of = o.reshape(B * H, N, d)
    lf = lse.reshape(B * H, N)
    assert np.abs(of[rows[:, 0], rows[:, 1]] - o_ref).max() <= O_TOL
    assert np.abs(lf[rows[:, 0], rows[:, 1]] - lse_ref).max() <= LSE_TOL
    assert np.isfinite(o).all() and np.isfinite(lse).all()


def test_deterministic():
    x = synth.make_inputs(1, 4, 1100, 128, "bf16", seed=3)
    a = _run_fwd(x, 1, 4, 1100, 128, True, "bf16")
    b = _run_fwd(x, 1, 4, 1100, 128, True, "bf16")
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
