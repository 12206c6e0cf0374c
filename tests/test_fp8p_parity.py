"""FP8 P-cast forward (fa_fwd_fp8p) against the E4M3 emulation oracle and the
page's closed form ("P-Cast precision in FP8 attention", sections 2-4)."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu
D4 = oracle.expected_max_normal(4)


def _close_up_to_code_flips(o, o_em):
    """The GPU scores are fp32 (tensor-core accumulation, ex2.approx) and the
    emulation's are fp64, so a P that sits on an E4M3 rounding boundary may take
    the neighbouring code on one side: with a 3-bit mantissa one code step is
    6-12% of that P, which moves the few rows it dominates by up to ~0.05.
    Everything else must agree to the bf16 output resolution."""
    diff = np.abs(o - o_em)
    assert (diff > 1e-2).mean() <= 1e-3
    assert diff.max() <= 0.1


def _run(x, B, H, N, d, causal, S, order, n_sink=4):
    from exact_io_aware_85_b200 import fa
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    stats = torch.zeros(4, dtype=torch.int64, device="cuda")
    fa.fa_fwd_fp8p(q, k, v, o, lse, causal, 1.0 / math.sqrt(d), S, order, stats, n_sink)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), stats.cpu().numpy()


@pytest.mark.parametrize("delta,S,order", [(0.0, 256.0, 0), (7.0, 1.0, 0), (10.0, 256.0, 0), (12.0, 256.0, 1),
                                           (8.0, 448.0, 0), (6.0, 1.0, 1)])
def test_fp8p_matches_emulation(delta, S, order):
    B, H, N, d = 1, 2, 1000, 128
    x = synth.make_sink_inputs(B, H, N, d, delta, seed=31)
    o, lse, st = _run(x, B, H, N, d, False, S, order)
    o_em, lse_em, c_em = oracle.attn_fwd_fp8p(x["q"], x["k"], x["v"], False, 1 / math.sqrt(d), S, order, 128, 4)
    o_ex, lse_ex = oracle.attn_fwd(x["q"], x["k"], x["v"], False, 1 / math.sqrt(d))
    # totals are exact counts; flushes may differ only on E4M3 rounding boundaries
    assert st[1] == c_em[1] and st[3] == c_em[3]
    for a, b in ((st[0], c_em[0]), (st[2], c_em[2])):
        assert abs(int(a) - int(b)) <= max(2, 1e-3 * max(int(b), 1))
    assert np.abs(lse - lse_ex).max() <= 1e-3
    mse_gpu = ((o - o_ex) ** 2).mean()
    mse_em = ((o_em - o_ex) ** 2).mean()
    assert abs(mse_gpu - mse_em) <= 0.1 * mse_em + 1e-7
    _close_up_to_code_flips(o, o_em)


@pytest.mark.parametrize("causal", [True, False])
def test_fp8p_causal_and_ragged(causal):
    B, H, N, d = 2, 1, 333, 64
    x = synth.make_inputs(B, H, N, d, "bf16", seed=41)
    for order in (0, 1):
        o, lse, st = _run(x, B, H, N, d, causal, 256.0, order, n_sink=3)
        o_em, _, c_em = oracle.attn_fwd_fp8p(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d), 256.0, order, 128, 3)
        _, lse_ex = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d))
        assert st[1] == c_em[1] and st[3] == c_em[3]
        assert abs(int(st[2]) - int(c_em[2])) <= 2
        _close_up_to_code_flips(o, o_em)
        assert np.abs(lse - lse_ex).max() <= 1e-3


def test_sink_workload_full_size_against_closed_form():
    """Full sink workload (B=1 H=32 N=16384 d=128): non-sink flush fraction under
    forward order tracks F(Delta, 256); reverse order flushes only inside the sink
    tile (predicted F * 124 / (N - 4))."""
    w = synth.WORKLOADS["sink"]
    for delta in (8.0, 10.0, 12.0):
        x = synth.make_sink_inputs(w.B, w.H, w.N, w.d, delta, seed=synth.workload_seed("sink"))
        _, _, st_f = _run(x, w.B, w.H, w.N, w.d, False, 256.0, 0)
        _, _, st_r = _run(x, w.B, w.H, w.N, w.d, False, 256.0, 1)
        F = oracle.p_collapse_fraction(delta, 256.0, D4)
        frac_f = st_f[2] / st_f[3]
        frac_r = st_r[2] / st_r[3]
        assert abs(frac_f - F) < 0.06, (delta, frac_f, F)
        assert frac_r <= 1.5 * max(frac_f, 1e-9) * 124 / (w.N - 4) + 1e-6, (delta, frac_r)


@pytest.mark.parametrize("N,causal,delta,S,order", [(1000, False, 10.0, 256.0, 0), (1000, False, 7.0, 1.0, 1),
                                                    (777, True, 8.0, 256.0, 1), (513, True, 0.0, 448.0, 0),
                                                    (64, False, 12.0, 256.0, 1)])
def test_fp8p_head_dim_256(N, causal, delta, S, order):
    """d = 256: the P-cast on 64-key tiles (the emulation with B_c = 64), both key
    orders; reverse order with the causal mask meets tiles wholly past a row's
    diagonal before any admissible key."""
    B, H, d = 1, 2, 256
    x = synth.make_sink_inputs(B, H, N, d, delta, seed=33 + N)
    o, lse, st = _run(x, B, H, N, d, causal, S, order)
    o_em, lse_em, c_em = oracle.attn_fwd_fp8p(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d), S, order, 64, 4)
    o_ex, lse_ex = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d))
    assert st[1] == c_em[1] and st[3] == c_em[3]
    for a, b in ((st[0], c_em[0]), (st[2], c_em[2])):
        assert abs(int(a) - int(b)) <= max(2, 1e-3 * max(int(b), 1))
    assert np.isfinite(o).all() and np.abs(lse - lse_ex).max() <= 1e-3
    mse_gpu = ((o - o_ex) ** 2).mean()
    mse_em = ((o_em - o_ex) ** 2).mean()
    assert abs(mse_gpu - mse_em) <= 0.1 * mse_em + 1e-7
    _close_up_to_code_flips(o, o_em)
