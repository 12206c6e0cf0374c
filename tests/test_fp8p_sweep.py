"""The FP8 P-cast sweep of the attention-sink workload at its own sequence length
("P-Cast precision in FP8 attention", section 2 "Marco Teorico" for F(Delta, S),
"Optimizacion 1/2" for reverse key order and S = 256, section 4 for the MSE
comparisons).

One head of the sink workload (N = 16384, d = 128, non-causal) for every Delta in
{0, 2, 4, 6, 7, 8, 10, 12} in both key-tile orders at S = 256, and the S = 1 and
S = 448 ablation in forward order at Delta in {7, 10}.  Each case runs
fa_fwd_fp8p once and checks, against the E4M3 emulation oracle on the same
inputs:
  * the whole O element by element (up to E4M3 code flips at rounding
    boundaries, see test_fp8p_parity._close_up_to_code_flips),
  * the MSE against exact attention within 10 % of the emulation's,
  * the flush counts (sink and non-sink) within max(2, 1e-3 of the count),
  * the LSE against exact attention within 1e-3.
Run with ``-s`` to print one markdown row per case: the numbers of the sweep
table (GPU and emulation MSE, flush fractions, the page's mean-field F at the
bf16-rounded Delta and the per-row predictor mean_i Phi(m_i - 10 ln 2 - ln S)).
"""
import functools
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev
from test_fp8p_parity import _close_up_to_code_flips

pytestmark = pytest.mark.gpu

N, D_HEAD = 16384, 128
SCALE = 1.0 / math.sqrt(D_HEAD)
CASES = ([(dl, 256.0, order) for dl in synth.SINK_DELTAS for order in (0, 1)] +
         [(dl, S, 0) for S in (1.0, 448.0) for dl in (7.0, 10.0)])


@functools.lru_cache(maxsize=None)
def _inputs(delta):
    seed = synth.workload_seed("sink") + 10 * synth.SINK_DELTAS.index(delta)
    return synth.make_sink_inputs(1, 1, N, D_HEAD, delta, seed=seed)


@functools.lru_cache(maxsize=None)
def _exact(delta):
    x = _inputs(delta)
    return oracle.attn_fwd(x["q"], x["k"], x["v"], False, SCALE)


@functools.lru_cache(maxsize=None)
def _row_max(delta):
    """m_i = max_j scale <q_i, k_j> over all keys, fp64 (the running max that every
    tile after the sink tile sees in forward order)."""
    x = _inputs(delta)
    q = x["q"][0, 0].astype(np.float64)
    k = x["k"][0, 0].astype(np.float64)
    m = np.empty(N)
    for r0 in range(0, N, 2048):
        m[r0:r0 + 2048] = (q[r0:r0 + 2048] @ k.T).max(axis=1) * SCALE
    return m


def _delta_eff(delta):
    """The sink logits sit bf16(Delta sqrt(d)) / sqrt(d) above the rest."""
    return float(synth.bf16_round(np.array([delta * math.sqrt(D_HEAD)], np.float32))[0]) / math.sqrt(D_HEAD)


def _run_gpu(x, S, order):
    from exact_io_aware_85_b200 import fa
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, N), dtype=torch.float32, device="cuda")
    stats = torch.zeros(4, dtype=torch.int64, device="cuda")
    fa.fa_fwd_fp8p(q, k, v, o, lse, False, SCALE, S, order, stats, synth.N_SINK)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), stats.cpu().numpy()


@pytest.mark.parametrize("delta,S,order", CASES)
def test_sink_sweep_case(delta, S, order):
    x = _inputs(delta)
    o, lse, st = _run_gpu(x, S, order)
    o_em, _, c_em = oracle.attn_fwd_fp8p(x["q"], x["k"], x["v"], False, SCALE, S, order, 128, synth.N_SINK)
    o_ex, lse_ex = _exact(delta)

    assert st[1] == c_em[1] and st[3] == c_em[3]
    for a, b in ((st[0], c_em[0]), (st[2], c_em[2])):
        assert abs(int(a) - int(b)) <= max(2, 1e-3 * int(b)), (st, c_em)
    assert np.abs(lse - lse_ex).max() <= 1e-3
    mse_gpu = float(((o - o_ex) ** 2).mean())
    mse_em = float(((o_em - o_ex) ** 2).mean())
    assert abs(mse_gpu - mse_em) <= 0.1 * mse_em + 1e-7, (mse_gpu, mse_em)
    _close_up_to_code_flips(o, o_em)

    # the sweep table's row: fractions and the page's predictors
    de = _delta_eff(delta)
    F = oracle.p_collapse_fraction(de, S, oracle.expected_max_normal(4))
    per_row = float(np.mean([oracle.normal_cdf(m - oracle.LN_ZERO_THRESHOLD - math.log(S))
                             for m in _row_max(delta)]))
    if order == 1:  # only the 124 non-sinks of the sink tile see the sink max
        F *= 124.0 / (N - 4)
        per_row *= 124.0 / (N - 4)
    print(f"\n| {delta:g} | {de:.3f} | {S:g} | {'reverse' if order else 'forward'} | {mse_gpu:.3e} | {mse_em:.3e} | "
          f"{st[2] / st[3]:.4g} | {c_em[2] / c_em[3]:.4g} | {F:.4g} | {per_row:.4g} | {st[0]}/{st[1]} |")
