"""Pins for the E4M3 P-cast emulation oracle and the page's closed forms
("P-Cast precision in FP8 attention", sections 2-4)."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from exact_io_aware_85_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pcast_page_numbers.json")))
D4 = oracle.expected_max_normal(4)


def test_expected_max_closed_forms():
    # textbook values: E[max of 1] = 0, of 2 = 1/sqrt(pi), of 3 = 3/(2 sqrt(pi))
    assert abs(oracle.expected_max_normal(1)) < 1e-9
    assert oracle.expected_max_normal(2) == pytest.approx(1 / math.sqrt(math.pi), abs=1e-9)
    assert oracle.expected_max_normal(3) == pytest.approx(3 / (2 * math.sqrt(math.pi)), abs=1e-9)
    assert abs(D4 - GOLD["delta_k4_approx"]["value"]) < GOLD["delta_k4_approx"]["tol"]


def test_threshold_and_onset():
    for S in (1.0, 256.0, 448.0):
        dc = oracle.collapse_threshold(S, D4)
        assert oracle.p_collapse_fraction(dc, S, D4) == pytest.approx(0.5, abs=1e-12)
    # without scaling (S = 1) the collapse switches on around Delta 6-7
    dc1 = oracle.collapse_threshold(1.0, D4)
    assert GOLD["collapse_onset"]["lo"] - 0.5 <= dc1 <= GOLD["collapse_onset"]["hi"]
    assert oracle.p_collapse_fraction(GOLD["collapse_onset"]["lo"] - 2, 1.0, D4) < 0.05
    assert oracle.p_collapse_fraction(GOLD["collapse_onset"]["hi"] + 1, 1.0, D4) > 0.95


def _sink(N, H, delta, seed=5, d=128):
    x = synth.make_sink_inputs(1, H, N, d, delta, seed=seed)
    return x["q"], x["k"], x["v"], 1.0 / math.sqrt(d)


def _count_flushes(q, k, S, order, Bc, n_sink, causal=False):
    """Brute-force count of P values that the E4M3 cast sends to zero, written
    without the oracle: S * exp(s - m) <= 2^-10 (2^-10 itself ties to zero),
    with m the running max including the current tile.  Also returns the count
    of flushed non-sinks outside the tile that holds the sinks."""
    B, H, N, d = q.shape
    q64, k64 = q.astype(np.float64), k.astype(np.float64)
    scale = 1.0 / math.sqrt(d)
    T = (N + Bc - 1) // Bc
    tiles = list(range(T))[::-1] if order else list(range(T))
    out = np.zeros(5, dtype=np.int64)
    for b in range(B):
        for h in range(H):
            s = scale * (q64[b, h] @ k64[b, h].T)
            m = np.full(N, -np.inf)
            for t in tiles:
                j0, j1 = t * Bc, min(N, (t + 1) * Bc)
                st = s[:, j0:j1]
                m = np.maximum(m, st.max(axis=1))
                flushed = S * np.exp(st - m[:, None]) <= 2.0 ** -10
                keys = np.arange(j0, j1)
                sink = keys < n_sink
                out[0] += flushed[:, sink].sum()
                out[1] += sink.sum() * N
                out[2] += flushed[:, ~sink].sum()
                out[3] += (~sink).sum() * N
                if j0 >= Bc:  # tiles other than the first (which holds the sinks)
                    out[4] += flushed[:, ~sink].sum()
    return out


@pytest.mark.parametrize("S,order,delta", [(1.0, 0, 6.0), (256.0, 0, 10.0), (256.0, 1, 12.0), (1.0, 1, 7.0)])
def test_flush_counts_match_bruteforce(S, order, delta):
    q, k, v, scale = _sink(768, 2, delta, d=64)
    _, _, counts = oracle.attn_fwd_fp8p(q, k, v, False, scale, S, order, Bc=128, n_sink=4)
    ref = _count_flushes(q, k, S, order, 128, 4)
    assert counts.tolist() == ref[:4].tolist()
    if order == 1 and S == 256.0:
        # reverse order with S = 256: no non-sink outside the sink tile flushes
        assert ref[4] == 0


def test_exactly_representable_p_gives_exact_attention():
    # K = 0: every score is 0, p = 1, S*p = 256 is an E4M3 value, so the cast is exact
    q, k, v, scale = _sink(300, 1, 0.0, d=64)
    k = np.zeros_like(k)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, False, scale)
    for order in (0, 1):
        o, lse, counts = oracle.attn_fwd_fp8p(q, k, v, False, scale, 256.0, order, Bc=128)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12)
        assert counts[0] == 0 and counts[2] == 0


def test_large_S_limit_reduces_to_exact_attention():
    # causal path of the emulator with a harmless cast: compare at the E4M3 error scale
    x = synth.make_inputs(1, 2, 200, 32, "bf16", seed=9)
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], True, 0.2)
    o, lse, _ = oracle.attn_fwd_fp8p(x["q"], x["k"], x["v"], True, 0.2, 256.0, 0, Bc=64)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)  # l uses the unquantised p
    assert np.abs(o - o_ref).max() < 0.1  # 3-bit mantissa on P: percent-level error


@pytest.fixture(scope="module")
def sweep():
    """Emulation at N=4096 (the page's section-4 length), 2 heads."""
    res = {}
    for delta in (7.0, 10.0, 12.0):
        q, k, v, scale = _sink(4096, 2, delta)
        o_ref, _ = oracle.attn_fwd(q, k, v, False, scale)
        for S, order in ((1.0, 0), (256.0, 0), (448.0, 0), (256.0, 1)):
            o, _, c = oracle.attn_fwd_fp8p(q, k, v, False, scale, S, order)
            res[(delta, S, order)] = (float(((o - o_ref) ** 2).mean()), c[2] / c[3])
    return res


def test_nonsink_flush_fraction_tracks_closed_form(sweep):
    # forward order: emulated fraction of flushed non-sinks vs F(Delta, S)
    for (delta, S, order), (_, frac) in sweep.items():
        if order == 0:
            F = oracle.p_collapse_fraction(delta, S, D4)
            assert abs(frac - F) < 0.06, (delta, S, frac, F)


def test_mse_orderings_from_the_page(sweep):
    mse = {kk: vv[0] for kk, vv in sweep.items()}
    r = mse[(7.0, 1.0, 0)] / mse[(7.0, 256.0, 0)]
    g = GOLD["mse_ratio_fwd_S1_vs_opt_at_delta7"]
    assert g["lo"] <= r <= g["hi"], r
    for delta in (7.0, 10.0, 12.0):
        assert mse[(delta, 448.0, 0)] > mse[(delta, 256.0, 0)]  # S=256 never worse than 448
        assert abs(mse[(delta, 256.0, 1)] / mse[(delta, 256.0, 0)] - 1.0) < 0.1  # reverse ~ forward at S=256


def _ln2_ladder(descending: bool):
    """Logits on a ln 2 ladder: key tile t of 4 keys holds a maximum 2 t ln 2 (or
    2 (T-1-t) ln 2 when descending) and keys 0, 1, 5, 9 ln 2 below it, so
    within a row every score sits a whole number n <= 17 of ln 2 below any
    running maximum it can meet, in either key order and at any causal cut.
    Then S p = 256 * 2^-n is an E4M3 value (2^-9 is the smallest), the cast is
    exact while the maximum keeps moving from tile to tile, and the emulation
    must reproduce exact attention, rescaling of the accumulator included."""
    T, steps = 5, (0, 1, 5, 9)
    ln2 = math.log(2.0)
    logits = []
    for t in range(T):
        top = 2 * (T - 1 - t if descending else t)
        logits += [(top - n) * ln2 for n in steps]
    N = len(logits)
    q = np.zeros((1, 1, N, 3))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, N, 3))
    k[0, 0, :, 0] = logits
    v = np.random.default_rng(3).standard_normal((1, 1, N, 3))
    return q, k, v


@pytest.mark.parametrize("descending", [False, True])
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("causal", [False, True])
def test_grid_exact_p_with_moving_max_gives_exact_attention(descending, order, causal):
    q, k, v = _ln2_ladder(descending)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, 1.0)
    o, lse, counts = oracle.attn_fwd_fp8p(q, k, v, causal, 1.0, 256.0, order, Bc=4, n_sink=0)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)
    assert counts[2] == 0


def test_flushed_p_leave_the_numerator_but_not_the_sum():
    """Scores 19 and 21 ln 2 below their tile's maximum (forward order, maxima
    growing tile by tile): S p = 2^-11 and 2^-13 round to zero, so those keys
    drop out of the numerator of O while their unquantised p stays in the
    denominator l; every other S p is on the E4M3 grid.  (The 2^-10 tie itself
    cannot be reached through exp in fp64, which misses 2^-18 by an ulp; the
    E4M3 tests pin it.)  The expected O is written from that definition."""
    ln2 = math.log(2.0)
    shifts = (0, 3, 19, 21)
    logits = [(2 * t - n) * ln2 for t in range(4) for n in shifts]
    N = len(logits)
    q = np.zeros((1, 1, N, 2))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, N, 2))
    k[0, 0, :, 0] = logits
    v = np.random.default_rng(4).standard_normal((1, 1, N, 2))
    s = np.array(logits)
    e = np.exp(s - s.max())
    kept = np.array([n <= 17 for _ in range(4) for n in shifts])
    o_want = (e[kept, None] * v[0, 0][kept]).sum(axis=0) / e.sum()
    o, lse, counts = oracle.attn_fwd_fp8p(q, k, v, False, 1.0, 256.0, 0, Bc=4, n_sink=0)
    for i in range(N):
        np.testing.assert_allclose(o[0, 0, i], o_want, atol=1e-12, rtol=0)
    assert counts[2] == N * 8 and counts[3] == N * N  # 2 flushed keys per tile, every row
    np.testing.assert_allclose(lse[0, 0], np.log(np.exp(s).sum()), atol=1e-12)
