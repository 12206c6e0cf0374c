"""Pins for the oracle's E4M3 rounding: the format decoded from its bit layout
(4 exponent bits with bias 7, 3 mantissa bits, subnormals, 0x7F/0xFF = NaN),
torch's float8_e4m3fn conversion as an independent library routine, and the
numbers the P-cast page prints about the format and about d_p(S)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pcast_page_numbers.json")))


def _grid():
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 0xF, code & 0x7
        if e == 15 and m == 7:
            continue  # NaN
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals.append((-mag if s else mag, m))
    return vals


def test_grid_extremes():
    pos = sorted({v for v, _ in _grid() if v > 0})
    assert pos[0] == 2.0 ** -9  # smallest subnormal
    assert pos[-1] == GOLD["e4m3_max_finite_pow2_scale"]["value"] == 448.0
    assert len(pos) == 126


def test_rounding_is_nearest_even_on_the_grid():
    grid = _grid()
    gv = np.array([v for v, _ in grid])
    gm = np.array([m for _, m in grid])
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.uniform(-448, 448, 4000),
        np.sign(rng.standard_normal(4000)) * 2.0 ** rng.uniform(-14, 9, 4000),
        gv,  # exact grid points
        (np.sort(np.unique(gv))[1:] + np.sort(np.unique(gv))[:-1]) / 2.0,  # exact midpoints
    ])
    x = x[np.abs(x) <= 448.0]
    y = oracle.e4m3(x)
    for xi, yi in zip(x, y):
        dist = np.abs(gv - xi)
        best = dist.min()
        cands = np.unique(gv[dist == best])
        if len(cands) == 1:
            assert yi == cands[0], (xi, yi, cands)
        else:  # tie: the candidate whose mantissa code is even
            even = [c for c in cands if any(gm[(gv == c)] % 2 == 0)]
            assert len(even) == 1 and yi == even[0], (xi, yi, cands)


def test_matches_torch_float8_e4m3fn():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 50, 2.0 ** rng.uniform(-13, 8.8, 20000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.e4m3(x.astype(np.float64)), ref)


def test_page_thresholds():
    thr = GOLD["zero_threshold"]["value"]
    assert oracle.e4m3(thr)[()] == 0.0  # 2^-10 rounds to zero (tie with 2^-9 goes to even = 0)
    assert oracle.e4m3(np.nextafter(thr, 1.0))[()] == 2.0 ** -9
    assert abs(10 * math.log(2) - GOLD["zero_threshold_log"]["value"]) < 0.005
    assert oracle.e4m3(1e6)[()] == 448.0 and oracle.e4m3(-1e6)[()] == -448.0  # satfinite
    assert GOLD["subnormal_coverage_S256"]["value"] == 2.0 ** -6 / 256


def _dp_bruteforce(S):
    pos = np.array(sorted({v for v, _ in _grid() if v > 0}))
    below = pos[pos < S]
    gaps = np.diff(np.concatenate([[0.0], below, pos[pos >= S][:1]]))
    return gaps[-1] / S  # step from the largest value below S up to the next grid value


@pytest.mark.parametrize("S", [1.0, 2.0, 16.0, 64.0, 256.0, 448.0, 100.0, 300.0])
def test_dp_sawtooth_against_grid(S):
    assert oracle.dp_sawtooth(S) == pytest.approx(_dp_bruteforce(S), rel=1e-12)


def test_dp_page_numbers():
    assert oracle.dp_sawtooth(256.0) == GOLD["dp_min"]["value"]
    excess = oracle.dp_sawtooth(448.0) / GOLD["dp_min"]["value"] - 1.0
    assert abs(excess - GOLD["dp_448_excess"]["value"]) < GOLD["dp_448_excess"]["tol"]
    for k in range(0, 9):  # powers of two sit on the lower envelope
        assert oracle.dp_sawtooth(2.0 ** k) == 2.0 ** -4


def test_power_of_two_scale_is_exact_in_fp32():
    rng = np.random.default_rng(2)
    p = rng.uniform(0, 1, 100000).astype(np.float32)
    assert np.array_equal((p * np.float32(256)) / np.float32(256), p)
    # a non power of two is not
    assert not np.array_equal((p * np.float32(448)) / np.float32(448), p)
