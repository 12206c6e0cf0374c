"""Pins for the FP8-operand oracle: the incoherent-processing rotation against
scipy's Hadamard matrix, block-scale invariants of the E4M3 quantiser, and the
page's FA3 claim that rotating before block quantisation lowers FP8 attention's
error about 2.6x on inputs with outliers."""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from exact_io_aware_85_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "fa3_page_numbers.json")))


@pytest.mark.parametrize("d", [2, 8, 64, 128])
def test_rotation_is_signed_hadamard(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((5, d))
    s = synth.random_signs(d, seed=d).astype(np.float64)
    ref = x @ np.diag(s) @ scipy.linalg.hadamard(d) / math.sqrt(d)
    np.testing.assert_allclose(oracle.hadamard_rotate(x, s), ref, atol=1e-12)


def test_rotation_preserves_scores():
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal((40, 128)), rng.standard_normal((30, 128))
    s = synth.random_signs(128, seed=3).astype(np.float64)
    qr, kr = oracle.hadamard_rotate(q, s), oracle.hadamard_rotate(k, s)
    np.testing.assert_allclose(qr @ kr.T, q @ k.T, atol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(qr, axis=1), np.linalg.norm(q, axis=1), rtol=1e-12)


@pytest.mark.parametrize("rot", [False, True])
def test_block_quantiser_invariants(rot):
    x = synth.make_outlier_inputs(1, 2, 300, 128, seed=5)["q"].astype(np.float64)
    s = synth.random_signs(128, seed=9) if rot else None
    xq, sc = oracle.fp8_quantize(x, s, block_rows=128)
    xr = oracle.hadamard_rotate(x, s) if rot else x
    assert sc.shape == (1, 2, 3)
    for h in range(2):
        for b in range(3):
            blk = slice(128 * b, min(300, 128 * (b + 1)))
            codes = xq[0, h, blk] / sc[0, h, b]
            amax = np.abs(xr[0, h, blk]).max()
            assert sc[0, h, b] == pytest.approx(amax / 448.0, rel=1e-15)
            assert np.abs(codes).max() == pytest.approx(448.0, rel=1e-12)  # the block max maps to 448
            # E4M3 rounding error: at most half a step (2^-4 relative in the normal range,
            # 2^-10 absolute on the code scale in the subnormal range)
            err = np.abs(codes - xr[0, h, blk] / sc[0, h, b])
            bound = np.maximum(np.abs(xr[0, h, blk] / sc[0, h, b]) * 2.0 ** -4, 2.0 ** -10)
            assert (err <= bound + 1e-12).all()
    # one scale per head when the block covers the sequence
    _, sc1 = oracle.fp8_quantize(x, s, block_rows=300)
    assert sc1.shape == (1, 2, 1)


def _fp8_rms_error(frac, rotate):
    B, H, N, d = 1, 2, 1024, 128
    x = synth.make_outlier_inputs(B, H, N, d, frac=frac, seed=21)
    scale = 1 / math.sqrt(d)
    o_ex, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], False, scale)
    s = synth.random_signs(d, seed=4) if rotate else None
    qq, _ = oracle.fp8_quantize(x["q"], s)
    kq, _ = oracle.fp8_quantize(x["k"], s)
    vq, _ = oracle.fp8_quantize(x["v"], None, block_rows=N)
    o, _, _ = oracle.attn_fwd_fp8p(qq, kq, vq, False, scale, 256.0, 0)
    return float(np.sqrt(((o - o_ex) ** 2).mean()))


def test_incoherent_processing_error_ratio_matches_page():
    ratio = _fp8_rms_error(0.01, False) / _fp8_rms_error(0.01, True)
    assert 2.0 <= ratio <= 3.5, ratio  # page: 2.6x lower error than naive FP8
    assert abs(ratio - GOLD["fp8_incoherent_error_ratio"]["value"]) < 0.6


def test_rotation_neutral_without_outliers():
    ratio = _fp8_rms_error(0.0, False) / _fp8_rms_error(0.0, True)
    assert 0.9 <= ratio <= 1.1
