"""Full FP8 forward (fa_fp8_quantize + fa_fwd_fp8) against the oracle: the
quantiser's E4M3 codes and scales, the attention output against the oracle's
emulation of the same pipeline (block quantisation, then the tile-by-tile
E4M3 P-cast), and the page's FA3 claim that incoherent processing lowers the
error of FP8 attention on inputs with outliers."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu


def _gpu_quant(x, signs):
    from exact_io_aware_85_b200 import fa
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    B, H, N, d = q.shape
    nb = (N + 127) // 128
    q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device="cuda") for _ in range(3))
    sq = torch.empty((B, H, nb), dtype=torch.float32, device="cuda")
    sk = torch.empty_like(sq)
    sv = torch.empty((B, H), dtype=torch.float32, device="cuda")
    sg = None if signs is None else torch.from_numpy(signs).cuda()
    fa.fa_fp8_quantize(q, k, v, sg, q8, k8, v8, sq, sk, sv)
    return q8, k8, v8, sq, sk, sv


def _code_values(codes):
    return codes.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


def _one_step_apart(got, ref):
    """Fraction of E4M3 codes that differ, and whether each difference is at most
    one code step (an fp32 vs fp64 rounding decision on a code boundary)."""
    diff = np.abs(got - ref)
    step = np.maximum(np.abs(ref) * 2.0 ** -3, 2.0 ** -9)
    # ref comes from fp64 code * scale / scale: allow its round-trip ulp
    return float((diff > 1e-9 * np.abs(ref)).mean()), bool((diff <= step * 1.0001).all())


@pytest.mark.parametrize("rotate,d", [(False, 128), (True, 128), (True, 64), (True, 256)])
def test_quantiser_matches_oracle(rotate, d):
    B, H, N = 1, 2, 300
    x = synth.make_outlier_inputs(B, H, N, d, seed=61)
    signs = synth.random_signs(d, seed=62) if rotate else None
    q8, k8, v8, sq, sk, sv = _gpu_quant(x, signs)
    torch.cuda.synchronize()
    for name, codes, sc, blk in (("q", q8, sq, 128), ("k", k8, sk, 128), ("v", v8, sv, N)):
        ref, ref_sc = oracle.fp8_quantize(x[name], signs if name != "v" else None, block_rows=blk)
        got_sc = sc.cpu().numpy().astype(np.float64).reshape(ref_sc.shape)
        np.testing.assert_allclose(got_sc, ref_sc, rtol=2e-6)
        sc_rows = np.repeat(ref_sc, blk, axis=2)[:, :, :N, None]
        frac, ok = _one_step_apart(_code_values(codes), ref / sc_rows)
        assert frac <= 1e-3 and ok, (name, frac)


def _fp8_forward(x, signs, causal, order=0):
    from exact_io_aware_85_b200 import fa
    q8, k8, v8, sq, sk, sv = _gpu_quant(x, signs)
    B, H, N, d = q8.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, causal, 1 / math.sqrt(d), 256.0, order)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _oracle_fp8(x, signs, causal, order=0):
    N, d = x["q"].shape[2], x["q"].shape[3]
    qq, _ = oracle.fp8_quantize(x["q"], signs)
    kq, _ = oracle.fp8_quantize(x["k"], signs)
    vq, _ = oracle.fp8_quantize(x["v"], None, block_rows=N)
    return oracle.attn_fwd_fp8p(qq, kq, vq, causal, 1 / math.sqrt(d), 256.0, order)[:2]


@pytest.mark.parametrize("B,H,N,causal,rotate,order", [(1, 2, 1000, False, True, 0), (2, 1, 777, True, True, 1),
                                                        (1, 2, 513, True, False, 0), (1, 1, 128, False, False, 1)])
def test_fp8_forward_matches_emulation(B, H, N, causal, rotate, order):
    d = 128
    x = synth.make_inputs(B, H, N, d, "bf16", seed=70 + N)
    signs = synth.random_signs(d, seed=71) if rotate else None
    o, lse = _fp8_forward(x, signs, causal, order)
    o_em, lse_em = _oracle_fp8(x, signs, causal, order)
    o_ex, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d))
    # the LSE of the quantised scores (fp32 vs fp64; rare code flips move it slightly)
    assert np.abs(lse - lse_em).max() <= 2e-3
    # the same error against exact attention as the emulation (code flips aside)
    mse, mse_em = ((o - o_ex) ** 2).mean(), ((o_em - o_ex) ** 2).mean()
    assert abs(mse - mse_em) <= 0.1 * mse_em
    diff = np.abs(o - o_em)
    assert (diff > 2e-2).mean() <= 1e-3 and diff.max() <= 0.15


def test_incoherent_processing_lowers_gpu_error():
    d = 128
    x = synth.make_outlier_inputs(1, 2, 1024, d, frac=0.01, seed=81)
    o_ex, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], False, 1 / math.sqrt(d))
    err = {}
    for rot in (False, True):
        o, _ = _fp8_forward(x, synth.random_signs(d, seed=82) if rot else None, False)
        err[rot] = float(np.sqrt(((o - o_ex) ** 2).mean()))
    ratio = err[False] / err[True]
    assert 2.0 <= ratio <= 3.5, (err, ratio)  # page: 2.6x lower than naive FP8


@pytest.mark.parametrize("B,H,N,causal,rotate,order", [(1, 2, 1000, False, True, 0), (2, 1, 777, True, True, 1),
                                                        (1, 2, 130, True, False, 0)])
def test_fp8_forward_head_dim_64(B, H, N, causal, rotate, order):
    """d = 64: 64-byte E4M3 rows, staged with the 64-byte swizzle."""
    d = 64
    x = synth.make_inputs(B, H, N, d, "bf16", seed=90 + N)
    signs = synth.random_signs(d, seed=91) if rotate else None
    o, lse = _fp8_forward(x, signs, causal, order)
    o_em, lse_em = _oracle_fp8(x, signs, causal, order)
    o_ex, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d))
    assert np.abs(lse - lse_em).max() <= 2e-3
    mse, mse_em = ((o - o_ex) ** 2).mean(), ((o_em - o_ex) ** 2).mean()
    assert abs(mse - mse_em) <= 0.1 * mse_em
    diff = np.abs(o - o_em)
    assert (diff > 2e-2).mean() <= 1e-3 and diff.max() <= 0.15


@pytest.mark.parametrize("B,H,N,causal,rotate,order", [(1, 2, 700, False, True, 0), (1, 1, 333, True, True, 1),
                                                        (1, 2, 200, True, False, 0)])
def test_fp8_forward_head_dim_256(B, H, N, causal, rotate, order):
    """d = 256: the 64-key-tile kernel on E4M3 operands (two 128-byte boxes per
    row); the running max moves once per 64 keys, so the emulation takes B_c = 64."""
    d = 256
    x = synth.make_inputs(B, H, N, d, "bf16", seed=95 + N)
    signs = synth.random_signs(d, seed=96) if rotate else None
    o, lse = _fp8_forward(x, signs, causal, order)
    qq, _ = oracle.fp8_quantize(x["q"], signs)
    kq, _ = oracle.fp8_quantize(x["k"], signs)
    vq, _ = oracle.fp8_quantize(x["v"], None, block_rows=N)
    o_em, lse_em = oracle.attn_fwd_fp8p(qq, kq, vq, causal, 1 / math.sqrt(d), 256.0, order, 64)[:2]
    o_ex, _ = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, 1 / math.sqrt(d))
    assert np.abs(lse - lse_em).max() <= 2e-3
    mse, mse_em = ((o - o_ex) ** 2).mean(), ((o_em - o_ex) ** 2).mean()
    assert abs(mse - mse_em) <= 0.1 * mse_em
    diff = np.abs(o - o_em)
    assert (diff > 2e-2).mean() <= 1e-3 and diff.max() <= 0.15
