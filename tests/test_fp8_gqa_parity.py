"""Grouped-query FP8 (fa_fp8_quantize_gqa + fa_fwd_fp8_gqa): key/value heads
shared by H / H_kv query heads ("FlashAttention (IT)", "FlashAttention-2 (2023)",
Multi-Query Attention) on the E4M3 operands of "flash-attention-trading-models",
"FA3" item 3.

Sharing a head changes nothing in the arithmetic of one query head, so:
  * the codes and scales of each key/value head equal those of the same head
    repeated over the group through fa_fp8_quantize (bit for bit);
  * the output equals fa_fwd_fp8 on the repeated codes (bit for bit);
  * the output matches the oracle's emulation of the FP8 pipeline on the
    repeated bf16 K and V, with the tolerances of test_fp8full_parity.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu

CASES = [(1, 8, 2, 513, True, True, 0, 128), (2, 4, 1, 300, False, True, 1, 128), (1, 4, 4, 256, True, False, 0, 128),
         (1, 6, 3, 129, False, False, 1, 128), (1, 8, 2, 300, True, True, 1, 64), (1, 4, 2, 200, True, True, 0, 256)]


def _quant(q, k, v, signs, gqa):
    from exact_io_aware_85_b200 import fa
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    nb = (N + 127) // 128
    q8 = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    k8, v8 = (torch.empty(k.shape, dtype=torch.uint8, device="cuda") for _ in range(2))
    sq = torch.empty((B, H, nb), dtype=torch.float32, device="cuda")
    sk = torch.empty((B, Hkv, nb), dtype=torch.float32, device="cuda")
    sv = torch.empty((B, Hkv), dtype=torch.float32, device="cuda")
    (fa.fa_fp8_quantize_gqa if gqa else fa.fa_fp8_quantize)(q, k, v, signs, q8, k8, v8, sq, sk, sv)
    return q8, k8, v8, sq, sk, sv


def _fwd(ops, causal, order, gqa):
    from exact_io_aware_85_b200 import fa
    q8, k8, v8, sq, sk, sv = ops
    B, H, N, d = q8.shape
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    (fa.fa_fwd_fp8_gqa if gqa else fa.fa_fwd_fp8)(q8, k8, v8, sq, sk, sv, o, lse, causal, 1 / math.sqrt(d), 256.0,
                                                   order)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    return o, lse


@pytest.mark.parametrize("B,H,Hkv,N,causal,rotate,order,d", CASES)
def test_fp8_gqa_matches_repeated_heads_and_emulation(B, H, Hkv, N, causal, rotate, order, d):
    g = H // Hkv
    xq = synth.make_inputs(B, H, N, d, "bf16", seed=300 + N)
    xkv = synth.make_inputs(B, Hkv, N, d, "bf16", seed=400 + N)
    k_rep = np.repeat(xkv["k"], g, axis=1)
    v_rep = np.repeat(xkv["v"], g, axis=1)
    signs = synth.random_signs(d, seed=301) if rotate else None
    sg = None if signs is None else torch.from_numpy(signs).cuda()
    q = to_dev(xq["q"], "bf16")
    ops = _quant(q, to_dev(xkv["k"], "bf16"), to_dev(xkv["v"], "bf16"), sg, True)
    rep = _quant(q, to_dev(k_rep, "bf16"), to_dev(v_rep, "bf16"), sg, False)
    torch.cuda.synchronize()
    # codes and scales: each key/value head once == the same head repeated
    assert torch.equal(ops[0], rep[0]) and torch.equal(ops[3], rep[3])
    for a, b in ((ops[1], rep[1]), (ops[2], rep[2]), (ops[4], rep[4]), (ops[5], rep[5])):
        assert torch.equal(a.repeat_interleave(g, dim=1), b)

    o, lse = _fwd(ops, causal, order, True)
    o_rep, lse_rep = _fwd(rep, causal, order, False)
    assert torch.equal(o, o_rep) and torch.equal(lse, lse_rep)

    qq, _ = oracle.fp8_quantize(xq["q"], signs)
    kq, _ = oracle.fp8_quantize(k_rep, signs)
    vq, _ = oracle.fp8_quantize(v_rep, None, block_rows=N)
    # key tiles of 64 at d = 256 (the running max of the P-cast moves once per tile)
    o_em, lse_em = oracle.attn_fwd_fp8p(qq, kq, vq, causal, 1 / math.sqrt(d), 256.0, order, 64 if d == 256 else 128)[:2]
    o_ex, _ = oracle.attn_fwd(xq["q"], k_rep, v_rep, causal, 1 / math.sqrt(d))
    o64 = o.float().cpu().numpy().astype(np.float64)
    assert np.abs(lse.cpu().numpy() - lse_em).max() <= 2e-3
    mse, mse_em = ((o64 - o_ex) ** 2).mean(), ((o_em - o_ex) ** 2).mean()
    assert abs(mse - mse_em) <= 0.1 * mse_em
    diff = np.abs(o64 - o_em)
    assert (diff > 2e-2).mean() <= 1e-3 and diff.max() <= 0.15
