"""The bench workloads that the other parity files check only at smaller sizes,
run here at their own sizes and through the calls bench.py times, against the
fp64 oracle on sampled outputs it can compute one by one:

  prefill_gqa   B4 H32 H_kv8 N8192 d128 causal   fa_fwd_gqa        sampled rows
  prefill_d256  B4 H16 N8192 d256 causal         fa_fwd            sampled rows
  prefill_fp8   B4 H32 N8192 d128 causal, E4M3   fa_fp8_quantize + fa_fwd_fp8, two whole heads against
                                                 the emulation of the E4M3 pipeline
  decode(_d256) B8 H32 H_kv8, 32K keys, d128/256 fa_decode         four (batch, key/value head) groups
  train_d256    B2 H8 N8192 d256 causal          fa_fwd + fa_bwd   one whole head (dQ, dK, dV)

Tolerances are those of the smaller parity tests: forward O max-abs 1e-2 and
LSE 1e-3; FP8 as test_fp8full_parity; backward relative L2 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import sample_rows, to_dev

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, REL_L2 = 1e-2, 1e-3, 2e-2


def _rows_by_head(rows):
    heads = {}
    for bh, n in rows:
        heads.setdefault(int(bh), []).append(int(n))
    return heads


def _check_rows(o, lse, x_q, x_k, x_v, rows, H, Hkv, causal, scale):
    """o, lse: GPU results [B,H,N,d], [B,H,N]; each sampled row against the oracle
    on its own head (key/value head h / (H / H_kv))."""
    g = H // Hkv
    for bh, ns in _rows_by_head(rows).items():
        b, h = divmod(bh, H)
        sub_rows = np.array([[0, n] for n in ns], dtype=np.int64)
        o_ref, lse_ref = oracle.attn_fwd_rows(x_q[b:b + 1, h:h + 1], x_k[b:b + 1, h // g:h // g + 1],
                                              x_v[b:b + 1, h // g:h // g + 1], sub_rows, causal, scale)
        assert np.abs(o[b, h, ns] - o_ref).max() <= O_TOL, (b, h)
        assert np.abs(lse[b, h, ns] - lse_ref).max() <= LSE_TOL, (b, h)


def test_prefill_gqa_full_size_sampled_rows():
    from exact_io_aware_85_b200 import fa
    w = synth.WORKLOADS["prefill_gqa"]
    seed = synth.workload_seed(w.name)
    xq = synth.make_inputs(w.B, w.H, w.N, w.d, "bf16", seed=seed)
    xkv = synth.make_inputs(w.B, w.hkv, w.N, w.d, "bf16", seed=seed + 1)
    q = to_dev(xq["q"], "bf16")
    k, v = to_dev(xkv["k"], "bf16"), to_dev(xkv["v"], "bf16")
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_gqa(q, k, v, o, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    rows = sample_rows(w.B * w.H, w.N, 64, seed=11)
    _check_rows(o, lse, xq["q"], xkv["k"], xkv["v"], rows, w.H, w.hkv, w.causal, w.scale)


def test_prefill_d256_full_size_sampled_rows():
    from exact_io_aware_85_b200 import fa
    w = synth.WORKLOADS["prefill_d256"]
    x = synth.make_inputs(w.B, w.H, w.N, w.d, "bf16", seed=synth.workload_seed(w.name))
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    fa.fa_fwd(q, k, v, o, lse, w.causal, w.scale)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    rows = sample_rows(w.B * w.H, w.N, 48, seed=12)
    _check_rows(o, lse, x["q"], x["k"], x["v"], rows, w.H, w.H, w.causal, w.scale)


def test_prefill_fp8_full_size_two_heads():
    """Quantisation and the E4M3 forward over the whole workload; two whole heads
    (the first and the last) against the oracle's emulation of the pipeline."""
    from exact_io_aware_85_b200 import fa
    w = synth.WORKLOADS["prefill_fp8"]
    x = synth.make_inputs(w.B, w.H, w.N, w.d, "bf16", seed=synth.workload_seed(w.name))
    signs = synth.random_signs(w.d, seed=synth.workload_seed(w.name))
    q, k, v = (to_dev(x[n], "bf16") for n in ("q", "k", "v"))
    nb = (w.N + 127) // 128
    q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device="cuda") for _ in range(3))
    sq = torch.empty((w.B, w.H, nb), dtype=torch.float32, device="cuda")
    sk = torch.empty_like(sq)
    sv = torch.empty((w.B, w.H), dtype=torch.float32, device="cuda")
    fa.fa_fp8_quantize(q, k, v, torch.from_numpy(signs).cuda(), q8, k8, v8, sq, sk, sv)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, w.causal, w.scale, 256.0, 0)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o, lse = o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        qq, _ = oracle.fp8_quantize(x["q"][sl], signs)
        kq, _ = oracle.fp8_quantize(x["k"][sl], signs)
        vq, _ = oracle.fp8_quantize(x["v"][sl], None, block_rows=w.N)
        o_em, lse_em = oracle.attn_fwd_fp8p(qq, kq, vq, w.causal, w.scale, 256.0, 0)[:2]
        assert np.abs(lse[sl] - lse_em).max() <= 2e-3, (b, h)
        diff = np.abs(o[sl] - o_em)
        assert (diff > 2e-2).mean() <= 1e-3 and diff.max() <= 0.15, (b, h)


@pytest.mark.parametrize("name", ["decode", "decode_d256"])
def test_decode_full_size_sampled_groups(name):
    """The 32K-token cache at the bench's shape; four (batch, key/value head)
    groups, every query head of each, against the oracle."""
    from exact_io_aware_85_b200 import fa
    w = synth.WORKLOADS[name]
    seed = synth.workload_seed(w.name)
    x = synth.make_inputs(w.B, w.hkv, w.N, w.d, "bf16", seed=seed)
    qx = np.ascontiguousarray(synth.make_inputs(w.B, w.H, 1, w.d, "bf16", seed=seed + 1)["q"][:, :, 0])
    q = to_dev(qx, "bf16")
    k, v = to_dev(x["k"], "bf16"), to_dev(x["v"], "bf16")
    o = torch.empty((w.B, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.H), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_workspace_bytes(w.B, w.H, w.hkv, w.N, w.d), dtype=torch.uint8, device="cuda")
    fa.fa_decode(q, k, v, o, lse, w.scale, ws)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    g = w.H // w.hkv
    for b, hk in ((0, 0), (w.B - 1, w.hkv - 1), (w.B // 2, 1), (1, w.hkv // 2)):
        hs = slice(hk * g, (hk + 1) * g)
        o_ref, lse_ref = oracle.attn_decode(qx[b:b + 1, hs], x["k"][b:b + 1, hk:hk + 1], x["v"][b:b + 1, hk:hk + 1],
                                            w.scale)
        assert np.abs(o[b:b + 1, hs] - o_ref).max() <= O_TOL, (b, hk)
        assert np.abs(lse[b:b + 1, hs] - lse_ref).max() <= LSE_TOL, (b, hk)


def _rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def test_train_d256_full_size_one_head():
    """The d = 256 training step (forward, then the CTA-pair backward) over the
    whole workload; the last head, every row, against the oracle's backward."""
    from exact_io_aware_85_b200 import fa
    w = synth.WORKLOADS["train_d256"]
    x = synth.make_inputs(w.B, w.H, w.N, w.d, "bf16", seed=synth.workload_seed(w.name), with_grad=True)
    q, k, v, do = (to_dev(x[n], "bf16") for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    fa.fa_fwd(q, k, v, o, lse, w.causal, w.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.H, w.N, w.d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, w.causal, w.scale, ws)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    b, h = w.B - 1, w.H - 1
    got = [t[b, h].float().cpu().numpy() for t in (dq, dk, dv)]
    sub = {n: x[n][b:b + 1, h:h + 1] for n in ("q", "k", "v", "do")}
    ref = oracle.attn_bwd(sub["q"], sub["k"], sub["v"], sub["do"], w.causal, w.scale)
    for name, g_, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(g_).all(), name
        assert _rel_l2(g_, r[0, 0]) <= REL_L2, (name, _rel_l2(g_, r[0, 0]))
