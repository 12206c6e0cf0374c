"""Degenerate and extreme inputs through the forward and backward kernels,
against the fp64 oracle (the forward bound for the peaked case is derived in
the test from the bf16 output and the bf16 P):
  * a strongly peaked softmax (Q and K scaled by 4: scores with a standard
    deviation of 16, the row max far above the rest, the running max growing
    by many 2^8 steps across key tiles, so the lazy O correction fires);
  * uniform attention (K = 0: every score 0, P uniform over the admissible keys,
    O the running mean of V);
at d = 64, 128 and 256, causal and not, on ragged lengths."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu


def _bf16_half_ulp(x):
    """Half a bf16 unit in the last place at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 8)


def _rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def _fwd_bwd(x, causal, d):
    from exact_io_aware_85_b200 import fa
    B, H, N, _ = x["q"].shape
    q, k, v, do = (to_dev(x[n], "bf16") for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    scale = 1 / math.sqrt(d)
    fa.fa_fwd(q, k, v, o, lse, causal, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, causal, scale, ws)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == 0
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    return f(o), f(lse), (f(dq), f(dk), f(dv)), scale


@pytest.mark.parametrize("d,N,causal", [(64, 333, True), (128, 300, False), (256, 257, True)])
def test_peaked_softmax(d, N, causal):
    x = synth.make_inputs(1, 2, N, d, "bf16", seed=500 + d, with_grad=True)
    x["q"] = synth.bf16_round(x["q"] * np.float32(4.0))
    x["k"] = synth.bf16_round(x["k"] * np.float32(4.0))
    o, lse, grads, scale = _fwd_bwd(x, causal, d)
    o_ref, lse_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], causal, scale)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    # A peaked row's O is close to one row of V (|O| up to ~4.5 here), so the
    # flat 1e-2 of the other tests, which assumes |O| <~ 1, does not hold.  The
    # bound per element: half a bf16 ulp of the output (O is stored in bf16)
    # plus the P rounding, |sum_j (bf16(p_j) - p_j) v_j| / l <= 2^-9 max|V|
    # (taken as 2^-8 for the fp32 scores' own rounding).
    bound = _bf16_half_ulp(o_ref) + 2.0 ** -8 * np.abs(x["v"]).max()
    assert (np.abs(o - o_ref) <= bound).all(), np.abs(o - o_ref).max()
    assert np.abs(lse - lse_ref).max() <= 1e-3
    ref = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], causal, scale)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
        assert np.isfinite(g).all(), name
        assert _rel_l2(g, r) <= 2e-2, (name, _rel_l2(g, r))


@pytest.mark.parametrize("d,N,causal", [(64, 200, True), (128, 129, True), (256, 150, False)])
def test_uniform_attention(d, N, causal):
    x = synth.make_inputs(1, 2, N, d, "bf16", seed=600 + d, with_grad=True)
    x["k"] = np.zeros_like(x["k"])
    o, lse, grads, scale = _fwd_bwd(x, causal, d)
    # P uniform over the admissible keys: O is the (running) mean of V, LSE = ln(count)
    v = x["v"].astype(np.float64)
    if causal:
        cnt = np.arange(1, N + 1, dtype=np.float64)
        mean = np.cumsum(v, axis=2) / cnt[None, None, :, None]
    else:
        cnt = np.full(N, float(N))
        mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    assert np.abs(o - mean).max() <= 1e-2
    assert np.abs(lse - np.log(cnt)[None, None, :]).max() <= 1e-3
    ref = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], causal, scale)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
        assert np.isfinite(g).all(), name
        if np.abs(r).max() == 0.0:
            assert np.abs(g).max() <= 1e-2, name
        else:
            assert _rel_l2(g, r) <= 2e-2, (name, _rel_l2(g, r))
