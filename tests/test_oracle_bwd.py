"""Pins for the backward oracle: central finite differences of the forward
oracle, torch autograd in float64, and identities the gradient must satisfy."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth


def _inputs(B, H, N, d, seed):
    x = synth.make_inputs(B, H, N, d, "f32", seed=seed, with_grad=True)
    return tuple(x[n].astype(np.float64) for n in ("q", "k", "v", "do"))


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_finite_differences(causal):
    B, H, N, d = 1, 1, 9, 4
    q, k, v, do = _inputs(B, H, N, d, seed=21)
    scale = 0.7
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attn_fwd(q_, k_, v_, causal, scale)
        return float((o * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [q, k, v]
            args_m = [q, k, v]
            pos = "qkv".index(name)
            args_p[pos], args_m[pos] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("d", [16, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_autograd_fp64(causal, d):
    B, H, N = 2, 2, 33
    q, k, v, do = _inputs(B, H, N, d, seed=23)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, scale)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    o.backward(torch.from_numpy(do))
    for g, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=0, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_identities(causal):
    # rows of P sum to one  =>  sum_j dV_j = sum_i dO_i ; rows of dS sum to zero  =>  sum_j dK_j = 0
    q, k, v, do = _inputs(1, 3, 41, 8, seed=29)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, 0.35)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-11)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    if causal:
        # the last key is seen only by the last query: dV_last = P_last,last * dO_last
        o, lse = oracle.attn_fwd(q, k, v, True, 0.35)
        s = 0.35 * np.einsum("bhd,bhd->bh", q[:, :, -1], k[:, :, -1])
        p = np.exp(s - lse[:, :, -1])
        np.testing.assert_allclose(dv[:, :, -1], p[..., None] * do[:, :, -1], atol=1e-12)
