"""Pins for the grouped-query oracle: it must agree with the multi-head oracle
on inputs whose heads within a group share K and V, reduce to it when every
group has one head, and its dK/dV must equal the group sums of the multi-head
gradients (checked against torch autograd on the expanded tensors)."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (6, 1), (8, 2)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_forward_is_mha_with_shared_heads(Hq, Hkv, causal):
    B, N, d = 2, 37, 16
    x = synth.make_inputs(B, Hq, N, d, "f32", seed=Hq * 10 + Hkv)
    k = x["k"][:, :Hkv].astype(np.float64)
    v = x["v"][:, :Hkv].astype(np.float64)
    g = Hq // Hkv
    k_full = np.stack([k[:, h // g] for h in range(Hq)], axis=1)
    v_full = np.stack([v[:, h // g] for h in range(Hq)], axis=1)
    o_ref, l_ref = oracle.attn_fwd(x["q"], k_full, v_full, causal, 0.25)
    o, l = oracle.attn_fwd_gqa(x["q"], k, v, causal, 0.25)
    np.testing.assert_allclose(o, o_ref, atol=1e-13)
    np.testing.assert_allclose(l, l_ref, atol=1e-13)


@pytest.mark.parametrize("d", [8, 256])
@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (3, 1)])
def test_gqa_backward_matches_torch_autograd(Hq, Hkv, d):
    B, N = 1, 23
    x = synth.make_inputs(B, Hq, N, d, "f32", seed=7, with_grad=True)
    q = x["q"].astype(np.float64)
    k = x["k"][:, :Hkv].astype(np.float64)
    v = x["v"][:, :Hkv].astype(np.float64)
    do = x["do"].astype(np.float64)
    dq, dk, dv = oracle.attn_bwd_gqa(q, k, v, do, True, 0.3)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    g = Hq // Hkv
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk.repeat_interleave(g, dim=1),
                                                         tv.repeat_interleave(g, dim=1), is_causal=True, scale=0.3)
    o.backward(torch.from_numpy(do))
    for a, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, t.grad.numpy(), atol=1e-11)
