"""Pins for the forward oracle.  None of these re-type the oracle's formula:
they check it against a library routine (torch SDPA in float64), against
invariants the definition implies, and against a different algorithm (the
pages' tiled online-softmax loop) on tiny inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_85_b200 import synth


def _rand(B, H, N, d, seed):
    x = synth.make_inputs(B, H, N, d, "f32", seed=seed)
    return x["q"].astype(np.float64), x["k"].astype(np.float64), x["v"].astype(np.float64)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 37, 16), (2, 1, 64, 32), (1, 1, 1, 8), (1, 2, 37, 256)])
def test_fwd_matches_torch_sdpa_fp64(shape, causal):
    q, k, v = _rand(*shape, seed=3)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    tq, tk, tv = (torch.from_numpy(a) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    s = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
    if causal:
        N = shape[2]
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    # with V = identity (d = N) the output row IS the softmax row of P
    N = 24
    q, k, _ = _rand(1, 1, N, N, seed=5)
    v = np.eye(N)[None, None]
    p, _ = oracle.attn_fwd(q, k, v, causal, 0.3)
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    if causal:
        assert np.all(np.triu(p[0, 0], 1) == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_allowed_values(causal):
    B, H, N, d = 1, 2, 50, 8
    _, k, v = _rand(B, H, N, d, seed=7)
    q = np.zeros((B, H, N, d))
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.125)
    counts = np.arange(1, N + 1) if causal else np.full(N, N)
    if causal:
        mean = np.cumsum(v, axis=2) / counts[None, None, :, None]
    else:
        mean = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
    np.testing.assert_allclose(o, mean, atol=1e-13)
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(counts), lse.shape), atol=1e-13)


def test_dominant_logit_selects_one_value_row():
    # key j points along dim j % d, query i along one chosen dim; with a logit gap
    # of 200 every non-matching key weighs e^-200, so O is the mean of the
    # matching V rows and LSE = gap + ln(#matches)
    B, H, N, d = 1, 1, 40, 16
    rng = np.random.default_rng(11)
    v = rng.standard_normal((B, H, N, d))
    k = np.zeros((B, H, N, d))
    q = np.zeros((B, H, N, d))
    for j in range(N):
        k[0, 0, j, j % d] = 1.0
    sel = rng.choice(np.arange(d), size=N)
    for i in range(N):
        q[0, 0, i, sel[i]] = 1.0
    scale = 200.0
    o, lse = oracle.attn_fwd(q, k, v, False, scale)
    for i in range(N):
        hits = [j for j in range(N) if j % d == sel[i]]
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, hits].mean(axis=0), atol=1e-12)
        assert abs(lse[0, 0, i] - (scale + math.log(len(hits)))) < 1e-12


def _tiled_online(q, k, v, causal, scale, Bc):
    """The pages' tiled loop (running max m, running sum l, O renormalised after
    every key block), written independently of the oracle, fp64."""
    B, H, N, d = q.shape
    O = np.zeros_like(q)
    L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                m, l, o = -np.inf, 0.0, np.zeros(d)
                for j0 in range(0, N, Bc):
                    j1 = min(N, j0 + Bc)
                    if causal:
                        j1 = min(j1, i + 1)
                    if j1 <= j0:
                        continue
                    s = scale * (k[b, h, j0:j1] @ q[b, h, i])
                    m_ij = s.max()
                    p = np.exp(s - m_ij)
                    l_ij = p.sum()
                    m_new = max(m, m_ij)
                    l_new = l * math.exp(m - m_new) + l_ij * math.exp(m_ij - m_new)
                    o = o * (l * math.exp(m - m_new) / l_new) + (p @ v[b, h, j0:j1]) * (math.exp(m_ij - m_new) / l_new)
                    m, l = m_new, l_new
                O[b, h, i] = o
                L[b, h, i] = m + math.log(l)
    return O, L


@pytest.mark.parametrize("Bc", [1, 3, 16, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_tiled_online_softmax_agrees_with_two_pass(Bc, causal):
    q, k, v = _rand(1, 2, 29, 8, seed=13)
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.4)
    o2, lse2 = _tiled_online(q, k, v, causal, 0.4, Bc)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, atol=1e-12)


def test_sampled_rows_match_full():
    q, k, v = _rand(2, 3, 70, 16, seed=17)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.25)
    rows = np.array([[0, 0], [5, 69], [3, 17], [1, 1]])
    orow, lrow = oracle.attn_fwd_rows(q, k, v, rows, True, 0.25)
    of, lf = o.reshape(6, 70, 16), lse.reshape(6, 70)
    for r, (bh, i) in enumerate(rows):
        assert np.array_equal(orow[r], of[bh, i])
        assert lrow[r] == lf[bh, i]


def test_large_logits_do_not_overflow():
    q, k, v = _rand(1, 1, 16, 4, seed=19)
    o, lse = oracle.attn_fwd(q * 1e3, k, v, False, 1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (q * 1e3, k, v)), scale=1.0)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
