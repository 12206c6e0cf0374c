"""Pins for the decode oracle: a decoding step is the last row of causal
attention over the sequence that ends with the new query, and grouped heads
follow the grouped-query oracle."""
import numpy as np
import pytest

import oracle
from exact_io_aware_85_b200 import synth


@pytest.mark.parametrize("d", [16, 256])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1), (6, 3)])
def test_decode_is_last_row_of_causal_attention(Hq, Hkv, d):
    B, N = 2, 53
    x = synth.make_inputs(B, Hq, N, d, "f32", seed=Hq + 3 * Hkv)
    k, v = x["k"][:, :Hkv], x["v"][:, :Hkv]
    o_full, lse_full = oracle.attn_fwd_gqa(x["q"], k, v, True, 0.2)
    o, lse = oracle.attn_decode(x["q"][:, :, -1], k, v, 0.2)
    np.testing.assert_allclose(o, o_full[:, :, -1], atol=1e-13)
    np.testing.assert_allclose(lse, lse_full[:, :, -1], atol=1e-13)


def test_decode_single_key_returns_its_value():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((1, 3, 8)), rng.standard_normal((1, 3, 1, 8)), rng.standard_normal((1, 3, 1, 8))
    o, lse = oracle.attn_decode(q, k, v, 0.5)
    np.testing.assert_allclose(o, v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("bhd,bhd->bh", q, k[:, :, 0]), atol=1e-14)
