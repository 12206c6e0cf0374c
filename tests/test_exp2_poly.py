"""The FMA-pipe exponential that the d = 64 softmax computes for a quarter of
its key pairs (range reduction x = j + f with |f| <= 1/2, then the degree-3
minimax polynomial of 2^f fitted by the Remez exchange algorithm) against the
hardware's ex2.approx and against float64 2^x."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _run(x_np):
    from exact_io_aware_85_b200 import fa
    x = torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()
    y_fma, y_mufu = torch.empty_like(x), torch.empty_like(x)
    fa.fa_exp2_selftest(x, y_fma, y_mufu)
    torch.cuda.synchronize()
    return y_fma.cpu().numpy().astype(np.float64), y_mufu.cpu().numpy().astype(np.float64)


def test_relative_error_over_the_softmax_range():
    # every argument the softmax can produce: from far below the row maximum up to
    # the lazy-rescale bound of +8, densely, plus the integers and half-integers
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9), np.arange(-126, 8) + 0.5])
    y_fma, y_mufu = _run(x)
    exact = np.exp2(x.astype(np.float32).astype(np.float64))
    rel_fma = np.abs(y_fma / exact - 1.0)
    rel_mufu = np.abs(y_mufu / exact - 1.0)
    normal = exact >= 2.0 ** -125  # the result at -126 < x <= -125 is subnormal-adjacent
    assert rel_fma[normal].max() < 8e-5      # the fit's 7.5e-5 plus float32 rounding
    assert rel_mufu[normal].max() < 2e-6     # the hardware's own bound, for scale
    assert np.abs(y_fma[normal] / y_mufu[normal] - 1.0).max() < 8e-5


def test_masked_and_extreme_arguments():
    # -inf (masked scores) and anything below -126 clamp to 2^-126 (a negligible
    # weight next to the row maximum's 1); 0 gives the fit's value at f = 0
    x = np.array([-np.inf, -1e30, -300.0, -126.0, 0.0, 8.0], dtype=np.float32)
    y_fma, _ = _run(x)
    assert np.all(np.isfinite(y_fma)) and np.all(y_fma >= 0.0)
    assert np.all(y_fma[:4] <= 2.0 ** -125)
    assert abs(y_fma[4] - 1.0) < 8e-5 and abs(y_fma[5] / 256.0 - 1.0) < 8e-5
