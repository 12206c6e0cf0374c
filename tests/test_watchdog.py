"""Failure detection without a GPU fault: a bounded wait on a barrier that
nothing signals gives up, the status word reports FA_ERR_TIMEOUT, and the
context stays usable for the next launch."""
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_unsignalled_wait_times_out_and_context_survives():
    from exact_io_aware_85_b200 import fa, synth
    assert fa.fa_check_status() == fa.FA_OK
    fa.fa_watchdog_selftest(20000)  # 20 ms bound
    assert fa.fa_check_status() == fa.FA_ERR_TIMEOUT
    assert fa.fa_check_status() == fa.FA_OK  # cleared by the read
    x = synth.make_inputs(1, 1, 200, 64, "bf16", seed=1)
    q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 200), dtype=torch.float32, device="cuda")
    fa.fa_fwd(q, k, v, o, lse, True, 0.125)
    torch.cuda.synchronize()
    assert fa.fa_check_status() == fa.FA_OK
    assert torch.isfinite(o.float()).all()


def test_status_is_read_after_the_given_stream():
    """fa_check_status(stream) waits for that stream only; a timeout raised by a
    kernel on a side stream is reported once that stream's work is done."""
    from exact_io_aware_85_b200 import fa
    side = torch.cuda.Stream()
    fa.fa_watchdog_selftest(20000, stream=side)
    assert fa.fa_check_status(side) == fa.FA_ERR_TIMEOUT
    assert fa.fa_check_status(side) == fa.FA_OK
