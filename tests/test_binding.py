"""The Python binding checks every tensor argument (CUDA, contiguous, dtype,
shape, one device) before it calls into the library; on this CPU host the
checks fire on CPU tensors, so no CUDA call is made."""
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fa():
    from exact_io_aware_85_b200 import fa
    return fa


def test_rejects_host_tensors():
    fa = _fa()
    q = torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16)
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, q, q, q, lse, False, 0.125)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    assert "fa_fwd(q:" in str(e.value)


def test_rejects_decode_host_tensors_and_bad_rank():
    fa = _fa()
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 1, 16, 64), dtype=torch.bfloat16)
    lse = torch.zeros((1, 4), dtype=torch.float32)
    ws = torch.zeros(256, dtype=torch.uint8)
    with pytest.raises(fa.FAError) as e:
        fa.fa_decode(q, k, k, q, lse, 0.125, ws)
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        fa.fa_decode(q[0], k, k, q, lse, 0.125, ws)


def test_need_checks_dtype_and_shape_in_order():
    fa = _fa()
    # the checker itself: None is accepted only where the shape is None
    fa._need("x", a=(None, torch.float32, None))
    with pytest.raises(fa.FAError):
        fa._need("x", a=(None, torch.float32, (4,)))


def test_every_entry_point_has_a_binding_of_the_same_name():
    """The Python layer mirrors the C ABI name for name (argument marshalling only)."""
    import re

    from exact_io_aware_85_b200 import fa
    header = open(os.path.join(ROOT, "include", "fa.h")).read()
    declared = set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(fa_\w+)\(", header, re.M))
    assert len(declared) >= 16
    assert sorted(n for n in declared if not callable(getattr(fa, n, None))) == []
