"""The C ABI: the library loads on a machine without a GPU and exports every
entry point that include/fa.h declares; bad arguments are rejected with an
error code before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_85_b200 import build
    build.build_library()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("fa_fwd", "fa_fwd_f32", "fa_bwd", "fa_bwd_workspace_bytes", "fa_fwd_fp8p", "fa_status_string",
              "fa_check_status", "fa_last_cuda_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    lib.fa_status_string.restype = ctypes.c_char_p
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(5) == b"FA_ERR_TIMEOUT"


def test_workspace_size(lib):
    lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_bwd_workspace_bytes.argtypes = [ctypes.c_int] * 4
    assert lib.fa_bwd_workspace_bytes(2, 16, 4096, 128) == 2 * 16 * 4096 * 130 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 1, 64) == 128 * 66 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 1, 96) == 0


def test_argument_errors_need_no_gpu(lib):
    """Validation runs before any CUDA call, so these hold on a CPU-only host."""
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp]
    good = vp(1 << 20)
    bad = vp((1 << 20) + 8)
    args = lambda q=good, d=128, scale=0.1, N=64: (q, good, good, good, good, 1, 1, N, d, 1, scale, None)
    assert lib.fa_fwd(*args(q=None)) == 1          # FA_ERR_INVALID_ARG
    assert lib.fa_fwd(*args(N=0)) == 1
    assert lib.fa_fwd(*args(scale=0.0)) == 1
    assert lib.fa_fwd(*args(scale=float("nan"))) == 1
    assert lib.fa_fwd(*args(d=96)) == 2            # FA_ERR_UNSUPPORTED
    assert lib.fa_fwd(*args(q=bad)) == 3           # FA_ERR_ALIGNMENT
    lib.fa_fwd_fp8p.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, cf, ci, vp, ci, vp]
    assert lib.fa_fwd_fp8p(good, good, good, good, good, 1, 1, 64, 128, 0, 0.1, 256.0, 2, None, 4, None) == 1
    assert lib.fa_fwd_fp8p(good, good, good, good, good, 1, 1, 64, 128, 0, 0.1, -1.0, 0, None, 4, None) == 1
    lib.fa_bwd.argtypes = [vp] * 9 + [ci] * 5 + [cf, vp, ctypes.c_size_t, vp]
    ws_small = 10
    assert lib.fa_bwd(*([good] * 9), 1, 1, 64, 128, 1, 0.1, good, ws_small, None) == 1
    assert lib.fa_bwd(*([good] * 9), 1, 1, 64, 128, 1, 0.1, vp((1 << 20) + 16), 1 << 30, None) == 3
