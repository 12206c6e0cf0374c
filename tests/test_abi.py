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
    assert lib.fa_bwd_workspace_bytes(1, 1, 1, 256) == 128 * 258 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 1, 96) == 0


def test_decode_workspace_size(lib):
    """The decode step splits each key/value head's cache into chunks of whole
    128-key tiles so that one wave of CTAs (one per SM of 148) covers the
    B*H_kv heads; the workspace holds one partial O row (d floats) plus (m, l)
    per query head and chunk, rounded up to 256 bytes."""
    lib.fa_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_decode_workspace_bytes.argtypes = [ctypes.c_int] * 5

    def expect(B, H, Hkv, N, d):
        tiles = -(-N // 128)
        ns = min(tiles, max(1, 148 // (B * Hkv)))
        tps = -(-tiles // ns)
        ns = -(-tiles // tps)
        return -(-(ns * B * H * (d + 2) * 4) // 256) * 256

    for args in [(8, 32, 8, 32768, 128), (1, 8, 8, 1000, 128), (2, 32, 8, 4097, 128), (4, 16, 1, 333, 64),
                 (1, 4, 4, 1, 64), (1, 16, 16, 70000, 128), (3, 12, 4, 65, 64), (64, 64, 8, 4096, 128)]:
        assert lib.fa_decode_workspace_bytes(*args) == expect(*args), args
    # the decode workload: 2 chunks of 128 tiles per key/value head
    assert expect(8, 32, 8, 32768, 128) == 2 * 8 * 32 * 130 * 4
    for args in ((1, 8, 2, 1000, 256), (2, 16, 1, 4097, 256)):
        assert lib.fa_decode_workspace_bytes(*args) == expect(*args) > 0
    assert lib.fa_decode_workspace_bytes(1, 6, 4, 100, 128) == 0   # H not a multiple of H_kv
    assert lib.fa_decode_workspace_bytes(1, 4, 4, 100, 96) == 0    # unsupported head dim


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


def test_head_dim_256_is_admitted_where_declared(lib):
    """d = 256 passes the argument checks of the entry points that declare it
    (their next check, a short workspace or a misaligned pointer, is the one that
    fails) and is refused with FA_ERR_UNSUPPORTED by those that do not."""
    vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    good = vp(1 << 20)
    bad = vp((1 << 20) + 8)
    lib.fa_bwd.argtypes = [vp] * 9 + [ci] * 5 + [cf, vp, sz, vp]
    assert lib.fa_bwd(*([good] * 9), 1, 1, 64, 256, 1, 0.1, good, 10, None) == 1          # workspace too small
    assert lib.fa_bwd(*([good] * 9), 1, 1, 64, 96, 1, 0.1, good, 1 << 30, None) == 2      # unsupported
    lib.fa_bwd_gqa.argtypes = [vp] * 9 + [ci] * 6 + [cf, vp, sz, vp]
    assert lib.fa_bwd_gqa(*([good] * 9), 1, 4, 2, 64, 256, 1, 0.1, good, 10, None) == 1
    lib.fa_bwd_noalloc.argtypes = [vp] * 9 + [ci] * 5 + [cf, vp]
    assert lib.fa_bwd_noalloc(*([good] * 4), bad, *([good] * 4), 1, 1, 64, 256, 1, 0.1, None) == 3  # dO misaligned
    lib.fa_decode.argtypes = [vp] * 5 + [ci] * 5 + [cf, vp, sz, vp]
    assert lib.fa_decode(good, good, good, good, good, 1, 4, 1, 64, 256, 0.1, good, 10, None) == 1
    assert lib.fa_decode(good, good, good, good, good, 1, 4, 1, 64, 96, 0.1, good, 1 << 30, None) == 2
    assert lib.fa_decode(good, good, good, good, good, 1, 32, 1, 64, 256, 0.1, good, 1 << 30, None) == 2  # g > 16
    lib.fa_fwd_fp8.argtypes = [vp] * 3 + [vp] * 3 + [vp, vp] + [ci] * 5 + [cf, cf, ci, vp]
    assert lib.fa_fwd_fp8(*([good] * 8), 1, 1, 64, 96, 1, 0.1, 256.0, 0, None) == 2       # FP8 takes d = 64, 128, 256
    lib.fa_fwd_fp8_gqa.argtypes = [vp] * 8 + [ci] * 6 + [cf, cf, ci, vp]
    assert lib.fa_fwd_fp8_gqa(*([good] * 8), 1, 6, 4, 64, 128, 1, 0.1, 256.0, 0, None) == 1  # H % H_kv != 0
    assert lib.fa_fwd_fp8_gqa(*([good] * 8), 1, 8, 0, 64, 128, 1, 0.1, 256.0, 0, None) == 1  # H_kv = 0
    assert lib.fa_fwd_fp8_gqa(*([good] * 8), 1, 8, 2, 64, 96, 1, 0.1, 256.0, 0, None) == 2   # d in {64, 128, 256}
    assert lib.fa_fwd_fp8_gqa(*([good] * 8), 1, 8, 2, 64, 128, 1, 0.1, 256.0, 2, None) == 1  # bad kv_order
    assert lib.fa_fwd_fp8_gqa(*([good] * 8), 1, 8, 2, 64, 256, 1, 0.1, 256.0, 2, None) == 1  # d = 256 admitted
    lib.fa_fp8_quantize_gqa.argtypes = [vp] * 10 + [ci] * 5 + [vp]
    assert lib.fa_fp8_quantize_gqa(*([good] * 10), 1, 6, 4, 64, 128, None) == 1             # H % H_kv != 0
    assert lib.fa_fp8_quantize_gqa(*([good] * 10), 1, 8, 2, 64, 96, None) == 2              # d in {64, 128, 256}


def test_size_limits_and_lse_alignment(lib):
    """Sizes are limited by what the launches express, not by a 2^31-element
    cap; lse needs 4-byte alignment only.  Every call here stops at a later
    argument check (an invalid S), so nothing is launched on the fake pointers:
    status 1 shows the earlier checks passed."""
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd_fp8p.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, cf, ci, vp, ci, vp]
    good = vp(1 << 20)

    def call(B, H, N, d=128, lse=good):
        return lib.fa_fwd_fp8p(good, good, good, good, lse, B, H, N, d, 0, 0.1, -1.0, 0, None, 4, None)

    assert call(4, 32, 131072) == 1             # 2^31 elements: a long-context prefill is taken
    assert call(1, 1, (1 << 30) + 1, 64) == 2   # N past 2^30
    assert call(65536, 32768, 1) == 2           # B*H = 2^31
    assert call(1 << 14, 1 << 14, 128, 64) == 2  # 2^28 CTAs would fit, but 2^41 elements do not
    assert call(1 << 10, 1 << 10, 128, 64) == 1  # 2^20 heads, 2^33 elements: taken
    assert call(1, 1, 64, lse=vp((1 << 20) + 4)) == 1   # lse 4-byte aligned: accepted
    assert call(1, 1, 64, lse=vp((1 << 20) + 2)) == 3   # lse 2-byte aligned: refused


def test_grid_y_limits_refused_before_launch(lib):
    """fa_decode puts B*H_kv and fa_fp8_quantize puts B*H on gridDim.y (at most
    65535); larger counts are refused before any launch."""
    vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    good = vp(1 << 20)
    lib.fa_decode.argtypes = [vp] * 5 + [ci] * 5 + [cf, vp, sz, vp]
    assert lib.fa_decode(good, good, good, good, good, 1024, 128, 128, 1, 64, 0.1, good, 1 << 40, None) == 2
    assert lib.fa_decode(good, good, good, good, good, 1023, 128, 64, 1, 64, 0.1, good, 10, None) == 1  # 65472: short workspace next
    lib.fa_fp8_quantize.argtypes = [vp] * 4 + [vp] * 3 + [vp] * 3 + [ci] * 4 + [vp]
    assert lib.fa_fp8_quantize(*([good] * 10), 256, 256, 1, 64, None) == 2
    assert lib.fa_fp8_quantize(*([good] * 10), 1, 1, 64, 96, None) == 2
