"""ctypes binding of libfa.so with the entry-point names of include/fa.h.

Argument marshalling only: sizes and raw device pointers are taken from torch
tensors (torch is the allocator and stream owner), every step of the
computation runs in the library's CUDA kernels.  There is no fallback: if the
library is missing the import fails, and a non-zero status raises FAError.
"""
from __future__ import annotations

import ctypes
import os

import torch

# FA_DEBUG=1 selects the build with device-side argument checks (FA_ERR_CHECK)
_DEBUG = os.environ.get("FA_DEBUG") == "1"
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_debug.so" if _DEBUG else "libfa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{os.path.basename(_LIB_PATH)} is not built ({_LIB_PATH}); run "
                      f"`python -m exact_io_aware_85_b200.build{' --debug' if _DEBUG else ''}`")

lib = ctypes.CDLL(_LIB_PATH)
_vp, _ci, _cf, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.fa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp]
lib.fa_fwd_f32.argtypes = [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp]
lib.fa_fwd_fp8p.argtypes = [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _cf, _ci, _vp, _ci, _vp]
lib.fa_bwd_workspace_bytes.restype = _sz
lib.fa_bwd_workspace_bytes.argtypes = [_ci, _ci, _ci, _ci]
lib.fa_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _sz, _vp]
lib.fa_status_string.restype = ctypes.c_char_p
lib.fa_status_string.argtypes = [_ci]
lib.fa_last_cuda_error.restype = _ci
lib.fa_check_status.restype = _ci
lib.fa_check_status.argtypes = [_vp]
lib.fa_watchdog_selftest.argtypes = [ctypes.c_uint, _vp]
lib.fa_exp2_selftest.argtypes = [_vp, _vp, _vp, _ci, _vp]

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_CHECK = range(7)
EXPORTS = ("fa_fwd", "fa_fwd_f32", "fa_fwd_fp8p", "fa_bwd_workspace_bytes", "fa_bwd", "fa_status_string",
           "fa_last_cuda_error", "fa_check_status", "fa_watchdog_selftest", "fa_exp2_selftest")


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.fa_status_string(status).decode()
        if status == FA_ERR_CUDA:
            msg += f" (cudaError {lib.fa_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str) -> None:
    if status != FA_OK:
        raise FAError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dims(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _need(where: str, **tensors) -> None:
    """Every tensor argument must be a contiguous CUDA tensor of the stated dtype
    and shape, on one device: the kernels take sizes from the leading tensor and
    would otherwise read or write past a mismatched buffer.  Each keyword is
    name=(tensor, dtype, shape); a None tensor with shape None is allowed."""
    dev = None
    for name, (t, dtype, shape) in tensors.items():
        if t is None and shape is None:
            continue
        ok = (isinstance(t, torch.Tensor) and t.is_cuda and t.is_contiguous() and t.dtype == dtype
              and (shape is None or tuple(t.shape) == tuple(shape)))
        if ok and dev is not None and t.device != dev:
            ok = False
        if not ok:
            got = "None" if t is None else f"{getattr(t, 'dtype', type(t))} {list(getattr(t, 'shape', []))}" + (
                f" on {t.device}, contiguous={t.is_contiguous()}" if isinstance(t, torch.Tensor) else "")
            raise FAError(FA_ERR_INVALID_ARG,
                          f"{where}({name}: expected contiguous {dtype} {list(shape) if shape else ''} on one CUDA "
                          f"device, got {got})")
        dev = t.device

_bf, _f32, _u8, _i64 = torch.bfloat16, torch.float32, torch.uint8, torch.int64


def fa_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """bf16 forward: writes o (bf16 [B,H,N,d]) and lse (fp32 [B,H,N])."""
    B, H, N, d = _dims(q)
    x = (B, H, N, d)
    _need("fa_fwd", q=(q, _bf, x), k=(k, _bf, x), v=(v, _bf, x), o=(o, _bf, x), lse=(lse, _f32, (B, H, N)))
    _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale),
                      _stream(stream)), "fa_fwd")


def fa_fwd_f32(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """fp32 forward on the tf32 tensor-core path."""
    B, H, N, d = _dims(q)
    x = (B, H, N, d)
    _need("fa_fwd_f32", q=(q, _f32, x), k=(k, _f32, x), v=(v, _f32, x), o=(o, _f32, x), lse=(lse, _f32, (B, H, N)))
    _check(lib.fa_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale),
                          _stream(stream)), "fa_fwd_f32")


def fa_fwd_fp8p(q, k, v, o, lse, causal: bool, scale: float, S: float, kv_order: int, stats=None, n_sink: int = 4,
                stream=None) -> None:
    """Forward with P cast to E4M3 under static scale S; stats (uint64 [4] as int64) is added to."""
    B, H, N, d = _dims(q)
    x = (B, H, N, d)
    _need("fa_fwd_fp8p", q=(q, _bf, x), k=(k, _bf, x), v=(v, _bf, x), o=(o, _bf, x), lse=(lse, _f32, (B, H, N)),
          stats=(stats, _i64, None if stats is None else (4,)))
    _check(lib.fa_fwd_fp8p(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale),
                           float(S), int(kv_order), _ptr(stats), int(n_sink), _stream(stream)), "fa_fwd_fp8p")


def fa_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, causal: bool, scale: float, workspace, stream=None) -> None:
    """Backward: writes dq, dk, dv (bf16 [B,H,N,d]); workspace is a uint8 device tensor."""
    B, H, N, d = _dims(q)
    x = (B, H, N, d)
    _need("fa_bwd", q=(q, _bf, x), k=(k, _bf, x), v=(v, _bf, x), o=(o, _bf, x), do=(do, _bf, x),
          lse=(lse, _f32, (B, H, N)), dq=(dq, _bf, x), dk=(dk, _bf, x), dv=(dv, _bf, x),
          workspace=(workspace, _u8, (int(workspace.numel()),)))
    _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                      N, d, int(causal), float(scale), _ptr(workspace), int(workspace.numel()),
                      _stream(stream)), "fa_bwd")


def fa_status_string(status: int) -> str:
    return lib.fa_status_string(int(status)).decode()


def fa_check_status(stream=None) -> int:
    """Status word of the current device once the work on `stream` (default:
    torch's current stream) has finished; reading clears it."""
    return int(lib.fa_check_status(_stream(stream)))


def fa_last_cuda_error() -> int:
    """The cudaError_t of this host thread's last failed CUDA call inside the library."""
    return int(lib.fa_last_cuda_error())


def fa_exp2_selftest(x, y_fma, y_mufu, stream=None) -> None:
    """y_fma = the FMA-pipe exponential of the d = 64 softmax, y_mufu = ex2.approx,
    both of the fp32 CUDA tensor x (same shape)."""
    _need("fa_exp2_selftest", x=(x, torch.float32, None), y_fma=(y_fma, torch.float32, tuple(x.shape)),
          y_mufu=(y_mufu, torch.float32, tuple(x.shape)))
    _check(lib.fa_exp2_selftest(_ptr(x), _ptr(y_fma), _ptr(y_mufu), int(x.numel()), _stream(stream)),
           "fa_exp2_selftest")


def fa_watchdog_selftest(limit_us: int, stream=None) -> None:
    _check(lib.fa_watchdog_selftest(int(limit_us), _stream(stream)), "fa_watchdog_selftest")


lib.fa_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp]


def fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal: bool, scale: float, stream=None) -> None:
    """Backward without a caller workspace: the library's own fixed device scratch
    array (32 MiB) is used, so nothing is allocated; larger sizes raise
    FA_ERR_UNSUPPORTED.  Calls that overlap on the GPU race on that array."""
    B, H, N, d = _dims(q)
    x = (B, H, N, d)
    _need("fa_bwd_noalloc", q=(q, _bf, x), k=(k, _bf, x), v=(v, _bf, x), o=(o, _bf, x), do=(do, _bf, x),
          lse=(lse, _f32, (B, H, N)), dq=(dq, _bf, x), dk=(dk, _bf, x), dv=(dv, _bf, x))
    _check(lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                              B, H, N, d, int(causal), float(scale), _stream(stream)), "fa_bwd_noalloc")


lib.fa_fp8_quantize.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _vp]
lib.fa_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _cf, _ci, _vp]
lib.fa_fp8_quantize_gqa.argtypes = [_vp] * 10 + [_ci] * 5 + [_vp]
lib.fa_fwd_fp8_gqa.argtypes = [_vp] * 8 + [_ci] * 6 + [_cf, _cf, _ci, _vp]


def fa_fp8_quantize(q, k, v, signs, q8, k8, v8, sq, sk, sv, stream=None) -> None:
    """E4M3 codes (uint8 tensors) and scales for fa_fwd_fp8; signs: fp32 [d] or None."""
    B, H, N, d = _dims(q)
    x, nb = (B, H, N, d), (N + 127) // 128
    _need("fa_fp8_quantize", q=(q, _bf, x), k=(k, _bf, x), v=(v, _bf, x), signs=(signs, _f32, None if signs is None else (d,)),
          q8=(q8, _u8, x), k8=(k8, _u8, x), v8=(v8, _u8, x), sq=(sq, _f32, (B, H, nb)), sk=(sk, _f32, (B, H, nb)),
          sv=(sv, _f32, (B, H)))
    _check(lib.fa_fp8_quantize(_ptr(q), _ptr(k), _ptr(v), _ptr(signs), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq),
                               _ptr(sk), _ptr(sv), B, H, N, d, _stream(stream)), "fa_fp8_quantize")


def fa_fwd_fp8(q8, k8, v8, sq, sk, sv, o, lse, causal: bool, scale: float, S: float = 256.0, kv_order: int = 0,
               stream=None) -> None:
    """Forward on E4M3 operands; o is bf16 [B,H,N,d]."""
    B, H, N, d = _dims(q8)
    x, nb = (B, H, N, d), (N + 127) // 128
    _need("fa_fwd_fp8", q8=(q8, _u8, x), k8=(k8, _u8, x), v8=(v8, _u8, x), sq=(sq, _f32, (B, H, nb)),
          sk=(sk, _f32, (B, H, nb)), sv=(sv, _f32, (B, H)), o=(o, _bf, x), lse=(lse, _f32, (B, H, N)))
    _check(lib.fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o), _ptr(lse), B, H, N,
                          d, int(causal), float(scale), float(S), int(kv_order), _stream(stream)), "fa_fwd_fp8")


def fa_fp8_quantize_gqa(q, k, v, signs, q8, k8, v8, sq, sk, sv, stream=None) -> None:
    """fa_fp8_quantize with k, v (and k8, v8, sk, sv) over H_kv key/value heads."""
    B, H, N, d = _dims(q)
    Hkv = int(k.shape[1]) if k.dim() == 4 else -1
    x, xkv, nb = (B, H, N, d), (B, Hkv, N, d), (N + 127) // 128
    _need("fa_fp8_quantize_gqa", q=(q, _bf, x), k=(k, _bf, xkv), v=(v, _bf, xkv),
          signs=(signs, _f32, None if signs is None else (d,)), q8=(q8, _u8, x), k8=(k8, _u8, xkv),
          v8=(v8, _u8, xkv), sq=(sq, _f32, (B, H, nb)), sk=(sk, _f32, (B, Hkv, nb)), sv=(sv, _f32, (B, Hkv)))
    _check(lib.fa_fp8_quantize_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(signs), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq),
                                   _ptr(sk), _ptr(sv), B, H, Hkv, N, d, _stream(stream)), "fa_fp8_quantize_gqa")


def fa_fwd_fp8_gqa(q8, k8, v8, sq, sk, sv, o, lse, causal: bool, scale: float, S: float = 256.0, kv_order: int = 0,
                   stream=None) -> None:
    """fa_fwd_fp8 with k8, v8, sk, sv over H_kv key/value heads."""
    B, H, N, d = _dims(q8)
    Hkv = int(k8.shape[1]) if k8.dim() == 4 else -1
    x, xkv, nb = (B, H, N, d), (B, Hkv, N, d), (N + 127) // 128
    _need("fa_fwd_fp8_gqa", q8=(q8, _u8, x), k8=(k8, _u8, xkv), v8=(v8, _u8, xkv), sq=(sq, _f32, (B, H, nb)),
          sk=(sk, _f32, (B, Hkv, nb)), sv=(sv, _f32, (B, Hkv)), o=(o, _bf, x), lse=(lse, _f32, (B, H, N)))
    _check(lib.fa_fwd_fp8_gqa(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o), _ptr(lse), B, H,
                              Hkv, N, d, int(causal), float(scale), float(S), int(kv_order), _stream(stream)),
           "fa_fwd_fp8_gqa")


lib.fa_fwd_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, _cf, _vp]
lib.fa_bwd_gqa.argtypes = [_vp] * 9 + [_ci] * 6 + [_cf, _vp, _sz, _vp]


def fa_fwd_gqa(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """Grouped-query forward: k, v have H_kv heads, q and o have H (a multiple)."""
    B, H, N, d = _dims(q)
    Hkv = int(k.shape[1]) if k.dim() == 4 else -1
    x, xkv = (B, H, N, d), (B, Hkv, N, d)
    _need("fa_fwd_gqa", q=(q, _bf, x), k=(k, _bf, xkv), v=(v, _bf, xkv), o=(o, _bf, x), lse=(lse, _f32, (B, H, N)))
    _check(lib.fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, N, d, int(causal), float(scale),
                          _stream(stream)), "fa_fwd_gqa")


def fa_bwd_gqa(q, k, v, o, do, lse, dq, dk, dv, causal: bool, scale: float, workspace, stream=None) -> None:
    """Grouped-query backward; dk, dv have H_kv heads (group sums)."""
    B, H, N, d = _dims(q)
    Hkv = int(k.shape[1]) if k.dim() == 4 else -1
    x, xkv = (B, H, N, d), (B, Hkv, N, d)
    _need("fa_bwd_gqa", q=(q, _bf, x), k=(k, _bf, xkv), v=(v, _bf, xkv), o=(o, _bf, x), do=(do, _bf, x),
          lse=(lse, _f32, (B, H, N)), dq=(dq, _bf, x), dk=(dk, _bf, xkv), dv=(dv, _bf, xkv),
          workspace=(workspace, _u8, (int(workspace.numel()),)))
    _check(lib.fa_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B,
                          H, Hkv, N, d, int(causal), float(scale), _ptr(workspace), int(workspace.numel()),
                          _stream(stream)), "fa_bwd_gqa")


lib.fa_decode_workspace_bytes.restype = _sz
lib.fa_decode_workspace_bytes.argtypes = [_ci] * 5
lib.fa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _ci, _ci, _ci, _ci, _ci, _cf, _vp, _sz, _vp]


def fa_decode_workspace_bytes(B: int, H: int, H_kv: int, N: int, d: int) -> int:
    return int(lib.fa_decode_workspace_bytes(B, H, H_kv, N, d))


def fa_decode(q, k, v, o, lse, scale: float, workspace, stream=None) -> None:
    """One decoding step: q, o [B,H,d]; k, v [B,H_kv,N,d]; lse [B,H]."""
    if q.dim() != 3 or k.dim() != 4:
        raise ValueError("expected q [B, H, d] and k, v [B, H_kv, N, d]")
    B, H, d = (int(x) for x in q.shape)
    Hkv, N = int(k.shape[1]), int(k.shape[2])
    _need("fa_decode", q=(q, _bf, (B, H, d)), k=(k, _bf, (B, Hkv, N, d)), v=(v, _bf, (B, Hkv, N, d)),
          o=(o, _bf, (B, H, d)), lse=(lse, _f32, (B, H)), workspace=(workspace, _u8, (int(workspace.numel()),)))
    _check(lib.fa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, N, d, float(scale),
                         _ptr(workspace), int(workspace.numel()), _stream(stream)), "fa_decode")
