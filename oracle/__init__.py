"""Float64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and shares no code with
it.  The arithmetic lives in ``oracle.c`` (plain loops, fp64, OpenMP); this
module only marshals numpy arrays and holds the closed-form analysis formulas
of the FP8 P-cast page.

Functions and the passages they follow:

* ``attn_fwd`` / ``attn_fwd_rows`` -- O = softmax(scale Q K^T) V and the row
  logsumexp, two-pass softmax over the fully materialised score row
  ("flash-attention-trading-models", "Por que la atencion esta ligada a la
  memoria"; "FlashAttention (IT)", "Problematica dell'attention standard").
* ``attn_bwd`` -- derivatives of that definition (the pages only say the
  backward recomputes the scores, "Pase hacia atras"; the calculus is standard).
* ``attn_fwd_gqa`` / ``attn_bwd_gqa`` -- grouped-query / multi-query attention as
  attention over key/value heads repeated across each query-head group.
* ``attn_decode`` -- one decoding step: a single new query row per head against
  the whole key/value cache (the last row of causal attention).
* ``attn_fwd_fp8p`` -- tile-by-tile emulation of the E4M3 P-cast with static
  scale S and forward/reverse key-tile order ("P-Cast precision in FP8
  attention", sections 1-2).
* ``fp8_quantize`` -- E4M3 block quantisation of Q/K/V, optionally after the
  random-sign Walsh-Hadamard rotation ("flash-attention-trading-models", section
  "FA3", item 3: incoherent processing before block quantisation).
* ``e4m3`` -- round to the E4M3 grid (same page: 3-bit mantissa, 448 max,
  2^-10 rounds to zero).
* ``p_collapse_fraction``, ``collapse_threshold``, ``expected_max_normal``,
  ``dp_sawtooth`` -- the page's closed forms F(Delta,S), Delta_c, delta_k and
  d_p(S) (section 2 "Marco Teorico", "Optimizacion 2", section 3).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc into liboracle.so (next to the source)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.oracle_e4m3.restype = cd
        lib.oracle_e4m3.argtypes = [cd]
        lib.oracle_e4m3_array.argtypes = [dp, dp, ctypes.c_int64]
        lib.oracle_attn_fwd.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, cd]
        lib.oracle_attn_fwd_rows.argtypes = [dp, dp, dp, ip, ctypes.c_int64, dp, dp, ci, ci, ci, cd]
        lib.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, cd]
        lib.oracle_attn_fwd_fp8p.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, cd, cd, ci, ci, ci, ip]
        lib.oracle_fp8_quantize.argtypes = [dp, dp, dp, dp, ci, ci, ci, ci]
        lib.oracle_hadamard_rotate.argtypes = [dp, dp, dp, ctypes.c_int64, ci]
        lib.oracle_attn_decode.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, cd]
        lib.oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def attn_fwd(q, k, v, causal: bool, scale: float):
    """O [B,H,N,d] and LSE [B,H,N] (natural log), all float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale))
    return o, lse


def attn_fwd_rows(q, k, v, rows, causal: bool, scale: float):
    """Forward on sampled rows only.  ``rows`` is an int array [R, 2] of
    (flattened b*H+h, query index).  Returns O [R, d] and LSE [R]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    R = rows.shape[0]
    o = np.empty((R, d), dtype=np.float64)
    lse = np.empty((R,), dtype=np.float64)
    _load().oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), R,
                                 _ptr(o), _ptr(lse), N, d, int(causal), float(scale))
    return o, lse


def attn_bwd(q, k, v, do, causal: bool, scale: float):
    """dQ, dK, dV [B,H,N,d] float64 for the loss <O, dO>."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d,
                            int(causal), float(scale))
    return dq, dk, dv


def attn_fwd_gqa(q, k, v, causal: bool, scale: float):
    """Grouped-query attention: q [B,Hq,N,d], k and v [B,Hkv,N,d] with Hq a multiple
    of Hkv; query head h attends with key/value head h // (Hq/Hkv) (multi-query
    attention is Hkv = 1).  By definition this is attention with every key/value
    head repeated for the query heads of its group ("FlashAttention for Scalable
    Vector Architectures", "Metodologia": the shared KV head; "FlashAttention
    (IT)", "FlashAttention-2": Multi-Query Attention)."""
    g = q.shape[1] // k.shape[1]
    return attn_fwd(q, np.repeat(_f64(k), g, axis=1), np.repeat(_f64(v), g, axis=1), causal, scale)


def attn_bwd_gqa(q, k, v, do, causal: bool, scale: float):
    """Gradients of grouped-query attention: dK and dV of a key/value head are the
    sums of the repeated heads' gradients over its group."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    dq, dk, dv = attn_bwd(q, np.repeat(_f64(k), g, axis=1), np.repeat(_f64(v), g, axis=1), do, causal, scale)
    return dq, dk.reshape(B, Hkv, g, N, d).sum(axis=2), dv.reshape(B, Hkv, g, N, d).sum(axis=2)


def attn_decode(q, k, v, scale: float):
    """One decoding step: q [B,Hq,d] (one new query row per head) against all
    Nk cached keys of k, v [B,Hkv,Nk,d]; returns o [B,Hq,d], lse [B,Hq]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = np.empty_like(q)
    lse = np.empty((B, Hq), dtype=np.float64)
    _load().oracle_attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nk, d, float(scale))
    return o, lse


def attn_fwd_fp8p(q, k, v, causal: bool, scale: float, S: float, kv_order: int, Bc: int = 128, n_sink: int = 4):
    """E4M3 P-cast emulation.  Returns O, LSE and counts
    [sink_flushed, sink_total, nonsink_flushed, nonsink_total]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    counts = np.zeros(4, dtype=np.int64)
    _load().oracle_attn_fwd_fp8p(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(causal), float(scale),
                                 float(S), int(kv_order), int(Bc), int(n_sink),
                                 counts.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    return o, lse, counts


def fp8_quantize(x, signs=None, block_rows: int = 128):
    """Block-quantise [B,H,N,d] to E4M3 (scale = block amax / 448), optionally after
    the rotation x -> x diag(signs) H / sqrt(d).  Returns the dequantised values
    (code * scale, fp64, in the rotated basis when signs is given) and the scales
    [B,H,ceil(N/block_rows)]."""
    x = _f64(x)
    B, H, N, d = x.shape
    nb = (N + block_rows - 1) // block_rows
    xq = np.empty_like(x)
    sc = np.empty((B, H, nb), dtype=np.float64)
    sg = None if signs is None else _f64(signs)
    _load().oracle_fp8_quantize(_ptr(x), None if sg is None else _ptr(sg), _ptr(xq), _ptr(sc), B * H, N, d,
                                int(block_rows))
    return xq, sc


def hadamard_rotate(x, signs):
    """x diag(signs) H / sqrt(d) applied to every row (last axis) of x, fp64."""
    x = _f64(x)
    d = x.shape[-1]
    y = np.empty_like(x)
    sg = _f64(signs)
    _load().oracle_hadamard_rotate(_ptr(x.reshape(-1)), _ptr(sg), _ptr(y.reshape(-1)), x.size // d, d)
    return y


def e4m3(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448."""
    x = _f64(x)
    y = np.empty_like(x)
    _load().oracle_e4m3_array(_ptr(x.reshape(-1)), _ptr(y.reshape(-1)), x.size)
    return y


# --------------------------------------------------------------------------
# Closed forms of "P-Cast precision in FP8 attention"
# --------------------------------------------------------------------------
E4M3_ZERO_THRESHOLD = 2.0 ** -10  # values at or below this round to zero
LN_ZERO_THRESHOLD = 10.0 * math.log(2.0)  # = 6.93..., the page's 6.93


def normal_cdf(x: float) -> float:
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def expected_max_normal(k: int, n_grid: int = 200001, lim: float = 12.0) -> float:
    """delta_k: expectation of the largest of k independent standard normals,
    E[max] = int x * k * phi(x) * Phi(x)^(k-1) dx, by the trapezoid rule."""
    xs = np.linspace(-lim, lim, n_grid)
    phi = np.exp(-0.5 * xs * xs) / math.sqrt(2.0 * math.pi)
    Phi = 0.5 * (1.0 + np.vectorize(math.erf)(xs / math.sqrt(2.0)))
    f = xs * k * phi * Phi ** (k - 1)
    return float(np.trapezoid(f, xs))


def p_collapse_fraction(delta: float, S: float, delta_k: float) -> float:
    """F(Delta, S) = Phi(Delta + delta_k - 10 ln 2 - ln S): the fraction of
    non-sink P values that flush to zero under forward key order."""
    return normal_cdf(delta + delta_k - LN_ZERO_THRESHOLD - math.log(S))


def collapse_threshold(S: float, delta_k: float) -> float:
    """Delta_c = 10 ln 2 + ln S - delta_k, where F crosses one half."""
    return LN_ZERO_THRESHOLD + math.log(S) - delta_k


def dp_sawtooth(S: float) -> float:
    """d_p(S): the E4M3 quantisation step of the binade just below S, divided
    by S (the largest normalised step that a P in [0, 1] can meet)."""
    # the largest E4M3 value strictly below S sits in binade floor(log2(S^-))
    e = math.ceil(math.log2(S)) - 1
    return 2.0 ** (e - 3) / S
