"""Exact IO-aware tiled attention for NVIDIA B200 (sm_100a).

The compute lives in ``libfa.so`` (hand-written CUDA behind a C ABI, see
``include/fa.h``); ``exact_io_aware_85_b200.fa`` is the thin ctypes binding with
the same entry-point names.  Importing the package does not load the library;
touching a binding attribute does, and fails loudly if it is missing.
"""

__all__ = ["fa", "synth"]


def __getattr__(name):
    if name in ("fa_fwd", "fa_fwd_f32", "fa_bwd", "fa_fwd_fp8p", "fa_bwd_workspace_bytes", "fa_check_status",
                "fa_status_string", "lib"):
        from . import fa as _fa

        return getattr(_fa, name)
    raise AttributeError(name)
