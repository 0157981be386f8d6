"""Split-KV GQA decode attention for NVIDIA B200 (sm_100a).

The compute runs in the CUDA library ``libfadecode.so`` (C ABI in
``include/fadecode.h``); this package is a thin ctypes binding over it that
marshals torch tensors into device pointers and streams.  The library is
loaded on first use and its absence is an error: there is no fallback.
"""
from .binding import (DecodePlan, FadecodeError, library_path, load_library, merge_states,
                      plan, run, decode_status, KV_BF16, KV_FP8_E4M3, PATH_AUTO, PATH_SIMT,
                      PATH_MMA)

__all__ = ["DecodePlan", "FadecodeError", "library_path", "load_library", "merge_states", "plan",
           "run", "decode_status", "KV_BF16", "KV_FP8_E4M3", "PATH_AUTO", "PATH_SIMT", "PATH_MMA"]
