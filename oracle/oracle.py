"""fp64 CPU oracle for GQA decode attention (Python side).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke entry point and the
benchmark's CPU-baseline leg are the only callers.  This module never imports
the CUDA library or its binding; it reads the raw input arrays of a
DecodeInputs-like object (duck-typed: q, k, v, kv_indptr, page_table, scales
and the shape fields) and calls the plain C code in decode_oracle.c, which
writes the attention definition out in double precision.

Build: ``build()`` compiles decode_oracle.c with gcc (-O2, OpenMP, no
fast-math) into liboracle.so next to this file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "decode_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle; returns the shared-library path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("qo_heads", ctypes.c_int32),
        ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("kv_kind", ctypes.c_int32), ("paged", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("page_table_stride", ctypes.c_int32),
        ("window", ctypes.c_int32), ("sm_scale", ctypes.c_double),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("kv_indptr", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
        ("q_len", ctypes.c_int32), ("logit_cap", ctypes.c_double),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_decode_all.argtypes = [P, dp, dp, ctypes.c_int]
        lib.oracle_decode_all.restype = ctypes.c_int
        lib.oracle_decode_rows.argtypes = [P, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                           dp, dp, ctypes.c_int]
        lib.oracle_decode_rows.restype = ctypes.c_int
        lib.oracle_merge.argtypes = [dp, dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, dp, dp]
        lib.oracle_merge.restype = None
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_int4_code.argtypes = [ctypes.c_uint8, ctypes.c_int]
        lib.oracle_int4_code.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _problem(x) -> Tuple[_Problem, list]:
    keep = []

    def c(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a

    kind = {"bf16": 0, "fp8_e4m3": 1, "int4": 2}[x.kv_dtype]
    quant = kind != 0
    q = c(x.q, np.uint16)
    k = c(x.k, np.uint8 if quant else np.uint16)
    v = c(x.v, np.uint8 if quant else np.uint16)
    ks = c(x.k_scale, np.float32) if quant else None
    vs = c(x.v_scale, np.float32) if quant else None
    ind = c(x.kv_indptr, np.int32)
    pt = c(x.page_table, np.int32) if x.paged else None
    p = _Problem(batch=x.batch, qo_heads=x.qo_heads, kv_heads=x.kv_heads,
                 head_dim=x.head_dim, kv_kind=kind, paged=int(bool(x.paged)),
                 page_size=int(x.page_size) if x.paged else 1,
                 page_table_stride=int(pt.shape[1]) if pt is not None else 0,
                 window=int(x.window), sm_scale=float(x.sm_scale),
                 q=_ptr(q), k=_ptr(k), v=_ptr(v), k_scale=_ptr(ks), v_scale=_ptr(vs),
                 kv_indptr=_ptr(ind), page_table=_ptr(pt), q_len=_q_len(x),
                 logit_cap=float(getattr(x, "logit_cap", 0.0) or 0.0))
    return p, keep


def _q_len(x) -> int:
    return int(getattr(x, "q_len", 1) or 1)


def _row_shape(x):
    """Leading dims of out / lse: [batch, qo_heads], or [batch, q_len,
    qo_heads] when a request has several query tokens."""
    Q = _q_len(x)
    return (x.batch, x.qo_heads) if Q == 1 else (x.batch, Q, x.qo_heads)


def decode_all(x, nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention for every (request, query token, query head).

    Returns out float64 [batch, qo_heads, head_dim] and lse float64
    [batch, qo_heads] (natural log; -inf for an empty key set); with several
    query tokens per request, [batch, q_len, qo_heads, head_dim] and
    [batch, q_len, qo_heads]."""
    lib = _load()
    p, keep = _problem(x)
    out = np.empty(_row_shape(x) + (x.head_dim,), dtype=np.float64)
    lse = np.empty(_row_shape(x), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.oracle_decode_all(ctypes.byref(p), out.ctypes.data_as(dp), lse.ctypes.data_as(dp),
                               int(nthreads))
    if rc != 0:
        raise MemoryError("oracle_decode_all failed")
    del keep
    return out, lse


def decode_rows(x, rows, nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention for selected rows r = (b * q_len + i) * qo_heads + h
    (r = b * qo_heads + h for one query token per request).

    Returns out float64 [len(rows), head_dim] and lse float64 [len(rows)]."""
    lib = _load()
    p, keep = _problem(x)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= x.batch * _q_len(x) * x.qo_heads):
        raise IndexError("row out of range")
    out = np.empty((rows.size, x.head_dim), dtype=np.float64)
    lse = np.empty((rows.size,), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.oracle_decode_rows(ctypes.byref(p), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                rows.size, out.ctypes.data_as(dp), lse.ctypes.data_as(dp),
                                int(nthreads))
    if rc != 0:
        raise MemoryError("oracle_decode_rows failed")
    del keep
    return out, lse


def merge(o_parts: np.ndarray, lse_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Exact merge of partial states: o_parts [n, rows, heads, d], lse_parts
    [n, rows, heads] (natural log).  Returns out [rows, heads, d], lse [rows, heads]."""
    lib = _load()
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, rows, heads, d = o.shape
    if l.shape != (n, rows, heads):
        raise ValueError("lse_parts shape mismatch")
    out = np.empty((rows, heads, d), dtype=np.float64)
    lse = np.empty((rows, heads), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_merge(o.ctypes.data_as(dp), l.ctypes.data_as(dp), n, rows, heads, d,
                     out.ctypes.data_as(dp), lse.ctypes.data_as(dp))
    return out, lse


def bf16_to_double(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.oracle_bf16_to_double(int(v)) for v in b.ravel()]).reshape(b.shape)


def e4m3_to_double(codes) -> np.ndarray:
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_to_double(int(v)) for v in c.ravel()]).reshape(c.shape)


def int4_codes(packed) -> np.ndarray:
    """Signed int4 codes of packed bytes [..., n] -> [..., 2n] (element 2i
    from the low nibble of byte i)."""
    lib = _load()
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    flat_b, flat_o = b.reshape(-1, b.shape[-1]), out.reshape(-1, out.shape[-1])
    for r in range(flat_b.shape[0]):
        for i in range(flat_b.shape[1]):
            flat_o[r, 2 * i] = lib.oracle_int4_code(int(flat_b[r, i]), 0)
            flat_o[r, 2 * i + 1] = lib.oracle_int4_code(int(flat_b[r, i]), 1)
    return out


def max_threads() -> int:
    return int(_load().oracle_max_threads())
