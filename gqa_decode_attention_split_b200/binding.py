"""ctypes binding over libfadecode.so (C ABI: include/fadecode.h).

Argument marshalling only: torch tensors become device pointers, the current
torch stream becomes the cudaStream_t, numpy/CPU tensors become host
pointers.  Every step of the decode path runs in the library's CUDA kernels.
The library is loaded on first use; a missing library raises FadecodeError
(there is no CPU or library fallback).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfadecode.so"

KV_BF16, KV_FP8_E4M3, KV_INT4 = 0, 1, 2
_KV_DTYPES = {"bf16": KV_BF16, "fp8_e4m3": KV_FP8_E4M3, "int4": KV_INT4}
PATH_AUTO, PATH_SIMT, PATH_MMA, PATH_TC = 0, 1, 2, 3
_PATH_NAMES = {"auto": PATH_AUTO, "simt": PATH_SIMT, "mma": PATH_MMA, "tc": PATH_TC}

FA_OK = 0
_STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
                 3: "FA_ERR_WORKSPACE_TOO_SMALL", 4: "FA_ERR_MISALIGNED", 5: "FA_ERR_CUDA",
                 6: "FA_ERR_DEVICE_CHECK"}


class FadecodeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        name = _STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {name}{(' - ' + detail) if detail else ''}")


# fadecode.h's FA_VERSION: the layouts of the structures below
ABI_VERSION = 300


class DecodeDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("qo_heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_dtype", ctypes.c_int32), ("paged", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("window", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("path", ctypes.c_int32),
                ("num_ctas", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("logit_cap", ctypes.c_float), ("unified_max", ctypes.c_int32),
                ("softmax_phi", ctypes.c_float), ("piece_cost", ctypes.c_int32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
                ("tile_tokens", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("total_tiles", ctypes.c_int32), ("max_partials", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_size_t), ("smem_bytes", ctypes.c_size_t),
                ("v_stages", ctypes.c_int32), ("heads_per_tile", ctypes.c_int32),
                ("piece_cost", ctypes.c_int32), ("launches", ctypes.c_int32)]


class TuningEntry(ctypes.Structure):
    """One row of the measured dataflow-choice table (fa_tuning_entry)."""
    _fields_ = [("head_dim", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("rows_min", ctypes.c_int32), ("rows_max", ctypes.c_int32),
                ("bytes_min", ctypes.c_int64), ("bytes_max", ctypes.c_int64),
                ("path", ctypes.c_int32), ("max_pieces", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    return os.environ.get("FADECODE_LIBRARY", os.path.join(_PKG, "lib", _LIB_NAME))


def load_library():
    """Load libfadecode.so and declare its signatures (raises if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise FadecodeError(5, "load_library",
                            f"{path} not found; build it with __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.fa_decode_plan.argtypes = [ctypes.POINTER(DecodeDesc), vp, i32, ctypes.POINTER(vp),
                                   ctypes.POINTER(sz)]
    lib.fa_decode_plan.restype = ctypes.c_int
    lib.fa_plan_get_info.argtypes = [vp, ctypes.POINTER(PlanInfo)]
    lib.fa_plan_get_info.restype = ctypes.c_int
    lib.fa_plan_destroy.argtypes = [vp]
    lib.fa_plan_destroy.restype = None
    lib.fa_decode_run.argtypes = [vp, vp, vp, vp, i64, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fa_decode_run.restype = ctypes.c_int
    lib.fa_decode_run_static.argtypes = [vp, vp, vp, vp, i64, vp, i32, vp, vp, vp, vp, vp, vp]
    lib.fa_decode_run_static.restype = ctypes.c_int
    lib.fa_decode_status.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_uint32), vp]
    lib.fa_decode_status.restype = ctypes.c_int
    lib.fa_decode_status_static.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
    lib.fa_decode_status_static.restype = ctypes.c_int
    lib.fa_selftest_wait.argtypes = [vp, sz, i64, i32, vp]
    lib.fa_selftest_wait.restype = ctypes.c_int
    lib.fa_merge_states.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.fa_merge_states.restype = ctypes.c_int
    lib.fa_status_string.argtypes = [ctypes.c_int]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_error.argtypes = []
    lib.fa_last_error.restype = ctypes.c_char_p
    lib.fa_set_tuning.argtypes = [ctypes.POINTER(TuningEntry), i32]
    lib.fa_set_tuning.restype = ctypes.c_int
    lib.fa_get_tuning.argtypes = [ctypes.POINTER(TuningEntry), i32, ctypes.POINTER(i32)]
    lib.fa_get_tuning.restype = ctypes.c_int
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i32
    if lib.fa_version() // 100 != ABI_VERSION // 100:
        raise RuntimeError(f"{path}: library version {lib.fa_version()}, this binding's structures "
                           f"are those of {ABI_VERSION}; rebuild the library")
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != FA_OK:
        lib = load_library()
        detail = lib.fa_status_string(status).decode()
        if status == 5:
            detail += f" [{lib.fa_last_error().decode()}]"
        raise FadecodeError(status, where, detail)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


class DecodePlan:
    """Host-side plan: the split of KV tiles over thread blocks and the
    workspace size.  Owns the C plan object."""

    def __init__(self, handle: int, desc: DecodeDesc, workspace_bytes: int):
        self._handle = ctypes.c_void_p(handle)
        self.desc = desc
        self.workspace_bytes = int(workspace_bytes)

    def info(self) -> dict:
        lib = load_library()
        inf = PlanInfo()
        _check(lib.fa_plan_get_info(self._handle, ctypes.byref(inf)), "fa_plan_get_info")
        return {f: getattr(inf, f) for f, _ in PlanInfo._fields_}

    def __del__(self):
        h = getattr(self, "_handle", None)
        if h is not None and h.value and _lib is not None:
            _lib.fa_plan_destroy(h)
            self._handle = None

    def new_workspace(self, device=None):
        """A zero-filled workspace tensor of the plan's size (256-byte aligned
        by torch's allocator)."""
        import torch
        return torch.zeros(max(self.workspace_bytes, 256), dtype=torch.uint8,
                           device=device or "cuda")


def plan(batch: int, qo_heads: int, kv_heads: int, head_dim: int, kv_indptr_host, *,
         kv_dtype: str = "bf16", paged: bool = False, page_size: int = 0, window: int = -1,
         sm_scale: Optional[float] = None, path: str = "auto", num_ctas: int = 0,
         num_sms: int = 0, q_len: int = 1, logit_cap: float = 0.0,
         softmax_phi: Optional[float] = None, piece_cost: int = 0) -> DecodePlan:
    """softmax_phi: None for the plain running max; a value turns on the
    unified max with that phi (natural-log units of the scaled score).
    piece_cost: tiles charged per segment when the runs are cut (0: the
    planner's choice, < 0: equal tiles)."""
    lib = load_library()
    ind = np.ascontiguousarray(np.asarray(
        kv_indptr_host.cpu().numpy() if hasattr(kv_indptr_host, "cpu") else kv_indptr_host,
        dtype=np.int32))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(head_dim)
    desc = DecodeDesc(batch=batch, qo_heads=qo_heads, kv_heads=kv_heads, head_dim=head_dim,
                      kv_dtype=_KV_DTYPES[kv_dtype],
                      paged=int(bool(paged)), page_size=int(page_size), window=int(window),
                      sm_scale=float(sm_scale), path=_PATH_NAMES[path], num_ctas=int(num_ctas),
                      q_len=int(q_len), logit_cap=float(logit_cap),
                      unified_max=0 if softmax_phi is None else 1,
                      softmax_phi=0.0 if softmax_phi is None else float(softmax_phi),
                      piece_cost=int(piece_cost))
    handle = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    _check(lib.fa_decode_plan(ctypes.byref(desc), ind.ctypes.data, int(num_sms),
                              ctypes.byref(handle), ctypes.byref(ws)), "fa_decode_plan")
    return DecodePlan(handle.value, desc, ws.value)


def _rows(d) -> tuple:
    """Leading dims of out / lse: [batch, qo_heads], or [batch, q_len,
    qo_heads] with several query tokens per request."""
    return (d.batch, d.qo_heads) if d.q_len <= 1 else (d.batch, d.q_len, d.qo_heads)


def run(p: DecodePlan, q, k, v, kv_indptr, *, page_table=None, k_scale=None, v_scale=None,
        out=None, lse=None, workspace=None, stream=None, want_lse: bool = True):
    """Enqueue one decode pass; returns (out, lse) torch tensors on q's device."""
    import torch
    lib = load_library()
    d = p.desc
    if out is None:
        out = torch.empty(_rows(d) + (d.head_dim,), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(_rows(d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = p.new_workspace(q.device)
    pt_stride = int(page_table.stride(0)) if page_table is not None else 0
    _check(lib.fa_decode_run(p._handle, _ptr(q), _ptr(k), _ptr(v), int(k.shape[0]),
                             _ptr(page_table), pt_stride, _ptr(kv_indptr), _ptr(k_scale),
                             _ptr(v_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                             int(workspace.numel() * workspace.element_size()),
                             _stream_handle(stream)), "fa_decode_run")
    return out, lse


def run_static(p: DecodePlan, q, k, v, kv_indptr, *, page_table=None, k_scale=None,
               v_scale=None, out=None, lse=None, stream=None, want_lse: bool = True):
    """Like run(), through fa_decode_run_static: no workspace, the library's
    fixed device scratch is used (for callers that cannot allocate; the
    output tensors here are allocated only when not passed in)."""
    import torch
    lib = load_library()
    d = p.desc
    if out is None:
        out = torch.empty(_rows(d) + (d.head_dim,), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(_rows(d), dtype=torch.float32, device=q.device)
    pt_stride = int(page_table.stride(0)) if page_table is not None else 0
    st = lib.fa_decode_run_static(p._handle, _ptr(q), _ptr(k), _ptr(v), int(k.shape[0]),
                                  _ptr(page_table), pt_stride, _ptr(kv_indptr), _ptr(k_scale),
                                  _ptr(v_scale), _ptr(out), _ptr(lse), _stream_handle(stream))
    if st != FA_OK:
        raise FadecodeError(st, "fa_decode_run_static",
                            f"{lib.fa_status_string(st).decode()} [{lib.fa_last_error().decode()}]")
    return out, lse


def decode_status(workspace, stream=None) -> int:
    """Synchronise and return (then clear) the device-side check bits."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.fa_decode_status(_ptr(workspace), int(workspace.numel() * workspace.element_size()),
                              ctypes.byref(flags), _stream_handle(stream))
    if st not in (FA_OK, 6):
        _check(st, "fa_decode_status")
    return int(flags.value)


def selftest_wait(workspace, limit_ns: int, arrive: bool, stream=None) -> None:
    """fa_selftest_wait: one bounded wait on the device, ended by an arrival
    (arrive=True) or by its time limit, which it then records in the
    workspace header as a pipeline wait that gave up."""
    lib = load_library()
    _check(lib.fa_selftest_wait(_ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                int(limit_ns), 1 if arrive else 0, _stream_handle(stream)),
           "fa_selftest_wait")


def decode_status_static(stream=None) -> int:
    """Synchronise and return (then clear) the device-side check bits of the
    fixed scratch used by run_static (fa_decode_status_static)."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.fa_decode_status_static(ctypes.byref(flags), _stream_handle(stream))
    if st not in (FA_OK, 6):
        _check(st, "fa_decode_status_static")
    return int(flags.value)


def merge_states(o_parts, lse_parts, *, out=None, lse=None, stream=None) -> Tuple:
    """Exact merge of partial states: o_parts fp32 [n, rows, heads, d],
    lse_parts fp32 [n, rows, heads] -> (out bf16 [rows, heads, d], lse fp32)."""
    import torch
    lib = load_library()
    n, rows, heads, d = (int(s) for s in o_parts.shape)
    if out is None:
        out = torch.empty((rows, heads, d), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((rows, heads), dtype=torch.float32, device=o_parts.device)
    _check(lib.fa_merge_states(_ptr(o_parts), _ptr(lse_parts), n, rows, heads, d, _ptr(out),
                               _ptr(lse), _stream_handle(stream)), "fa_merge_states")
    return out, lse


_TUNING_FIELDS = [f for f, _ in TuningEntry._fields_]


def get_tuning() -> list:
    """The active dataflow-choice table as a list of dicts."""
    lib = load_library()
    n = ctypes.c_int32(0)
    _check(lib.fa_get_tuning(None, 0, ctypes.byref(n)), "fa_get_tuning")
    arr = (TuningEntry * max(n.value, 1))()
    _check(lib.fa_get_tuning(arr, n.value, ctypes.byref(n)), "fa_get_tuning")
    return [{f: getattr(arr[i], f) for f in _TUNING_FIELDS} for i in range(n.value)]


def set_tuning(rows) -> None:
    """Install a dataflow-choice table (list of dicts with the fields of
    TuningEntry; path and kv_dtype as the C enum values); None restores the
    built-in table."""
    lib = load_library()
    if rows is None:
        _check(lib.fa_set_tuning(None, 0), "fa_set_tuning")
        return
    arr = (TuningEntry * max(len(rows), 1))()
    for i, r in enumerate(rows):
        for f in _TUNING_FIELDS:
            setattr(arr[i], f, int(r[f]))
    _check(lib.fa_set_tuning(arr, len(rows)), "fa_set_tuning")

