"""Small helpers shared by the tests: exact bf16 encoding of hand-picked
values and hand-built DecodeInputs.  No attention arithmetic lives here."""
from __future__ import annotations

import numpy as np
import torch

from gqa_decode_attention_split_b200.synth import DecodeInputs


def bf16_bits(values) -> np.ndarray:
    """Encode values that are exactly representable in bf16 (asserted)."""
    shape = np.shape(values)
    a = np.ascontiguousarray(np.asarray(values, dtype=np.float32).reshape(-1))
    t = torch.from_numpy(a).to(torch.bfloat16)
    back = t.to(torch.float32).numpy()
    finite = np.isfinite(a)
    if not np.array_equal(back[finite], a[finite]):
        raise ValueError("value not exactly representable in bf16")
    return t.view(torch.int16).numpy().view(np.uint16).reshape(shape)


def bf16_values(bits) -> np.ndarray:
    """Decode bf16 bit patterns with torch (independent of the oracle)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def e4m3_values(codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    return torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def int4_values(packed) -> np.ndarray:
    """Signed int4 codes of packed bytes [..., n] as float64 [..., 2n]: the
    low nibble of byte i is element 2i, the high nibble element 2i + 1, each
    a two's-complement 4-bit number (decoded here with numpy shifts, apart
    from the oracle's decoder)."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = b & 15, b >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.float64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def contiguous_inputs(q, k, v, kv_lens, *, sm_scale=1.0, window=-1, name="hand") -> DecodeInputs:
    """q [B, Hq, d], k/v [rows, Hkv, d] as float values exactly representable in bf16."""
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    lens = list(kv_lens)
    indptr = np.zeros(len(lens) + 1, dtype=np.int32)
    indptr[1:] = np.cumsum(lens)
    return DecodeInputs(name=name, batch=q.shape[0], qo_heads=q.shape[1], kv_heads=k.shape[1],
                        head_dim=q.shape[2], kv_dtype="bf16", paged=False, page_size=0,
                        window=window, sm_scale=float(sm_scale), q=bf16_bits(q),
                        k=bf16_bits(k), v=bf16_bits(v), kv_indptr=indptr)


def dense_kv(x: DecodeInputs, b: int):
    """Float64 K and V rows [L_b, Hkv, d] of request b, decoded with torch
    (independent of the oracle's decoders).  Reads only the request's own
    rows/pages."""
    L = int(x.kv_indptr[b + 1] - x.kv_indptr[b])
    if x.paged:
        rows_k, rows_v = [], []
        for t in range(L):
            pg = int(x.page_table[b, t // x.page_size])
            rows_k.append(x.k[pg, t % x.page_size])
            rows_v.append(x.v[pg, t % x.page_size])
        kk = np.stack(rows_k) if L else np.zeros((0, x.kv_heads, x.k.shape[-1]), x.k.dtype)
        vv = np.stack(rows_v) if L else np.zeros((0, x.kv_heads, x.v.shape[-1]), x.v.dtype)
    else:
        a = int(x.kv_indptr[b])
        kk, vv = x.k[a:a + L], x.v[a:a + L]
    if x.kv_dtype == "fp8_e4m3":
        kf = e4m3_values(kk) * x.k_scale.astype(np.float64)[None, :, None]
        vf = e4m3_values(vv) * x.v_scale.astype(np.float64)[None, :, None]
    elif x.kv_dtype == "int4":
        kf = int4_values(kk) * x.k_scale.astype(np.float64)[None, :, None]
        vf = int4_values(vv) * x.v_scale.astype(np.float64)[None, :, None]
    else:
        kf, vf = bf16_values(kk), bf16_values(vv)
    return kf, vf


def visible(x: DecodeInputs, b: int):
    L = int(x.kv_indptr[b + 1] - x.kv_indptr[b])
    lo = max(0, L - x.window) if x.window > 0 else 0
    return lo, L
