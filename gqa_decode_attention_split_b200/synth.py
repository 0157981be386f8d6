"""Seeded synthetic inputs for decode attention.

This module only makes input arrays: it holds none of the attention
arithmetic.  Both the CUDA path and the fp64 oracle consume exactly the
arrays produced here (raw bf16 bit patterns, e4m3 codes with per-head fp32
scales, int32 index arrays), so the two sides see bit-identical inputs.

Value recipe: i.i.d. standard normal draws from numpy's PCG64, rounded to
bf16 with round-to-nearest-even.  FP8 KV: the same normal draws, divided by a
per-kv-head scale amax/448 and rounded to e4m3 "fn" (round-to-nearest-even,
clamped to +-448); the scales are returned with the codes.  INT4 KV: the same
draws divided by a per-kv-head scale amax/7, rounded to the nearest integer
(ties to even) and clamped to [-7, 7], stored as two's-complement nibbles,
two per byte with the even element in the low nibble.  Random streams are
keyed by (seed, stream id) and generated in fixed-size chunks, so the values
do not depend on the number of threads used to draw them.

Named workloads mirror the shapes the pages discuss: a small GQA decode, a
Gemma-3-1B-shaped layer (global and 512-token sliding window, "FlashInfer x
JAX via jax-tvm-ffi", section "Applying it to Gemma 3"), a Llama-2-7B-shaped
MHA layer over growing KV ("FlashDecoding++" explainer, section "Experiments
and results": inputs 1k..32k), a batched paged decode ("Beyond the Memory
Wall", section "2. FlashInfer": paged KV), and a long-context FP8-KV decode
(same section: FP8 KV caches).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_CHUNK = 1 << 22  # elements per independently seeded chunk

# stream ids
_S_Q, _S_K, _S_V, _S_LEN, _S_PERM = 0, 1, 2, 3, 4

FP8_MAX = 448.0
INT4_MAX = 7.0
KV_DTYPES = ("bf16", "fp8_e4m3", "int4")


def _normals(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard-normal float32 draws, deterministic in (seed, stream)."""
    out = np.empty(n, dtype=np.float32)
    nch = max(1, (n + _CHUNK - 1) // _CHUNK)
    seqs = np.random.SeedSequence([seed, stream]).spawn(nch)

    def fill(i: int) -> None:
        a, b = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        if a < b:
            np.random.Generator(np.random.PCG64(seqs[i])).standard_normal(
                b - a, dtype=np.float32, out=out[a:b])

    if nch == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(max_workers=8) as ex:
            list(ex.map(fill, range(nch)))
    return out


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) and return the uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Round float32 (already within +-448) to e4m3fn codes (uint8)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).clamp_(-FP8_MAX, FP8_MAX)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@dataclass
class DecodeInputs:
    """Host-side inputs of one decode-attention call (all numpy arrays)."""
    name: str
    batch: int
    qo_heads: int
    kv_heads: int
    head_dim: int
    kv_dtype: str          # "bf16", "fp8_e4m3" or "int4" (k, v: packed bytes [..., d / 2])
    paged: bool
    page_size: int
    window: int            # <= 0: all keys
    sm_scale: float
    q: np.ndarray          # uint16 [batch, qo_heads, head_dim] ([batch, q_len, ...] if q_len > 1)
    k: np.ndarray          # contiguous [rows, kv_heads, d]; paged [pages, page_size, kv_heads, d]
    v: np.ndarray
    kv_indptr: np.ndarray  # int32 [batch + 1]
    page_table: Optional[np.ndarray] = None  # int32 [batch, stride]
    k_scale: Optional[np.ndarray] = None     # float32 [kv_heads]
    v_scale: Optional[np.ndarray] = None
    q_len: int = 1         # query tokens per request: the request's newest keys
    logit_cap: float = 0.0  # > 0: scores s become cap * tanh(s / cap)

    @property
    def group(self) -> int:
        return self.qo_heads // self.kv_heads

    @property
    def kv_rows(self) -> int:
        """Rows of K/V (contiguous) or pages in each pool (paged)."""
        return int(self.k.shape[0])

    @property
    def kv_lens(self) -> np.ndarray:
        return np.diff(self.kv_indptr.astype(np.int64))

    @property
    def elem_bytes(self) -> int:
        """Bytes per element (int4: 1, the packed byte unit; see row_bytes)."""
        return 2 if self.kv_dtype == "bf16" else 1

    @property
    def row_bytes(self) -> int:
        """Bytes of one token's row of one kv head (K or V)."""
        return {"bf16": 2 * self.head_dim, "fp8_e4m3": self.head_dim,
                "int4": self.head_dim // 2}[self.kv_dtype]

    def visible_lens(self) -> np.ndarray:
        """Keys some query token of the request sees (the union of the
        tokens' windows: the last query token's window plus the q_len - 1
        keys before it)."""
        L = self.kv_lens
        if self.window > 0:
            return np.minimum(L, self.window + self.q_len - 1)
        return L

    def kv_bytes(self) -> int:
        """Algorithmic bytes: K and V of every visible key, read once."""
        return int(self.visible_lens().sum()) * self.kv_heads * self.row_bytes * 2

    def with_window(self, window: int, name: Optional[str] = None) -> "DecodeInputs":
        """Same arrays, different window."""
        d = dict(self.__dict__)
        d["window"] = window
        d["name"] = name or f"{self.name}_w{window}"
        return DecodeInputs(**d)


def generate(batch: int, qo_heads: int, kv_heads: int, head_dim: int,
             kv_lens: Sequence[int], *, kv_dtype: str = "bf16", paged: bool = False,
             page_size: int = 16, window: int = -1, sm_scale: Optional[float] = None,
             seed: int = 0, name: str = "custom", page_order: str = "random",
             unused_slot_fill: Optional[str] = None, extra_rows: int = 0,
             q_len: int = 1, logit_cap: float = 0.0) -> DecodeInputs:
    """Draw one decode problem.

    kv_lens: per-request key counts.  paged: pool of sum(ceil(L/page_size))
    pages in a random permutation (page_order="random") or in request order
    ("sequential").  unused_slot_fill="nan" writes NaN codes into pool slots
    past each request's last key (they must never be read as values).
    extra_rows: contiguous layout only, rows of random data appended after
    the last request (tiles that run past a request read them).
    q_len: query tokens per request (q is [batch, q_len, qo_heads, head_dim]
    when q_len > 1); they are the request's q_len newest keys.
    """
    if kv_dtype not in KV_DTYPES:
        raise ValueError(kv_dtype)
    if kv_dtype == "int4" and head_dim % 2:
        raise ValueError("int4 rows hold whole bytes: head_dim must be even")
    lens = np.asarray(list(kv_lens), dtype=np.int64)
    if lens.shape != (batch,):
        raise ValueError("kv_lens must have one entry per request")
    indptr = np.zeros(batch + 1, dtype=np.int64)
    indptr[1:] = np.cumsum(lens)
    if indptr[-1] >= 2**31:
        raise ValueError("total kv length exceeds int32")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(head_dim)
    d = head_dim

    if q_len < 1:
        raise ValueError("q_len must be >= 1")
    qshape = (batch, qo_heads, d) if q_len == 1 else (batch, q_len, qo_heads, d)
    q = _to_bf16_bits(_normals(seed, _S_Q, batch * q_len * qo_heads * d)).reshape(qshape)

    page_table = None
    if paged:
        npages = [(int(L) + page_size - 1) // page_size for L in lens]
        total_pages = int(sum(npages))
        if page_order == "random":
            perm = np.random.Generator(np.random.PCG64(
                np.random.SeedSequence([seed, _S_PERM]))).permutation(max(total_pages, 1))
        else:
            perm = np.arange(max(total_pages, 1))
        stride = max(1, max(npages) if npages else 1)
        page_table = np.full((batch, stride), -1, dtype=np.int32)
        off = 0
        for b, n in enumerate(npages):
            page_table[b, :n] = perm[off:off + n]
            off += n
        shape = (max(total_pages, 1), page_size, kv_heads, d)
    else:
        shape = (int(indptr[-1]) + extra_rows, kv_heads, d)

    n_el = int(np.prod(shape))
    k_scale = v_scale = None
    if kv_dtype == "bf16":
        k = _to_bf16_bits(_normals(seed, _S_K, n_el)).reshape(shape)
        v = _to_bf16_bits(_normals(seed, _S_V, n_el)).reshape(shape)
    elif kv_dtype == "int4":
        arrs, scales = [], []
        for stream in (_S_K, _S_V):
            x = _normals(seed, stream, n_el).reshape(shape)
            amax = np.abs(x).reshape(-1, kv_heads, d).max(axis=(0, 2)).astype(np.float32)
            scale = np.where(amax > 0, amax / np.float32(INT4_MAX), np.float32(1.0)).astype(np.float32)
            x /= scale.reshape((1,) * (len(shape) - 2) + (kv_heads, 1))
            arrs.append(_pack_int4(np.clip(np.rint(x), -INT4_MAX, INT4_MAX).astype(np.int8)))
            scales.append(scale)
        k, v = arrs
        k_scale, v_scale = scales
    else:
        arrs, scales = [], []
        for stream in (_S_K, _S_V):
            x = _normals(seed, stream, n_el).reshape(shape)
            amax = np.abs(x).reshape(-1, kv_heads, d).max(axis=(0, 2)).astype(np.float32)
            scale = np.where(amax > 0, amax / np.float32(FP8_MAX), np.float32(1.0)).astype(np.float32)
            x /= scale.reshape((1,) * (len(shape) - 2) + (kv_heads, 1))
            arrs.append(_to_e4m3_codes(x).reshape(shape))
            scales.append(scale)
        k, v = arrs
        k_scale, v_scale = scales

    if paged and unused_slot_fill == "nan":
        # int4 has no NaN: the extreme code -8 in every nibble instead
        nan_code = {"bf16": np.uint16(0x7FC0), "fp8_e4m3": np.uint8(0x7F),
                    "int4": np.uint8(0x88)}[kv_dtype]
        for b in range(batch):
            L = int(lens[b])
            n = (L + page_size - 1) // page_size
            if n and L % page_size:
                pg = page_table[b, n - 1]
                k[pg, L % page_size:] = nan_code
                v[pg, L % page_size:] = nan_code

    return DecodeInputs(name=name, batch=batch, qo_heads=qo_heads, kv_heads=kv_heads,
                        head_dim=d, kv_dtype=kv_dtype, paged=paged,
                        page_size=page_size if paged else 0, window=window,
                        sm_scale=float(sm_scale), q=q, k=k, v=v,
                        kv_indptr=indptr.astype(np.int32), page_table=page_table,
                        k_scale=k_scale, v_scale=v_scale, q_len=q_len,
                        logit_cap=float(logit_cap))


def _pack_int4(codes: np.ndarray) -> np.ndarray:
    """Signed codes [..., d] (int8 in [-8, 7]) -> bytes [..., d / 2], element
    2i in the low nibble of byte i (two's complement nibbles)."""
    u = codes.astype(np.uint8) & np.uint8(0xF)
    return (u[..., 0::2] | (u[..., 1::2] << np.uint8(4))).astype(np.uint8)


def c4_lengths(seed: int = 4, batch: int = 64, lo: int = 512, hi: int = 16384) -> np.ndarray:
    """Per-request lengths of the batched paged workload: uniform in [lo, hi]."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _S_LEN])))
    return rng.integers(lo, hi, size=batch, endpoint=True)


# Named workloads: (description, factory).
def _c1():
    return generate(1, 8, 2, 64, [512], sm_scale=1.0 / 8.0, seed=1, name="gqa4_d64_L512")


def _c2_global():
    return generate(1, 4, 1, 256, [8192], seed=2, name="gemma3_1b_global_L8192")


def _c2_local():
    return _c2_global().with_window(512, name="gemma3_1b_local_w512_L8192")


def _c3(L):
    return lambda: generate(1, 32, 32, 128, [L], seed=3, name=f"llama2_7b_mha_L{L}")


def _c4():
    return generate(64, 32, 8, 128, c4_lengths(), paged=True, page_size=16, seed=4,
                    name="paged_b64_gqa4_L512-16384")


def _c4_small():
    """Same recipe as the batch-64 paged workload, first 16 requests (~0.56 GB
    of K/V: larger than L2, small enough for a many-pass profiler capture)."""
    return generate(16, 32, 8, 128, c4_lengths()[:16], paged=True, page_size=16, seed=4,
                    name="paged_b16_gqa4_L512-16384")


def _c4_q2():
    """The batch-64 paged workload with two query tokens per request (a draft
    token verified next to the regular decode token)."""
    return generate(64, 32, 8, 128, c4_lengths(), paged=True, page_size=16, seed=4, q_len=2,
                    name="paged_b64_gqa4_q2_L512-16384")


def _c4_q(q_len):
    def f():
        """The batch-64 paged workload with q_len query tokens per request
        (q_len - 1 draft tokens verified next to the decode token): 4 x q_len
        rows per segment."""
        return generate(64, 32, 8, 128, c4_lengths(), paged=True, page_size=16, seed=4, q_len=q_len,
                        name=f"paged_b64_gqa4_q{q_len}_L512-16384")
    return f


def _c4_small_q4():
    """The first 16 requests of the batch-64 paged workload with 4 query
    tokens (16 rows per segment): a profiler-sized case of the row teams."""
    return generate(16, 32, 8, 128, c4_lengths()[:16], paged=True, page_size=16, seed=4, q_len=4,
                    name="paged_b16_gqa4_q4_L512-16384")


def _c4_small_q8():
    """The first 16 requests of the batch-64 paged workload with 8 query
    tokens (32 rows per segment): a profiler-sized case of two row teams."""
    return generate(16, 32, 8, 128, c4_lengths()[:16], paged=True, page_size=16, seed=4, q_len=8,
                    name="paged_b16_gqa4_q8_L512-16384")


def _gqa16():
    """A Llama-3.1-405B-shaped layer on one of eight tensor-parallel GPUs
    (128 query / 8 kv heads in all: 16 query heads on one kv head per GPU),
    batch-64 paged decode with the same length mix."""
    return generate(64, 16, 1, 128, c4_lengths(), paged=True, page_size=16, seed=7,
                    name="llama3_405b_tp8_gqa16_paged_b64_L512-16384")


def _c3_q8():
    """Llama-2-7B-shaped MHA layer at 32k keys with eight query tokens per
    request (seven draft tokens)."""
    return generate(1, 32, 32, 128, [32768], seed=3, q_len=8, name="llama2_7b_mha_q8_L32768")


def _gemma2_softcap():
    """A Gemma-2-2B-shaped global layer (8 query / 4 kv heads, head_dim 256,
    scores scaled by 1/16) with its logit soft-cap of 50."""
    return generate(1, 8, 4, 256, [8192], seed=6, sm_scale=1.0 / 16.0, logit_cap=50.0,
                    name="gemma2_2b_softcap50_L8192")


def _c5():
    return generate(1, 64, 8, 128, [131072], kv_dtype="fp8_e4m3", seed=5,
                    name="fp8_gqa8_L131072")


def _c5_int4():
    """The long-context GQA-8 decode with an INT4 KV cache (half the bytes of
    FP8; "Beyond the Memory Wall", section "2. FlashInfer")."""
    return generate(1, 64, 8, 128, [131072], kv_dtype="int4", seed=5, name="int4_gqa8_L131072")


def _c4_int4():
    """The batch-64 paged decode with an INT4 KV cache."""
    return generate(64, 32, 8, 128, c4_lengths(), paged=True, page_size=16, seed=4,
                    kv_dtype="int4", name="int4_paged_b64_gqa4_L512-16384")


WORKLOADS = {
    "gqa4_d64_L512": _c1,
    "gemma3_1b_global_L8192": _c2_global,
    "gemma3_1b_local_w512_L8192": _c2_local,
    "llama2_7b_mha_L1024": _c3(1024),
    "llama2_7b_mha_L4096": _c3(4096),
    "llama2_7b_mha_L16384": _c3(16384),
    "llama2_7b_mha_L32768": _c3(32768),
    "paged_b64_gqa4_L512-16384": _c4,
    "paged_b16_gqa4_L512-16384": _c4_small,
    "fp8_gqa8_L131072": _c5,
    "int4_gqa8_L131072": _c5_int4,
    "int4_paged_b64_gqa4_L512-16384": _c4_int4,
    "paged_b64_gqa4_q2_L512-16384": _c4_q2,
    "paged_b64_gqa4_q4_L512-16384": _c4_q(4),
    "paged_b64_gqa4_q8_L512-16384": _c4_q(8),
    "paged_b16_gqa4_q4_L512-16384": _c4_small_q4,
    "paged_b16_gqa4_q8_L512-16384": _c4_small_q8,
    "llama3_405b_tp8_gqa16_paged_b64_L512-16384": _gqa16,
    "llama2_7b_mha_q8_L32768": _c3_q8,
    "gemma2_2b_softcap50_L8192": _gemma2_softcap,
}


def workload(name: str) -> DecodeInputs:
    return WORKLOADS[name]()
