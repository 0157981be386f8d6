"""GPU-side helpers for the parity tests: move DecodeInputs to the device,
run the library through the binding (C ABI), and compare with the oracle
under the stated tolerances."""
from __future__ import annotations

import numpy as np

from gqa_decode_attention_split_b200 import binding

# Tolerances: bf16 output within max-abs 1e-2 and max-rel 1e-2 (relative error
# taken over elements with |ref| >= 1e-3; smaller ones are covered by the
# absolute bound), fp32 lse within 1e-3 absolute.
OUT_ABS = 1e-2
OUT_REL = 1e-2
REL_FLOOR = 1e-3
LSE_ABS = 1e-3


class DeviceInputs:
    def __init__(self, x, device="cuda"):
        import torch
        self.x = x
        bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)
        self.q = bits(x.q)
        if x.kv_dtype != "bf16":  # fp8 / int4 codes (bytes) with per-head scales
            self.k = torch.from_numpy(np.ascontiguousarray(x.k)).to(device)
            self.v = torch.from_numpy(np.ascontiguousarray(x.v)).to(device)
            self.k_scale = torch.from_numpy(x.k_scale).to(device)
            self.v_scale = torch.from_numpy(x.v_scale).to(device)
        else:
            self.k, self.v = bits(x.k), bits(x.v)
            self.k_scale = self.v_scale = None
        self.kv_indptr = torch.from_numpy(x.kv_indptr).to(device)
        self.page_table = (torch.from_numpy(x.page_table).to(device) if x.paged else None)

    def plan(self, path="auto", num_ctas=0, piece_cost=0):
        x = self.x
        return binding.plan(x.batch, x.qo_heads, x.kv_heads, x.head_dim, x.kv_indptr,
                            kv_dtype=x.kv_dtype, paged=x.paged, page_size=x.page_size,
                            window=x.window, sm_scale=x.sm_scale, path=path, num_ctas=num_ctas,
                            q_len=getattr(x, "q_len", 1), logit_cap=getattr(x, "logit_cap", 0.0),
                            piece_cost=piece_cost)

    def run(self, p, workspace=None, out=None, lse=None, want_lse=True):
        return binding.run(p, self.q, self.k, self.v, self.kv_indptr, page_table=self.page_table,
                           k_scale=self.k_scale, v_scale=self.v_scale, workspace=workspace,
                           out=out, lse=lse, want_lse=want_lse)


def to_numpy(out, lse):
    import torch
    o = out.view(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64) if lse is not None else None
    return o, l


def run_gpu(x, path="auto", num_ctas=0, dev=None, piece_cost=0):
    """Returns (out float64, lse float64, device flags, plan info)."""
    dev = dev or DeviceInputs(x)
    p = dev.plan(path=path, num_ctas=num_ctas, piece_cost=piece_cost)
    ws = p.new_workspace()
    out, lse = dev.run(p, workspace=ws)
    flags = binding.decode_status(ws)
    o, l = to_numpy(out, lse)
    return o, l, flags, p.info()


def assert_matches(out, lse, ref_out, ref_lse, what=""):
    out = np.asarray(out, np.float64)
    ref_out = np.asarray(ref_out, np.float64)
    assert out.shape == ref_out.shape, what
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    assert err.max() <= OUT_ABS, f"{what}: max-abs {err.max():.3e}"
    big = np.abs(ref_out) >= REL_FLOOR
    if big.any():
        rel = (err[big] / np.abs(ref_out[big])).max()
        assert rel <= OUT_REL, f"{what}: max-rel {rel:.3e}"
    if lse is not None:
        lse = np.asarray(lse, np.float64)
        ref_lse = np.asarray(ref_lse, np.float64)
        ninf = np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(lse), ninf), f"{what}: -inf lse mismatch"
        if (~ninf).any():
            le = np.abs(lse[~ninf] - ref_lse[~ninf]).max()
            assert le <= LSE_ABS, f"{what}: lse max-abs {le:.3e}"
