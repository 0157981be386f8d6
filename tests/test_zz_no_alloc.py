"""fa_decode_run_static: the decode pass for callers that cannot allocate
device memory where they run attention (a runtime that owns all device memory
and hands out only input and output buffers, a plugin host, or a path that
must not synchronise the device, which cudaMalloc and cudaFree may do).  It
takes no workspace: the library's fixed device scratch is used instead.

Its output must match the fp64 oracle within the parity tolerances, and
fa_decode_run's (with a caller-allocated workspace) on the same inputs, on
consecutive calls that reuse the scratch.  Its device-side checks must be
readable through fa_decode_status_static.

This file is collected last on purpose, so that a failure here comes after
every other test has run; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

from gqa_decode_attention_split_b200 import binding, synth
from gpu_util import DeviceInputs, assert_matches, to_numpy
from oracle import oracle

pytestmark = pytest.mark.gpu

STATIC_BYTES = 4 << 20  # FA_STATIC_WORKSPACE_BYTES

CASES = [
    ("paged_gqa4_uneven", dict(batch=8, qo=32, kv=8, d=128,
                               lens=[700, 5000, 17, 2048, 1, 333, 4096, 950],
                               kw=dict(paged=True, page_size=16, unused_slot_fill="nan"))),
    ("fp8_gqa8_long", dict(batch=1, qo=64, kv=8, d=128, lens=[20000],
                           kw=dict(kv_dtype="fp8_e4m3"))),
    ("mha_window", dict(batch=2, qo=16, kv=16, d=128, lens=[3000, 64], kw=dict(window=700))),
    ("int4_gqa4_q2_paged", dict(batch=3, qo=8, kv=2, d=128, lens=[900, 40, 2100],
                                kw=dict(kv_dtype="int4", q_len=2, paged=True, page_size=32))),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_the_oracle_and_the_workspace_entry_point(case):
    import torch
    name, c = case
    x = synth.generate(c["batch"], c["qo"], c["kv"], c["d"], c["lens"], seed=31, name=name, **c["kw"])
    dev = DeviceInputs(x)
    p = dev.plan()
    assert p.workspace_bytes <= STATIC_BYTES
    ref_o, ref_l = oracle.decode_all(x)
    ws = p.new_workspace()
    ws_out, ws_lse = dev.run(p, workspace=ws)
    wo, wl = to_numpy(ws_out, ws_lse)
    assert binding.decode_status(ws) == 0
    assert_matches(wo, wl, ref_o, ref_l, what=f"{name} workspace entry point")
    for call in range(2):  # the scratch keeps the previous call's contents
        out, lse = binding.run_static(p, dev.q, dev.k, dev.v, dev.kv_indptr,
                                      page_table=dev.page_table, k_scale=dev.k_scale,
                                      v_scale=dev.v_scale)
        assert binding.decode_status_static() == 0
        torch.cuda.synchronize()
        o, l = to_numpy(out, lse)
        assert_matches(o, l, ref_o, ref_l, what=f"{name} static call {call} vs the oracle")
        assert_matches(o, l, wo, wl, what=f"{name} static call {call} vs fa_decode_run")


def test_static_scratch_reports_a_bad_page():
    """A page id outside the pool, written by the test on the host, is never
    dereferenced (its tokens read as zeros) and is reported through the
    static status call; the next clean call reports nothing."""
    import torch
    x = synth.generate(2, 8, 2, 128, [64, 64], paged=True, page_size=16, seed=25)
    good = synth.DecodeInputs(**{**x.__dict__, "page_table": x.page_table.copy()})
    x.page_table[1, 2] = x.k.shape[0] + 5  # outside the pool
    dev = DeviceInputs(x)
    p = dev.plan(path="mma")
    out, lse = binding.run_static(p, dev.q, dev.k, dev.v, dev.kv_indptr, page_table=dev.page_table)
    assert binding.decode_status_static() & 1  # FA_DEVICE_BAD_PAGE
    assert binding.decode_status_static() == 0  # cleared by the first read
    o, l = to_numpy(out, lse)
    # the request whose pages are all valid is unaffected
    one = synth.DecodeInputs(**{**x.__dict__, "batch": 1, "q": x.q[:1],
                                "kv_indptr": x.kv_indptr[:2], "page_table": x.page_table[:1]})
    ro, rl = oracle.decode_all(one)
    assert_matches(o[:1], l[:1], ro, rl, what="unaffected request")
    # a clean call after it: no flags, and the oracle's result
    gdev = DeviceInputs(good)
    out, lse = binding.run_static(p, gdev.q, gdev.k, gdev.v, gdev.kv_indptr,
                                  page_table=gdev.page_table)
    assert binding.decode_status_static() == 0
    torch.cuda.synchronize()
    o, l = to_numpy(out, lse)
    ro, rl = oracle.decode_all(good)
    assert_matches(o, l, ro, rl, what="clean call after a flagged one")


def test_static_scratch_rejects_larger_plans():
    lib = binding.load_library()
    B = 512  # 4096 (request, kv head) segments of 8 query heads x 128 dims
    p = binding.plan(B, 64, 8, 128, np.arange(B + 1, dtype=np.int32) * 100, num_sms=148)
    assert p.workspace_bytes > STATIC_BYTES
    g = 0x10000  # never dereferenced: the size check comes first
    st = lib.fa_decode_run_static(p._handle, g, g, g, B * 100, None, 0, g, None, None, g, g, None)
    assert st == 3  # FA_ERR_WORKSPACE_TOO_SMALL
    assert b"static scratch" in lib.fa_last_error()
