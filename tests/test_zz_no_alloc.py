"""fa_decode_run_static: the decode pass for callers that cannot allocate
device memory (an allocator-free runtime, a plugin that only receives its
input and output buffers, a path that must not synchronise the device).  It
takes no workspace: the library's fixed device scratch is used instead.  Its
output must match fa_decode_run's (with a caller-allocated workspace) on the
same inputs, on consecutive calls that reuse the scratch.

This file is collected last on purpose, so that a failure here comes after
every other test has run; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from gqa_decode_attention_split_b200 import binding, synth
from gpu_util import DeviceInputs, assert_matches, to_numpy

pytestmark = pytest.mark.gpu

STATIC_BYTES = 4 << 20  # FA_STATIC_WORKSPACE_BYTES

CASES = [
    ("paged_gqa4_uneven", dict(batch=8, qo=32, kv=8, d=128,
                               lens=[700, 5000, 17, 2048, 1, 333, 4096, 950],
                               kw=dict(paged=True, page_size=16, unused_slot_fill="nan"))),
    ("fp8_gqa8_long", dict(batch=1, qo=64, kv=8, d=128, lens=[20000],
                           kw=dict(kv_dtype="fp8_e4m3"))),
    ("mha_window", dict(batch=2, qo=16, kv=16, d=128, lens=[3000, 64], kw=dict(window=700))),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_workspace_entry_point(case):
    import torch
    name, c = case
    x = synth.generate(c["batch"], c["qo"], c["kv"], c["d"], c["lens"], seed=31, name=name, **c["kw"])
    dev = DeviceInputs(x)
    p = dev.plan()
    assert p.workspace_bytes <= STATIC_BYTES
    ws = p.new_workspace()
    ref_out, ref_lse = dev.run(p, workspace=ws)
    ref_o, ref_l = to_numpy(ref_out, ref_lse)
    assert binding.decode_status(ws) == 0
    for call in range(2):  # the scratch keeps the previous call's contents
        out, lse = binding.run_static(p, dev.q, dev.k, dev.v, dev.kv_indptr,
                                      page_table=dev.page_table, k_scale=dev.k_scale,
                                      v_scale=dev.v_scale)
        torch.cuda.synchronize()
        o, l = to_numpy(out, lse)
        assert_matches(o, l, ref_o, ref_l, what=f"{name} static call {call}")


def test_static_scratch_rejects_larger_plans():
    lib = binding.load_library()
    B = 512  # 4096 (request, kv head) segments of 8 query heads x 128 dims
    p = binding.plan(B, 64, 8, 128, np.arange(B + 1, dtype=np.int32) * 100, num_sms=148)
    assert p.workspace_bytes > STATIC_BYTES
    g = 0x10000  # never dereferenced: the size check comes first
    st = lib.fa_decode_run_static(p._handle, g, g, g, B * 100, None, 0, g, None, None, g, g, None)
    assert st == 3  # FA_ERR_WORKSPACE_TOO_SMALL
    assert b"static scratch" in lib.fa_last_error()
