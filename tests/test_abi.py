"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/fadecode.h, plans the workloads, and rejects bad
arguments with the documented status codes before touching the device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from gqa_decode_attention_split_b200 import binding, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fadecode.h")
B200_SMS = 148


@pytest.fixture(scope="module")
def lib():
    from gqa_decode_attention_split_b200 import build_lib
    build_lib.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    assert {"fa_decode_plan", "fa_decode_run", "fa_merge_states", "fa_plan_destroy",
            "fa_plan_get_info", "fa_decode_status", "fa_status_string", "fa_version"} <= names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.fa_version() >= 100


def test_selftest_wait_checks_its_arguments(lib):
    """fa_selftest_wait rejects a missing or short workspace, a limit outside
    1 ns .. 1 s and a misaligned workspace before it launches anything."""
    vp = ctypes.c_void_p
    assert lib.fa_selftest_wait(None, 256, 1000, 0, None) == 1
    assert lib.fa_selftest_wait(vp(0x1000), 255, 1000, 0, None) == 1
    assert lib.fa_selftest_wait(vp(0x1000), 256, 0, 0, None) == 1
    assert lib.fa_selftest_wait(vp(0x1000), 256, 1_000_000_001, 0, None) == 1
    assert lib.fa_selftest_wait(vp(0x1010), 256, 1000, 0, None) == 4  # FA_ERR_MISALIGNED


def test_status_strings(lib):
    for code in range(7):
        s = lib.fa_status_string(code)
        assert s and isinstance(s, bytes)
    assert lib.fa_status_string(99) == b"unknown status"


def _desc(**kw):
    base = dict(batch=1, qo_heads=8, kv_heads=2, head_dim=128, kv_dtype=0, paged=0, page_size=0,
                window=-1, sm_scale=1.0 / math.sqrt(128), path=0, num_ctas=0)
    base.update(kw)
    return binding.DecodeDesc(**base)


def _plan(lib, desc, indptr, num_sms=B200_SMS):
    ind = np.ascontiguousarray(indptr, dtype=np.int32)
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    st = lib.fa_decode_plan(ctypes.byref(desc), ind.ctypes.data, num_sms, ctypes.byref(h),
                            ctypes.byref(ws))
    return st, h, ws.value


def _info(lib, h):
    inf = binding.PlanInfo()
    assert lib.fa_plan_get_info(h, ctypes.byref(inf)) == 0
    return inf


@pytest.mark.parametrize("name", ["gqa4_d64_L512", "gemma3_1b_global_L8192",
                                  "gemma3_1b_local_w512_L8192", "llama2_7b_mha_L32768"])
def test_plans_for_named_workloads(lib, name):
    spec = {"gqa4_d64_L512": (1, 8, 2, 64, [512], -1),
            "gemma3_1b_global_L8192": (1, 4, 1, 256, [8192], -1),
            "gemma3_1b_local_w512_L8192": (1, 4, 1, 256, [8192], 512),
            "llama2_7b_mha_L32768": (1, 32, 32, 128, [32768], -1)}[name]
    B, Hq, Hk, d, lens, w = spec
    ind = np.concatenate([[0], np.cumsum(lens)])
    st, h, ws = _plan(lib, _desc(batch=B, qo_heads=Hq, kv_heads=Hk, head_dim=d, window=w), ind)
    assert st == 0
    inf = _info(lib, h)
    assert 1 <= inf.num_ctas <= B200_SMS
    assert ws == inf.workspace_bytes and ws >= 256 and ws % 256 == 0
    assert inf.smem_bytes <= 232448
    T = inf.tile_tokens
    L = lens[0]
    lo = max(0, L - w) if w > 0 else 0
    # tiles count (request, block of heads_per_tile kv heads) segments
    assert Hk % inf.heads_per_tile == 0
    assert inf.total_tiles == Hk // inf.heads_per_tile * ((L + T - 1) // T - lo // T)
    lib.fa_plan_destroy(h)


@pytest.mark.parametrize("L,d,ctas", [
    (8192, 256, 64),      # 8.4 MB in one segment: 64 runs (the per-segment cap)
    (16384, 128, 64),     # 8.4 MB: capped at 64 as well
    (131072, 128, 148),   # 67 MB: every SM gets over 256 KB, so all take part
    (1024, 128, 64),      # 0.5 MB: fewer tiles than the cap, one per block
])
def test_blocks_per_segment(lib, L, d, ctas):
    """One segment is cut into at most 64 runs (its merge stays short) unless
    its K/V give every SM at least 256 KB; a measured-table cap overrides."""
    st, h, _ = _plan(lib, _desc(qo_heads=4, kv_heads=1, head_dim=d), [0, L])
    assert st == 0
    inf = _info(lib, h)
    assert inf.path == binding.PATH_MMA
    tiles = inf.total_tiles
    assert inf.num_ctas == min(ctas, tiles), (inf.num_ctas, tiles)
    lib.fa_plan_destroy(h)
    try:
        binding.set_tuning([_row(head_dim=d, rows_min=4, rows_max=4, bytes_max=1 << 40,
                                 path=binding.PATH_MMA, max_pieces=8)])
        st, h, _ = _plan(lib, _desc(qo_heads=4, kv_heads=1, head_dim=d), [0, L])
        assert st == 0 and _info(lib, h).num_ctas == min(8, tiles)
        lib.fa_plan_destroy(h)
    finally:
        binding.set_tuning(None)


def test_plan_paged_and_fp8(lib):
    lens = synth.c4_lengths()
    ind = np.concatenate([[0], np.cumsum(lens)])
    st, h, ws = _plan(lib, _desc(batch=64, qo_heads=32, kv_heads=8, paged=1, page_size=16), ind)
    assert st == 0
    inf = _info(lib, h)
    assert inf.num_ctas == B200_SMS and inf.path == binding.PATH_MMA
    assert inf.max_partials == B200_SMS + 64 * 8
    lib.fa_plan_destroy(h)
    st, h, ws = _plan(lib, _desc(qo_heads=64, kv_heads=8, kv_dtype=1), [0, 131072])
    assert st == 0 and _info(lib, h).path == binding.PATH_MMA
    # 8 equal segments of 128-byte rows: 18 whole runs per segment, so no run
    # crosses a segment boundary (144 of the 148 SMs)
    inf = _info(lib, h)
    assert inf.heads_per_tile == 1 and inf.num_ctas == 144
    lib.fa_plan_destroy(h)
    # int4 at head_dim 128: tiles of 4 kv heads, 2 equal segments x 74 runs
    st, h, ws = _plan(lib, _desc(qo_heads=64, kv_heads=8, kv_dtype=2), [0, 131072])
    inf = _info(lib, h)
    assert st == 0 and inf.heads_per_tile == 4 and inf.num_ctas == 2 * 74
    lib.fa_plan_destroy(h)
    # the same shape in bf16 (256-byte rows) keeps equal runs over every SM
    st, h, ws = _plan(lib, _desc(qo_heads=64, kv_heads=8), [0, 131072])
    assert st == 0 and _info(lib, h).num_ctas == B200_SMS
    lib.fa_plan_destroy(h)


def test_forced_split_and_paths(lib):
    for path in (binding.PATH_SIMT, binding.PATH_MMA):
        for n in (1, 2, 7, 64):
            st, h, _ = _plan(lib, _desc(path=path, num_ctas=n), [0, 1000])
            assert st == 0
            inf = _info(lib, h)
            assert inf.num_ctas == n and inf.path == path
            lib.fa_plan_destroy(h)


@pytest.mark.parametrize("kw,indptr,code", [
    (dict(qo_heads=6, kv_heads=4), [0, 10], 1),          # group not integral
    (dict(batch=0), [0], 1),
    (dict(head_dim=96), [0, 10], 2),                     # no kernel
    (dict(kv_dtype=1, head_dim=64), [0, 10], 2),         # fp8 needs 128-byte rows
    (dict(qo_heads=32, kv_heads=2, path=1), [0, 10], 2),  # SIMT group 16
    (dict(qo_heads=64, kv_heads=1, path=2), [0, 10], 2),  # MMA group 64 (rows > 32)
    (dict(paged=1, page_size=12), [0, 10], 1),           # not a power of two
    (dict(paged=1, page_size=512), [0, 10], 1),
    (dict(sm_scale=float("nan")), [0, 10], 1),
    (dict(kv_dtype=3), [0, 10], 1),
    (dict(path=7), [0, 10], 1),
    (dict(num_ctas=-1), [0, 10], 1),
    (dict(batch=2), [0, 10, 5], 1),                      # decreasing indptr
    (dict(), [3, 10], 1),                                # indptr[0] != 0
])
def test_plan_rejects_bad_descriptions(lib, kw, indptr, code):
    st, h, _ = _plan(lib, _desc(**kw), indptr)
    assert st == code
    assert not h.value


def test_plan_null_arguments(lib):
    d = _desc()
    ind = np.array([0, 10], np.int32)
    h = ctypes.c_void_p()
    assert lib.fa_decode_plan(None, ind.ctypes.data, 148, ctypes.byref(h), None) == 1
    assert lib.fa_decode_plan(ctypes.byref(d), None, 148, ctypes.byref(h), None) == 1
    assert lib.fa_decode_plan(ctypes.byref(d), ind.ctypes.data, 148, None, None) == 1
    assert lib.fa_plan_get_info(None, None) == 1
    lib.fa_plan_destroy(None)


def test_plan_without_device_needs_sm_count(lib):
    st, h, _ = _plan(lib, _desc(), [0, 10], num_sms=0)
    if st == 0:  # a device is present
        lib.fa_plan_destroy(h)
    else:
        assert st == 5


def test_run_validates_before_touching_the_device(lib):
    st, h, ws = _plan(lib, _desc(batch=1, qo_heads=8, kv_heads=2, paged=1, page_size=16), [0, 100])
    assert st == 0
    good = 0x10000  # never dereferenced: every call below fails validation first
    args = dict(q=good, k=good, v=good, rows=8, pt=good, pts=7, ind=good, ks=None, vs=None,
                out=good, lse=good, ws=good, wsb=ws)

    def run(**kw):
        a = dict(args, **kw)
        return lib.fa_decode_run(h, a["q"], a["k"], a["v"], a["rows"], a["pt"], a["pts"],
                                 a["ind"], a["ks"], a["vs"], a["out"], a["lse"], a["ws"], a["wsb"],
                                 None)

    assert run(q=None) == 1
    assert run(out=None) == 1
    assert run(ind=None) == 1
    assert run(pt=None) == 1
    assert run(pts=0) == 1
    assert run(rows=0) == 1
    assert run(q=good + 8) == 4
    assert run(out=good + 2) == 4
    assert run(ws=good + 128) == 4
    assert run(wsb=ws - 1) == 3
    assert lib.fa_decode_run(None, good, good, good, 8, good, 7, good, None, None, good, good,
                             good, ws, None) == 1
    lib.fa_plan_destroy(h)
    # fp8 needs both scales
    st, h, ws = _plan(lib, _desc(kv_dtype=1), [0, 100])
    assert st == 0
    assert lib.fa_decode_run(h, good, good, good, 100, None, 0, good, None, good, good, good, good,
                             ws, None) == 1
    lib.fa_plan_destroy(h)


def test_merge_states_validation(lib):
    g = 0x10000
    assert lib.fa_merge_states(None, g, 2, 1, 1, 128, g, g, None) == 1
    assert lib.fa_merge_states(g, g, 0, 1, 1, 128, g, g, None) == 1
    assert lib.fa_merge_states(g, g, 2, 1, 1, 126, g, g, None) == 1
    assert lib.fa_merge_states(g + 4, g, 2, 1, 1, 128, g, g, None) == 4
    assert lib.fa_merge_states(g, g, 2, 1, 1, 128, g + 8, g, None) == 4


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setenv("FADECODE_LIBRARY", str(tmp_path / "missing.so"))
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(binding.FadecodeError):
            binding.load_library()
    finally:
        binding._lib = saved


def test_plan_with_several_query_tokens(lib):
    """q_len multiplies the rows of a segment (group * q_len <= 32 on the MMA
    dataflow) and widens the tile range by q_len - 1 keys under a window."""
    st, h, ws = _plan(lib, _desc(qo_heads=8, kv_heads=2, q_len=2), [0, 1000])
    assert st == 0
    inf = _info(lib, h)
    assert inf.path == binding.PATH_MMA
    lib.fa_plan_destroy(h)
    # rows 4 * 4 = 16 and 4 * 8 = 32: the tcgen05 dataflow (bf16, head_dim
    # 128), or row teams on the MMA dataflow when that one is asked for or
    # the unified max is on
    for q_len in (4, 8):
        st, h, ws = _plan(lib, _desc(qo_heads=8, kv_heads=2, q_len=q_len), [0, 1000])
        assert st == 0
        inf = _info(lib, h)
        assert inf.path == binding.PATH_TC and inf.tile_tokens == 128
        lib.fa_plan_destroy(h)
        for kw in (dict(path=binding.PATH_MMA), dict(unified_max=1, softmax_phi=2.0)):
            st, h, ws = _plan(lib, _desc(qo_heads=8, kv_heads=2, q_len=q_len, **kw), [0, 1000])
            assert st == 0
            assert _info(lib, h).path == binding.PATH_MMA
            lib.fa_plan_destroy(h)
    # rows 8 * 8 = 64 exceed every kernel
    st, h, ws = _plan(lib, _desc(qo_heads=16, kv_heads=2, q_len=8), [0, 1000])
    assert st == 2 and not h  # FA_ERR_UNSUPPORTED
    # window 128 with 8 query tokens: the union spans 135 keys
    st, h, ws = _plan(lib, _desc(qo_heads=1, kv_heads=1, q_len=8, window=128), [0, 4096])
    assert st == 0
    inf = _info(lib, h)
    T = inf.tile_tokens
    assert inf.total_tiles == (4096 + T - 1) // T - (4096 - 135) // T
    lib.fa_plan_destroy(h)
    for bad in (-1, 65):
        st, h, ws = _plan(lib, _desc(q_len=bad), [0, 100])
        assert st == 1  # FA_ERR_INVALID_ARG


def test_row_team_variants(lib):
    """Segments of 9..32 rows take the MMA variants whose warps hold two row
    blocks of 8 (head_dim 128): one team with 64-token tiles up to 16 rows,
    two teams with 48-token tiles up to 32, equal K and V rings; 8 rows or
    fewer keep the one-block variant."""
    cases = [(dict(qo_heads=8, kv_heads=8), 1, 64), (dict(qo_heads=16, kv_heads=1), 2, 64),
             (dict(qo_heads=32, kv_heads=8, q_len=3), 2, 64),
             (dict(qo_heads=32, kv_heads=8, q_len=8), 4, 48),
             (dict(qo_heads=32, kv_heads=1), 4, 48)]
    for kw, teams, T in cases:
        st, h, ws = _plan(lib, _desc(path=2, **kw), [0, 5000])
        assert st == 0, kw
        inf = _info(lib, h)
        assert inf.path == binding.PATH_MMA and inf.tile_tokens == T, (kw, inf.tile_tokens)
        if teams > 1:
            assert inf.stages == inf.v_stages  # equal rings
        lib.fa_plan_destroy(h)
    # SIMT keeps exact groups of at most 8 rows
    st, h, _ = _plan(lib, _desc(path=1, qo_heads=16, kv_heads=1), [0, 100])
    assert st == 2 and not h.value


def _row(**kw):
    r = dict(head_dim=128, kv_dtype=0, rows_min=1, rows_max=8, bytes_min=0, bytes_max=1 << 40,
             path=binding.PATH_SIMT, max_pieces=0)
    r.update(kw)
    return r


def test_tuning_table_drives_the_auto_choice(lib):
    """The planner takes the first table row that covers a decode (head_dim,
    dtype, rows, visible K/V bytes) when the path is AUTO and the grid is not
    forced; rows that do not cover it, or name a dataflow without a kernel,
    are passed over and the fixed rule applies."""
    builtin = binding.get_tuning()
    try:
        # 1000 keys x 2 kv heads x 2 x 256 B = 1,024,000 visible bytes
        binding.set_tuning([_row(rows_min=4, rows_max=4, bytes_max=1_024_000, max_pieces=2)])
        assert binding.get_tuning()[0]["max_pieces"] == 2
        st, h, _ = _plan(lib, _desc(), [0, 1000])
        inf = _info(lib, h)
        assert st == 0 and inf.path == binding.PATH_SIMT
        assert inf.num_ctas <= 2 * 2  # at most 2 blocks per segment on average
        lib.fa_plan_destroy(h)
        # one key more: outside the row -> fixed rule (MMA, up to 32 per segment)
        st, h, _ = _plan(lib, _desc(), [0, 1001])
        inf = _info(lib, h)
        assert inf.path == binding.PATH_MMA and inf.num_ctas > 4
        lib.fa_plan_destroy(h)
        # a window bounds the visible bytes: 1001 keys, window 1000 -> covered
        st, h, _ = _plan(lib, _desc(window=1000), [0, 1001])
        assert _info(lib, h).path == binding.PATH_SIMT
        lib.fa_plan_destroy(h)
        # forced path or forced grid: the table is not consulted
        for kw in (dict(path=binding.PATH_MMA), dict(num_ctas=7)):
            st, h, _ = _plan(lib, _desc(**kw), [0, 1000])
            assert _info(lib, h).path == binding.PATH_MMA
            lib.fa_plan_destroy(h)
        # a SIMT row for 16 rows has no kernel: passed over, the fixed rule
        # (the tcgen05 dataflow for bf16 head_dim 128) runs it
        binding.set_tuning([_row(rows_min=16, rows_max=16)])
        st, h, _ = _plan(lib, _desc(qo_heads=16, kv_heads=1), [0, 1000])
        assert st == 0 and _info(lib, h).path == binding.PATH_TC
        lib.fa_plan_destroy(h)
        # a measured MMA row for 16 rows takes precedence over it
        binding.set_tuning([_row(rows_min=16, rows_max=16, path=binding.PATH_MMA)])
        st, h, _ = _plan(lib, _desc(qo_heads=16, kv_heads=1), [0, 1000])
        assert st == 0 and _info(lib, h).path == binding.PATH_MMA
        lib.fa_plan_destroy(h)
        # an empty table: fixed rule only
        binding.set_tuning([])
        assert binding.get_tuning() == []
    finally:
        binding.set_tuning(None)
    assert binding.get_tuning() == builtin


@pytest.mark.parametrize("bad", [dict(rows_min=0), dict(rows_min=5, rows_max=4),
                                 dict(bytes_min=10, bytes_max=9), dict(bytes_min=-1),
                                 dict(path=0), dict(path=4), dict(kv_dtype=3),
                                 dict(max_pieces=-1), dict(max_pieces=1025), dict(head_dim=0)])
def test_tuning_table_rejects_bad_rows(lib, bad):
    before = binding.get_tuning()
    with pytest.raises(binding.FadecodeError):
        binding.set_tuning([_row(), _row(**bad)])
    assert binding.get_tuning() == before  # nothing installed
    n = ctypes.c_int32(0)
    assert lib.fa_set_tuning(None, 3) == 1
    assert lib.fa_get_tuning(None, 0, None) == 1
    assert lib.fa_get_tuning(None, 2, ctypes.byref(n)) == 1


def test_builtin_tuning_table_is_well_formed(lib):
    for r in binding.get_tuning():
        assert r["rows_min"] <= r["rows_max"] and r["bytes_min"] <= r["bytes_max"]
        assert r["path"] in (binding.PATH_SIMT, binding.PATH_MMA)
        assert r["head_dim"] in (64, 128, 256) and r["kv_dtype"] in (0, 1)


def test_builtin_tuning_rows_take_effect(lib):
    """Every row of the built-in (measured) table decides the plan of a
    decode inside its range: batch 1, 8 kv heads, as many keys as put the
    visible K/V bytes at the row's lower bound (or 1 MiB above zero)."""
    rows = binding.get_tuning()
    for r in rows:
        es = 1 if r["kv_dtype"] == 1 else 2
        per_key = 8 * 2 * r["head_dim"] * es
        target = max(r["bytes_min"], 1 << 20)
        L = -(-target // per_key)
        assert L * per_key <= r["bytes_max"]
        st, h, _ = _plan(lib, _desc(head_dim=r["head_dim"], kv_dtype=r["kv_dtype"], kv_heads=8,
                                    qo_heads=8 * r["rows_min"],
                                    sm_scale=1.0 / math.sqrt(r["head_dim"])), [0, L])
        assert st == 0, r
        inf = _info(lib, h)
        assert inf.path == r["path"], r
        if r["max_pieces"]:
            assert inf.num_ctas <= r["max_pieces"] * 8, r
        lib.fa_plan_destroy(h)


def test_int4_plans(lib):
    """INT4 KV runs on the MMA dataflow (head_dim 128 and 256, up to 32
    rows); SIMT has no INT4 kernel, head_dim 64 has none, an odd head_dim is
    not a whole number of bytes."""
    st, h, _ = _plan(lib, _desc(kv_dtype=binding.KV_INT4), [0, 1000])
    assert st == 0
    inf = _info(lib, h)
    assert inf.path == binding.PATH_MMA and inf.tile_tokens == 64  # 64-byte rows, 4 KB tiles
    lib.fa_plan_destroy(h)
    st, h, _ = _plan(lib, _desc(kv_dtype=binding.KV_INT4, head_dim=256, qo_heads=32, kv_heads=1),
                     [0, 1000])
    assert st == 0 and _info(lib, h).path == binding.PATH_MMA
    lib.fa_plan_destroy(h)
    # one-token pages of 64-byte rows: a copy would land off a 128-byte boundary
    for kw, code in ((dict(path=binding.PATH_SIMT), 2), (dict(head_dim=64), 2),
                     (dict(head_dim=127), 1), (dict(paged=1, page_size=1), 2)):
        st, h, _ = _plan(lib, _desc(kv_dtype=binding.KV_INT4, **kw), [0, 1000])
        assert st == code and not h.value, kw
    for ps in (2, 16):
        st, h, _ = _plan(lib, _desc(kv_dtype=binding.KV_INT4, paged=1, page_size=ps), [0, 1000])
        assert st == 0
        lib.fa_plan_destroy(h)



def test_unified_max_fields_are_validated(lib):
    """unified_max is 0 or 1; with it on, softmax_phi must be finite (a
    zero-filled descriptor keeps the plain running max)."""
    for kw, code in ((dict(unified_max=1, softmax_phi=3.0), 0), (dict(unified_max=1, softmax_phi=-1e30), 0),
                     (dict(unified_max=2), 1), (dict(unified_max=1, softmax_phi=float("nan")), 1),
                     (dict(unified_max=1, softmax_phi=float("inf")), 1),
                     (dict(unified_max=0, softmax_phi=float("nan")), 0)):
        st, h, _ = _plan(lib, _desc(**kw), [0, 100])
        assert st == code, kw
        if h.value:
            lib.fa_plan_destroy(h)


def test_head_tile_choice(lib):
    """INT4 on the MMA dataflow, one query token, at most 8 rows per head and
    a kv-head count the block divides: tiles of 256 / row-bytes heads;
    otherwise (and for bf16 / fp8) one head per tile."""
    cases = [(dict(kv_dtype=2), 4), (dict(kv_dtype=2, head_dim=256), 2),
             (dict(kv_dtype=1), 1), (dict(head_dim=64), 1), (dict(), 1),
             (dict(kv_dtype=2, q_len=2), 1), (dict(kv_dtype=2, kv_heads=1, qo_heads=4), 1),
             (dict(kv_dtype=2, kv_heads=2, qo_heads=8), 1),                # 2 heads, int4 wants 4
             (dict(kv_dtype=2, qo_heads=64), 1)]                           # 16 rows per head
    for kw, ht in cases:
        kw = {"qo_heads": 16, "kv_heads": 4, **kw}
        st, h, _ = _plan(lib, _desc(**kw), [0, 3000])
        assert st == 0, kw
        assert _info(lib, h).heads_per_tile == ht, kw
        lib.fa_plan_destroy(h)



def test_piece_cost_choice(lib):
    """The split's charge per segment: the caller's value when positive,
    none when negative; otherwise 2 tiles up to 8 rows, 4 with int4 head
    tiles, 8 with 16 or 32 rows on the MMA dataflow, 3 (128-token) tiles on
    the tcgen05 one.  Never on the segment-aligned split nor when blocks get
    a tile each; a charge above 4096 is rejected."""
    lens = np.concatenate([[0], np.cumsum([3000, 100, 9000, 40] * 16)])
    B = len(lens) - 1
    cases = [(dict(), 2), (dict(q_len=2), 2), (dict(qo_heads=32), 3), (dict(q_len=4), 3),
             (dict(qo_heads=32, path=2), 8), (dict(q_len=4, path=2), 8),
             (dict(qo_heads=16, kv_heads=4, kv_dtype=2), 4), (dict(piece_cost=5), 5),
             (dict(piece_cost=-1), 0), (dict(q_len=4, piece_cost=-7), 0),
             (dict(piece_cost=4096), 4096), (dict(path=1), 2)]
    for kw, want in cases:
        st, h, _ = _plan(lib, _desc(batch=B, **kw), lens)
        assert st == 0, kw
        assert _info(lib, h).piece_cost == want, kw
        lib.fa_plan_destroy(h)
    st, h, _ = _plan(lib, _desc(batch=B, piece_cost=4097), lens)
    assert st == 1 and not h.value
    # one block per tile: nothing to balance
    st, h, _ = _plan(lib, _desc(), [0, 300])
    assert st == 0 and _info(lib, h).piece_cost == 0
    lib.fa_plan_destroy(h)
    # equal fp8 segments of 128-byte rows: segment-aligned runs, no charge
    st, h, _ = _plan(lib, _desc(qo_heads=64, kv_heads=8, kv_dtype=1), [0, 131072])
    assert st == 0 and _info(lib, h).piece_cost == 0
    lib.fa_plan_destroy(h)


def _largest_plannable_batch(lib, **kw):
    def ok(batch):
        lens = np.full(batch, 20)
        st, h, _ = _plan(lib, _desc(batch=batch, paged=1, page_size=16, **kw),
                         np.concatenate([[0], np.cumsum(lens)]))
        if h.value:
            lib.fa_plan_destroy(h)
        assert st in (0, 2)
        return st == 0
    lo, hi = 1, 1 << 17
    assert ok(lo) and not ok(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if ok(mid) else (lo, mid)
    return lo


def test_plan_batch_limit(lib):
    """A block keeps every request's start, length and tile prefix in shared
    memory next to its tile ring: the planner accepts every batch whose
    block fits the 227 KB of shared memory and refuses larger ones as
    unsupported (never a device fault); at least 682 requests always fit."""
    for kw in (dict(), dict(kv_dtype=1), dict(path=binding.PATH_SIMT)):
        top = _largest_plannable_batch(lib, **kw)
        assert top >= 682, kw
        lens = np.full(top, 20)
        st, h, _ = _plan(lib, _desc(batch=top, paged=1, page_size=16, **kw),
                         np.concatenate([[0], np.cumsum(lens)]))
        assert st == 0 and _info(lib, h).smem_bytes <= 232448
        lib.fa_plan_destroy(h)


@pytest.mark.parametrize("q_len", [4, 8])
def test_tc_batch_limit(lib, q_len):
    """The tcgen05 dataflow keeps the schedule arrays next to its rings: it is
    chosen up to the largest batch whose block fits 227 KB of shared memory
    (at least 682 requests), and beyond it the plan is refused as
    unsupported, by both tensor-core dataflows alike (never a launch that
    cannot fit)."""
    def plan(batch, **kw):
        lens = np.concatenate([[0], np.cumsum(np.full(batch, 300))])
        return _plan(lib, _desc(batch=batch, q_len=q_len, paged=1, page_size=16, **kw), lens)
    lo, hi = 10, 20000
    while hi - lo > 1:  # the largest batch the tcgen05 dataflow takes
        mid = (lo + hi) // 2
        st, h, _ = plan(mid, path=binding.PATH_TC)
        if st == 0:
            lib.fa_plan_destroy(h)
            lo = mid
        else:
            assert st == 2 and not h.value
            hi = mid
    assert lo >= 682
    st, h, _ = plan(lo)
    inf = _info(lib, h)
    assert st == 0 and inf.path == binding.PATH_TC and inf.smem_bytes <= 232448
    lib.fa_plan_destroy(h)
    for kw in (dict(), dict(path=binding.PATH_MMA), dict(path=binding.PATH_TC)):
        st, h, _ = plan(lo + 2, **kw)
        assert st == 2 and not h.value, kw


def test_tiles_fit_the_pages(lib):
    """A paged tile is one page per box or a slice of one page, so tile and
    page lengths must divide one another: 32 rows take 48-token tiles with
    pages of 16 tokens or fewer, and the 32-token variant with 32- or
    64-token pages.  The tcgen05 dataflow copies 8 tokens at a time into
    128-token tiles: pages of 8 tokens or more; shorter pages take the MMA
    dataflow."""
    for ps, T in ((1, 48), (16, 48), (32, 32), (64, 32), (256, 32)):
        st, h, _ = _plan(lib, _desc(qo_heads=32, kv_heads=1, paged=1, page_size=ps,
                                    path=binding.PATH_MMA), [0, 3000])
        assert st == 0, ps
        inf = _info(lib, h)
        assert inf.tile_tokens == T, (ps, inf.tile_tokens)
        assert (ps % T == 0) if ps >= T else (T % ps == 0)
        lib.fa_plan_destroy(h)
    for ps, path in ((1, binding.PATH_MMA), (4, binding.PATH_MMA), (8, binding.PATH_TC),
                     (16, binding.PATH_TC), (256, binding.PATH_TC)):
        st, h, _ = _plan(lib, _desc(qo_heads=32, kv_heads=1, paged=1, page_size=ps), [0, 3000])
        assert st == 0, ps
        assert _info(lib, h).path == path, ps
        lib.fa_plan_destroy(h)
    st, h, _ = _plan(lib, _desc(qo_heads=32, kv_heads=1, paged=1, page_size=4,
                                path=binding.PATH_TC), [0, 3000])
    assert st == 2 and not h.value  # no tcgen05 kernel for 4-token pages



def test_one_block_per_segment_needs_no_merge(lib):
    """A measured cap of one block per segment gives every (request, kv head)
    segment one block and one launch per pass (no segment is ever split, so
    no merge kernel), whatever the lengths."""
    try:
        binding.set_tuning([_row(rows_min=4, rows_max=4, path=binding.PATH_MMA, max_pieces=1)])
        st, h, _ = _plan(lib, _desc(batch=3, qo_heads=8, kv_heads=2), [0, 5000, 5001, 9000])
        assert st == 0
        inf = _info(lib, h)
        assert inf.num_ctas == 3 * 2 and inf.launches == 1 and inf.piece_cost == 0
        lib.fa_plan_destroy(h)
    finally:
        binding.set_tuning(None)
    # the default cut splits segments: two launches
    st, h, _ = _plan(lib, _desc(batch=3, qo_heads=8, kv_heads=2), [0, 5000, 5001, 9000])
    inf = _info(lib, h)
    assert inf.num_ctas > 6 and inf.launches == 2
    lib.fa_plan_destroy(h)
    # one block: one launch
    st, h, _ = _plan(lib, _desc(num_ctas=1), [0, 5000])
    assert _info(lib, h).launches == 1
    lib.fa_plan_destroy(h)
