"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle,
element by element, on seeded inputs.  Small cases span several KV tiles and
a ragged tail; the full-size workloads run in the launch configuration the
benchmark times and are checked on sampled (request, head) rows."""
import zlib

import numpy as np
import pytest

from gqa_decode_attention_split_b200 import binding, synth
from gpu_util import LSE_ABS, DeviceInputs, assert_matches, run_gpu, to_numpy
from oracle import oracle

pytestmark = pytest.mark.gpu

PATHS = ["simt", "mma"]


def _has_path(x, path):
    """Whether a kernel exists: rows per segment (group x query tokens) of
    1, 2, 4 or 8 on SIMT (no int4), up to 32 on MMA."""
    rows = x.group * x.q_len
    if path == "simt":
        return x.kv_dtype != "int4" and rows in (1, 2, 4, 8)
    return rows <= 32


def _check(x, path="auto", num_ctas=0, what="", piece_cost=0, ref=None):
    ref_out, ref_lse = ref if ref is not None else oracle.decode_all(x)
    out, lse, flags, info = run_gpu(x, path=path, num_ctas=num_ctas, piece_cost=piece_cost)
    assert flags == 0, f"{what}: device flags {flags}"
    assert_matches(out, lse, ref_out, ref_lse,
                   what=f"{x.name} {path} ctas={num_ctas} cost={piece_cost} {what}")
    return out, lse, info


SMALL = [
    # (name, batch, qo, kv, d, lens, kw)
    ("gqa4_d64", 1, 8, 2, 64, [517], {}),
    ("mha_d128", 2, 4, 4, 128, [301, 77], {}),
    ("gqa8_d128", 2, 16, 2, 128, [1000, 33], {}),
    ("gqa4_d256", 1, 4, 1, 256, [777], {}),
    ("gqa2_d128_win", 3, 4, 2, 128, [500, 37, 1], {"window": 45}),
    ("gqa3_d128", 2, 6, 2, 128, [129, 300], {}),
    ("gqa5_d64", 1, 5, 1, 64, [250], {}),
    ("fp8_gqa8", 1, 16, 2, 128, [1111], {"kv_dtype": "fp8_e4m3"}),
    ("fp8_gqa4_d256", 2, 8, 2, 256, [333, 64], {"kv_dtype": "fp8_e4m3"}),
    ("fp8_mha", 1, 4, 4, 128, [257], {"kv_dtype": "fp8_e4m3", "window": 100}),
    ("paged16_gqa4", 4, 8, 2, 128, [40, 16, 1, 300], {"paged": True, "page_size": 16}),
    ("paged1_gqa4", 2, 8, 2, 128, [70, 9], {"paged": True, "page_size": 1}),
    ("paged4_d64", 2, 8, 2, 64, [70, 33], {"paged": True, "page_size": 4}),
    ("paged64_d256", 2, 4, 1, 256, [200, 65], {"paged": True, "page_size": 64}),
    ("paged256_fp8", 2, 16, 2, 128, [600, 20], {"paged": True, "page_size": 256,
                                                 "kv_dtype": "fp8_e4m3"}),
    ("paged8_fp8_win", 3, 8, 8, 128, [90, 8, 150], {"paged": True, "page_size": 8,
                                                     "kv_dtype": "fp8_e4m3", "window": 17}),
    # INT4 KV (64-byte rows at head_dim 128, 128-byte rows at 256)
    ("int4_gqa8", 1, 16, 2, 128, [1111], {"kv_dtype": "int4"}),
    ("int4_gqa4_d256", 2, 8, 2, 256, [333, 64], {"kv_dtype": "int4"}),
    ("int4_mha_win", 1, 4, 4, 128, [257], {"kv_dtype": "int4", "window": 100}),
    ("int4_gqa3", 2, 6, 2, 128, [129, 300], {"kv_dtype": "int4"}),
    ("paged16_int4", 4, 8, 2, 128, [40, 16, 1, 300], {"paged": True, "page_size": 16,
                                                      "kv_dtype": "int4"}),
    ("paged2_int4", 2, 8, 2, 128, [70, 9], {"paged": True, "page_size": 2, "kv_dtype": "int4"}),
    ("paged64_int4_d256_win", 2, 4, 1, 256, [200, 65], {"paged": True, "page_size": 64,
                                                        "kv_dtype": "int4", "window": 70}),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("path", PATHS)
def test_small_cases(case, path):
    name, B, Hq, Hk, d, lens, kw = case
    kw = dict(kw)
    x = synth.generate(B, Hq, Hk, d, lens, seed=zlib.crc32(name.encode()) % 1000, name=name,
                       unused_slot_fill="nan" if kw.get("paged") else None,
                       extra_rows=0 if kw.get("paged") else 40, **kw)
    if not _has_path(x, path):
        pytest.skip("no kernel for this group on this path")
    _check(x, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_empty_and_degenerate_requests(path):
    x = synth.generate(5, 8, 2, 128, [0, 1, 0, 17, 16], seed=21, extra_rows=16)
    _check(x, path=path)
    y = x.with_window(1)
    _check(y, path=path, what="window 1")
    z = synth.generate(2, 8, 2, 128, [0, 0], seed=22, extra_rows=8)
    out, lse, flags, _ = run_gpu(z, path=path)
    assert flags == 0 and (out == 0).all() and np.isneginf(lse).all()


@pytest.mark.parametrize("path", PATHS)
def test_forced_splits_agree(path):
    """Splitting the KV sequence over more blocks, then merging, gives the
    oracle's result at every granularity (one block up to one tile per block)."""
    x = synth.generate(2, 8, 2, 128, [1500, 203], seed=23)
    results = []
    total = None
    for n in (1, 2, 7, 64, 0):
        out, lse, info = _check(x, path=path, num_ctas=n)
        total = info["total_tiles"]
        results.append((out, lse))
    out, lse, info = _check(x, path=path, num_ctas=total)
    results.append((out, lse))
    for o, l in results[1:]:
        assert np.abs(l - results[0][1]).max() <= 2e-5
        assert np.abs(o - results[0][0]).max() <= 4e-3


# Lengths that put cuts inside segments' charges: empty requests, one-key
# requests and lengths around tile edges among long ones.
COST_LENS = [1500, 0, 40, 1, 0, 700, 63, 64, 65, 0, 2000, 17]


@pytest.mark.parametrize("path", PATHS)
def test_piece_cost_splits_agree(path):
    """A split that charges every segment a fixed cost in tile units ahead of
    its tiles moves the cuts (a block that starts more segments takes fewer
    tiles; a run may end inside a segment's charge, and empty requests carry
    a charge but no tile) and gives the oracle's result at every charge and
    grid, up to a charge so large that most blocks hold no tile."""
    x = synth.generate(len(COST_LENS), 8, 2, 128, COST_LENS, seed=31)
    ref = oracle.decode_all(x)
    for cost in (-1, 1, 3, 17, 4096):
        for n in (0, 5, 37):
            _, _, info = _check(x, path=path, num_ctas=n, piece_cost=cost, ref=ref)
            if cost > 0 and n > 0:
                assert info["piece_cost"] == cost


@pytest.mark.parametrize("kw", [
    {"q_len": 4},
    {"q_len": 2, "window": 50, "paged": True, "page_size": 16},
    {"kv_dtype": "fp8_e4m3", "paged": True, "page_size": 32},
    {"kv_dtype": "int4"},
], ids=["q4_rows16", "q2_win_paged", "fp8_paged", "int4_head_tiles"])
def test_piece_cost_variants(kw):
    """The charged split on the row-team, paged, fp8 and int4 head-tile
    variants, with the planner's own charge and with forced ones."""
    kv = 4 if kw.get("kv_dtype") == "int4" else 2
    x = synth.generate(len(COST_LENS), 4 * kv, kv, 128, COST_LENS, seed=32, **kw)
    ref = oracle.decode_all(x)
    for cost in (0, 2, 9):
        for n in (0, 11):
            _check(x, path="mma", num_ctas=n, piece_cost=cost, ref=ref)


@pytest.mark.parametrize("window", [-1, 1500])
def test_segment_aligned_split(window):
    """Equal segments of 128-byte rows are cut into whole runs per segment
    (here 41 tiles into 18 runs of 2 or 3 tiles, with a ragged last tile)."""
    x = synth.generate(1, 64, 8, 128, [2597], kv_dtype="fp8_e4m3", window=window, seed=28)
    out, lse, info = _check(x, path="mma")
    if window < 0:
        assert info["num_ctas"] == 8 * 18
    # int4 with tiles of 4 kv heads: 2 segments (81 tiles each) x 74 runs
    y = synth.generate(1, 64, 8, 128, [5141], kv_dtype="int4", window=window * 2, seed=28)
    out, lse, info = _check(y, path="mma")
    if window < 0:
        assert info["heads_per_tile"] == 4 and info["num_ctas"] == 2 * 74


def test_paged_equals_contiguous_on_gpu():
    x = synth.generate(3, 16, 2, 128, [250, 31, 1024], seed=24)
    ps = 16
    npg = [(int(L) + ps - 1) // ps for L in x.kv_lens]
    perm = np.random.default_rng(5).permutation(sum(npg))
    kp = np.full((sum(npg), ps, 2, 128), 0x7FC0, np.uint16)
    vp = kp.copy()
    pt = np.full((3, max(npg)), -1, np.int32)
    off = 0
    for b in range(3):
        a = int(x.kv_indptr[b])
        for t in range(int(x.kv_lens[b])):
            kp[perm[off + t // ps], t % ps] = x.k[a + t]
            vp[perm[off + t // ps], t % ps] = x.v[a + t]
        pt[b, :npg[b]] = perm[off:off + npg[b]]
        off += npg[b]
    y = synth.DecodeInputs(**{**x.__dict__, "paged": True, "page_size": ps, "k": kp, "v": vp,
                              "page_table": pt})
    for path in PATHS:
        o1, l1, f1, _ = run_gpu(x, path=path, num_ctas=5)
        o2, l2, f2, _ = run_gpu(y, path=path, num_ctas=5)
        assert f1 == 0 and f2 == 0
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("path", PATHS)
def test_one_block_per_segment(path):
    """With a measured cap of one block per segment the pass is one launch
    and every segment is computed whole by one block: the oracle's result,
    also when the device lengths are not the plan's (shorter requests)."""
    x = synth.generate(4, 8, 2, 128, [700, 1, 0, 2300], seed=37, paged=True, page_size=16)
    try:
        binding.set_tuning([dict(head_dim=128, kv_dtype=0, rows_min=4, rows_max=4, bytes_min=0,
                                 bytes_max=1 << 40, path=binding.PATH_SIMT if path == "simt"
                                 else binding.PATH_MMA, max_pieces=1)])
        dev = DeviceInputs(x)
        p = dev.plan()
        info = p.info()
        assert info["launches"] == 1 and info["num_ctas"] == 8
        ws = p.new_workspace()
        o, l = to_numpy(*dev.run(p, workspace=ws))
        assert binding.decode_status(ws) == 0
        ref_out, ref_lse = oracle.decode_all(x)
        assert_matches(o, l, ref_out, ref_lse, what=f"one block per segment {path}")
        # shorter requests on the device than at planning time
        import torch
        short = np.array([0, 300, 301, 301, 1001], dtype=np.int32)
        dev.kv_indptr.copy_(torch.from_numpy(short))
        y = synth.DecodeInputs(**{**x.__dict__, "kv_indptr": short})
        o, l = to_numpy(*dev.run(p, workspace=ws))
        assert binding.decode_status(ws) == 0
        ref_out, ref_lse = oracle.decode_all(y)
        assert_matches(o, l, ref_out, ref_lse, what=f"one block per segment, shorter {path}")
    finally:
        binding.set_tuning(None)


def test_bad_page_id_is_flagged_not_read():
    x = synth.generate(2, 8, 2, 128, [64, 64], paged=True, page_size=16, seed=25)
    x.page_table[1, 2] = x.k.shape[0] + 5  # outside the pool
    out, lse, flags, _ = run_gpu(x, path="mma")
    assert flags & 1
    ref_out, ref_lse = oracle.decode_all(synth.DecodeInputs(**{**x.__dict__, "batch": 1,
                                                               "q": x.q[:1],
                                                               "kv_indptr": x.kv_indptr[:2],
                                                               "page_table": x.page_table[:1]}))
    assert_matches(out[:1], lse[:1], ref_out, ref_lse, what="unaffected request")


def test_status_word_is_reported_and_cleared():
    """fa_decode_status returns the check bits found in the workspace header
    and clears them, and a pass into that workspace still computes the right
    result.  The bits (a timeout and its record) are written by the test:
    no fault or timeout is provoked on the device."""
    import torch
    x = synth.generate(1, 8, 2, 128, [300], seed=27)
    dev = DeviceInputs(x)
    p = dev.plan(num_ctas=4)
    ws = p.new_workspace()
    hdr = ws[:64].view(torch.int32)
    hdr[0] = 2       # FA_DEVICE_TIMEOUT
    hdr[8] = 3       # timeout site: a consumer's wait on a full stage
    hdr[9] = 7       # its block
    assert binding.decode_status(ws) == 2
    torch.cuda.synchronize()
    # the whole header is cleared: a record left behind would keep the next
    # timeout from being recorded (a record is written only into a clear slot)
    assert int(hdr.abs().sum()) == 0
    assert binding.decode_status(ws) == 0   # cleared by the first read
    out, lse = dev.run(p, workspace=ws)
    o, l = to_numpy(out, lse)
    ref_out, ref_lse = oracle.decode_all(x)
    assert_matches(o, l, ref_out, ref_lse, what="after a reported status")
    assert binding.decode_status(ws) == 0


def test_bounded_wait_gives_up_and_is_reported():
    """The failure path on the device: a wait that nothing ends gives up after
    its limit (the kernels' own bounded wait, 50 ms here), records itself in
    the workspace header as a pipeline wait that timed out, and
    fa_decode_status reports and clears it; the context stays usable.  No
    fault is provoked: the wait is bounded by the global timer."""
    import time
    import torch
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    binding.selftest_wait(ws, 50_000_000, arrive=True)  # ended by an arrival
    assert binding.decode_status(ws) == 0
    t0 = time.perf_counter()
    binding.selftest_wait(ws, 50_000_000, arrive=False)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    hdr = ws[:64].view(torch.int32).cpu().numpy()
    assert hdr[0] == 2 and hdr[8] == 99 and hdr[9] == 0 and hdr[10] == 0  # FA_DEVICE_TIMEOUT, site, block, warp
    assert waited >= 0.045, waited
    assert binding.decode_status(ws) == 2
    assert int(ws.sum()) == 0 and binding.decode_status(ws) == 0
    # a pass after it computes the right result
    x = synth.generate(2, 8, 2, 128, [500, 70], seed=29)
    out, lse, flags, _ = run_gpu(x)
    ref_out, ref_lse = oracle.decode_all(x)
    assert flags == 0
    assert_matches(out, lse, ref_out, ref_lse, what="after a timed-out wait")


def test_lse_optional_and_workspace_reuse():
    x = synth.generate(2, 8, 2, 128, [700, 900], seed=26)
    dev = DeviceInputs(x)
    p = dev.plan(num_ctas=16)
    ws = p.new_workspace()
    ref_out, ref_lse = oracle.decode_all(x)
    for _ in range(3):  # the workspace keeps the previous call's records and partials
        out, lse = dev.run(p, workspace=ws)
        o, l = to_numpy(out, lse)
        assert_matches(o, l, ref_out, ref_lse, what="reuse")
    out, lse = dev.run(p, workspace=ws, want_lse=False)
    assert lse is None
    o, _ = to_numpy(out, None)
    assert_matches(o, None, ref_out, None, what="no lse")
    assert binding.decode_status(ws) == 0


def test_merge_states_kernel():
    import torch
    rng = np.random.default_rng(27)
    n, rows, heads, d = 5, 3, 4, 128
    o = rng.standard_normal((n, rows, heads, d)).astype(np.float32)
    l = (3 * rng.standard_normal((n, rows, heads))).astype(np.float32)
    l[1, 0, 0] = -np.inf
    l[:, 2, 3] = -np.inf
    ref_o, ref_l = oracle.merge(o.astype(np.float64), l.astype(np.float64))
    out, lse = binding.merge_states(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda())
    go, gl = to_numpy(out, lse)
    assert_matches(go, gl, ref_o, ref_l, what="merge_states")
    assert (go[2, 3] == 0).all() and np.isneginf(gl[2, 3])


# ---------------------------------------------------------------- full size
def _sample_rows(x, n, rng):
    rows = rng.choice(x.batch * x.qo_heads, size=min(n, x.batch * x.qo_heads), replace=False)
    return np.sort(rows)


def _check_full(x, path="auto", nrows=48, seed=0):
    dev = DeviceInputs(x)
    p = dev.plan(path=path)
    ws = p.new_workspace()
    out, lse = dev.run(p, workspace=ws)
    o, l = to_numpy(out, lse)
    assert binding.decode_status(ws) == 0
    rows = _sample_rows(x, nrows, np.random.default_rng(seed))
    ref_o, ref_l = oracle.decode_rows(x, rows)
    b, h = rows // x.qo_heads, rows % x.qo_heads
    assert_matches(o[b, h], l[b, h], ref_o, ref_l, what=f"{x.name} {path} sampled")
    return p.info()


@pytest.mark.parametrize("name", ["gqa4_d64_L512", "gemma3_1b_global_L8192",
                                  "gemma3_1b_local_w512_L8192", "llama2_7b_mha_L1024",
                                  "llama2_7b_mha_L4096"])
@pytest.mark.parametrize("path", PATHS)
def test_full_size_small_workloads(name, path):
    x = synth.workload(name)
    ref_o, ref_l = oracle.decode_all(x)
    out, lse, flags, _ = run_gpu(x, path=path)
    assert flags == 0
    assert_matches(out, lse, ref_o, ref_l, what=f"{name} {path}")


@pytest.mark.parametrize("path", PATHS)
def test_full_size_llama2_32k(path):
    _check_full(synth.workload("llama2_7b_mha_L32768"), path=path, nrows=32)


@pytest.fixture(scope="module")
def paged_workload():
    return synth.workload("paged_b64_gqa4_L512-16384")


@pytest.mark.parametrize("path", PATHS)
def test_full_size_batched_paged(paged_workload, path):
    x = paged_workload
    info = _check_full(x, path=path, nrows=96, seed=1)
    assert info["num_ctas"] > 1


@pytest.mark.parametrize("path", ["mma"])
def test_full_size_fp8_long_context(path):
    _check_full(synth.workload("fp8_gqa8_L131072"), path=path, nrows=24, seed=2)


# ------------------------------------------------------ several query tokens
MULTI = [
    # (name, batch, qo, kv, d, lens, kw)
    ("q2_gqa4_paged", 3, 8, 2, 128, [300, 2, 65], {"q_len": 2, "paged": True, "page_size": 16}),
    ("q8_mha_d64_win", 2, 4, 4, 64, [500, 9], {"q_len": 8, "window": 100}),
    ("q4_gqa2_d256", 2, 8, 4, 256, [700, 40], {"q_len": 4}),
    ("q4_gqa2_fp8_paged", 2, 16, 8, 128, [333, 70], {"q_len": 4, "kv_dtype": "fp8_e4m3",
                                                     "paged": True, "page_size": 32}),
    ("q4_short_request", 2, 2, 1, 128, [2, 90], {"q_len": 4}),
    # more than 8 rows: two or four row teams on the MMA dataflow
    ("q3_gqa4_d64_rows12", 2, 8, 2, 64, [260, 31], {"q_len": 3}),
    ("q4_gqa4_paged_rows16", 3, 8, 2, 128, [300, 2, 65], {"q_len": 4, "paged": True, "page_size": 16}),
    ("q8_gqa4_paged_rows32", 3, 8, 2, 128, [411, 17, 96], {"q_len": 8, "paged": True,
                                                           "page_size": 16}),
    ("q8_gqa4_paged32_rows32", 3, 8, 2, 128, [411, 17, 96], {"q_len": 8, "paged": True,
                                                             "page_size": 32}),
    ("gqa32_paged64_rows32", 2, 32, 1, 128, [700, 130], {"paged": True, "page_size": 64}),
    ("q8_gqa4_fp8_win_rows32", 2, 8, 2, 128, [700, 50], {"q_len": 8, "kv_dtype": "fp8_e4m3",
                                                         "window": 200}),
    ("q2_gqa8_fp8_paged_rows16", 2, 16, 2, 128, [333, 70], {"q_len": 2, "kv_dtype": "fp8_e4m3",
                                                            "paged": True, "page_size": 32}),
    ("gqa16_d128_rows16", 1, 16, 1, 128, [2000], {}),
    ("gqa32_d256_rows32", 1, 32, 1, 256, [900], {}),
    ("q4_gqa8_d256_fp8_rows32", 1, 16, 2, 256, [530], {"q_len": 4, "kv_dtype": "fp8_e4m3"}),
    ("q2_gqa4_int4_paged", 3, 8, 2, 128, [300, 2, 65], {"q_len": 2, "paged": True,
                                                        "page_size": 16, "kv_dtype": "int4"}),
    ("q8_gqa4_int4_win_rows32", 2, 8, 2, 128, [700, 50], {"q_len": 8, "kv_dtype": "int4",
                                                          "window": 200}),
    ("q4_gqa4_int4_d256_rows16", 1, 8, 2, 256, [530], {"q_len": 4, "kv_dtype": "int4"}),
]


@pytest.mark.parametrize("case", MULTI, ids=[c[0] for c in MULTI])
@pytest.mark.parametrize("path", PATHS)
def test_several_query_tokens(case, path):
    name, B, Hq, Hk, d, lens, kw = case
    x = synth.generate(B, Hq, Hk, d, lens, seed=zlib.crc32(name.encode()) & 0xFFFF, name=name, **kw)
    if not _has_path(x, path):
        pytest.skip("no kernel for these rows on this path")
    _check(x, path=path)


@pytest.mark.parametrize("path", PATHS)
def test_several_query_tokens_forced_splits_agree(path):
    x = synth.generate(2, 4, 2, 128, [1500, 203], q_len=4, seed=29, window=700)
    _forced_splits_agree(x, path)


@pytest.mark.parametrize("q_len", [3, 8])
def test_row_teams_forced_splits_agree(q_len):
    """12 and 32 rows (two and four row teams): any split of the tiles over
    blocks merges to the same result."""
    x = synth.generate(2, 16, 4, 128, [1500, 203], q_len=q_len, seed=31, paged=True, page_size=16)
    _forced_splits_agree(x, "mma")


def _forced_splits_agree(x, path):
    results = []
    for n in (1, 7, 64, 0):
        out, lse, info = _check(x, path=path, num_ctas=n)
        results.append((out, lse))
    for o, l in results[1:]:
        assert np.abs(l - results[0][1]).max() <= 2e-5
        assert np.abs(o - results[0][0]).max() <= 4e-3


@pytest.mark.parametrize("q_len", [2, 8])
def test_several_query_tokens_full_size_batched_paged(q_len):
    """The batch-64 paged workload with 2 query tokens per request (one draft
    token being verified; 8 rows per segment) and with 8 (32 rows, four row
    teams), sampled rows against the oracle."""
    lens = synth.c4_lengths()
    x = synth.generate(64, 32, 8, 128, lens, paged=True, page_size=16, seed=4, q_len=q_len,
                       name=f"paged_b64_gqa4_q{q_len}")
    out, lse, flags, info = run_gpu(x)
    # 8 rows: the warp-level MMA dataflow; 32 rows: the tcgen05 one
    assert flags == 0 and info["path"] == (binding.PATH_MMA if q_len == 2 else binding.PATH_TC)
    rng = np.random.default_rng(5)
    per = q_len * 32
    rows = np.sort(rng.choice(64 * per, 48, replace=False))
    ro, rl = oracle.decode_rows(x, rows)
    b, rem = rows // per, rows % per
    i, h = rem // 32, rem % 32
    assert_matches(out[b, i, h], lse[b, i, h], ro, rl, what=f"paged b64 q{q_len} sampled")


# ------------------------------------------------------------ logit soft-cap
CAPPED = [
    # (name, batch, qo, kv, d, lens, kw); sm_scale raised so the cap bends the scores
    ("cap20_gqa4", 2, 8, 2, 128, [700, 33], {"logit_cap": 20.0, "sm_scale": 0.5}),
    ("cap50_d256", 1, 8, 4, 256, [3000], {"logit_cap": 50.0, "sm_scale": 0.25}),
    ("cap10_fp8_paged_q2", 2, 8, 4, 128, [500, 77], {"logit_cap": 10.0, "sm_scale": 0.4,
                                                     "kv_dtype": "fp8_e4m3", "paged": True,
                                                     "page_size": 16, "q_len": 2}),
    ("cap30_gqa16_q2_rows32", 1, 32, 2, 128, [1200], {"logit_cap": 30.0, "sm_scale": 0.5,
                                                       "q_len": 2}),
    ("cap15_int4", 2, 8, 2, 128, [700, 33], {"logit_cap": 15.0, "sm_scale": 0.5,
                                             "kv_dtype": "int4"}),
    # small caps: the capped scores sit within [-c, c], so a masked key (window
    # start, ragged tail, causal edge) given the cap's floor -c instead of -inf
    # would carry a visible weight
    ("cap1_window_q2_gqa2", 2, 4, 2, 128, [700, 45], {"logit_cap": 1.0, "sm_scale": 0.05,
                                                       "window": 150, "q_len": 2}),
    ("cap1_fp8_window", 2, 8, 2, 128, [500, 70], {"logit_cap": 1.0, "sm_scale": 0.05,
                                                  "kv_dtype": "fp8_e4m3", "window": 100}),
    ("cap2_int4_tail", 2, 8, 2, 128, [130, 33], {"logit_cap": 2.0, "sm_scale": 0.1,
                                                 "kv_dtype": "int4"}),
]


@pytest.mark.parametrize("case", CAPPED, ids=[c[0] for c in CAPPED])
@pytest.mark.parametrize("path", PATHS)
def test_logit_softcap(case, path):
    name, B, Hq, Hk, d, lens, kw = case
    x = synth.generate(B, Hq, Hk, d, lens, seed=zlib.crc32(name.encode()) & 0xFFFF, name=name, **kw)
    if not _has_path(x, path):
        pytest.skip("no kernel for these rows on this path")
    out, lse, _ = _check(x, path=path)
    # the cap must matter here: the uncapped lse differs by far more than
    # the lse tolerance (the small-cap cases move it by about 0.1)
    plain = synth.DecodeInputs(**{**x.__dict__, "logit_cap": 0.0})
    po, pl = oracle.decode_all(plain)
    assert np.abs(pl - lse).max() > 20 * LSE_ABS


def test_logit_softcap_forced_splits():
    x = synth.generate(1, 8, 2, 128, [2500], seed=30, logit_cap=15.0, sm_scale=0.5)
    for n in (1, 9, 0):
        _check(x, path="mma", num_ctas=n)


# ------------------------------------------------- measured dataflow choice
def test_tuned_choices_match_the_oracle():
    """Decodes that fall in a row of the built-in measured table (those of at
    most 48 MB of visible K/V) run on the chosen dataflow and piece cap and
    still match the oracle."""
    rows = [r for r in binding.get_tuning() if r["bytes_min"] <= 48 << 20]
    assert rows, "the built-in table has small-problem rows"
    for r in rows:
        d, rows_per = r["head_dim"], r["rows_min"]
        es = 1 if r["kv_dtype"] == 1 else 2
        per_key = 8 * 2 * d * es
        L = -(-max(r["bytes_min"], 1 << 20) // per_key) + 3
        assert L * per_key <= r["bytes_max"]
        x = synth.generate(1, 8 * rows_per, 8, d, [L], seed=L % 1000,
                           kv_dtype="fp8_e4m3" if r["kv_dtype"] == 1 else "bf16",
                           name=f"tuned_d{d}_r{rows_per}_L{L}")
        out, lse, info = _check(x, path="auto")
        assert info["path"] == r["path"]


# ------------------------------------------------------------------ INT4 KV
def test_int4_forced_splits_agree():
    """INT4 KV: every split of the tiles over blocks merges to the oracle's
    result (one block, a few, one tile each)."""
    x = synth.generate(2, 16, 2, 128, [2500, 203], kv_dtype="int4", seed=33)
    _forced_splits_agree(x, "mma")


def test_full_size_int4_long_context():
    """The long-context GQA-8 decode with an INT4 cache at full size
    (131072 keys), sampled rows against the oracle."""
    _check_full(synth.workload("int4_gqa8_L131072"), path="mma", nrows=24, seed=3)



# ------------------------------------------------------------ unified max
UNIFIED = [
    # (name, batch, qo, kv, d, lens, kw)
    ("gqa4_paged", 3, 8, 2, 128, [900, 33, 260], {"paged": True, "page_size": 16}),
    ("fp8_gqa8", 1, 16, 2, 128, [1500], {"kv_dtype": "fp8_e4m3"}),
    ("int4_gqa4", 2, 8, 2, 128, [700, 90], {"kv_dtype": "int4"}),
    ("q4_rows16_win", 2, 8, 2, 128, [800, 40], {"q_len": 4, "window": 300}),
    ("cap20_d256", 1, 8, 4, 256, [1000], {"logit_cap": 20.0, "sm_scale": 0.5}),
]


@pytest.mark.parametrize("phi", [2.0, 30.0, 500.0, -500.0])
@pytest.mark.parametrize("case", UNIFIED, ids=[c[0] for c in UNIFIED])
@pytest.mark.parametrize("path", PATHS)
def test_unified_max_matches_the_oracle(case, path, phi):
    """The unified max ("FlashDecoding++", "Asynchronous softmax and unified
    max value") changes where the running max starts, not the result: with
    phi near the scores (2), above them (30: no rescale ever), far above
    (500: every row restarts from its own maximum) and far below (-500:
    the exact rescale takes over at the first tile) the pass equals the
    plain definition."""
    name, B, Hq, Hk, d, lens, kw = case
    x = synth.generate(B, Hq, Hk, d, lens, seed=zlib.crc32(name.encode()) & 0xFFFF, name=name, **kw)
    if not _has_path(x, path):
        pytest.skip("no kernel for these rows on this path")
    ref_out, ref_lse = oracle.decode_all(x)
    dev = DeviceInputs(x)
    for n in (0, 7):
        p = binding.plan(x.batch, x.qo_heads, x.kv_heads, x.head_dim, x.kv_indptr,
                         kv_dtype=x.kv_dtype, paged=x.paged, page_size=x.page_size,
                         window=x.window, sm_scale=x.sm_scale, path=path, num_ctas=n,
                         q_len=x.q_len, logit_cap=x.logit_cap, softmax_phi=phi)
        ws = p.new_workspace()
        out, lse = dev.run(p, workspace=ws)
        assert binding.decode_status(ws) == 0
        o, l = to_numpy(out, lse)
        assert_matches(o, l, ref_out, ref_lse, what=f"{name} {path} phi={phi} ctas={n}")


# ------------------------------------------------------------------ limits
def test_largest_batch():
    """The largest batch the planner accepts for this shape (its block's
    schedule arrays fill the shared memory the tile ring leaves), short and
    ragged requests, paged: every row against the oracle."""
    import ctypes
    lib = binding.load_library()

    def ok(batch):
        d = binding.DecodeDesc(batch=batch, qo_heads=8, kv_heads=2, head_dim=128, kv_dtype=0,
                               paged=1, page_size=16, window=-1, sm_scale=0.1, path=0,
                               num_ctas=0)
        ind = np.arange(batch + 1, dtype=np.int32) * 20
        h, ws = ctypes.c_void_p(), ctypes.c_size_t()
        st = lib.fa_decode_plan(ctypes.byref(d), ind.ctypes.data, 0, ctypes.byref(h),
                                ctypes.byref(ws))
        if h.value:
            lib.fa_plan_destroy(h)
        return st == 0
    lo, hi = 682, 1 << 17
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if ok(mid) else (lo, mid)
    rng = np.random.default_rng(50)
    lens = rng.integers(0, 70, size=lo)
    x = synth.generate(lo, 8, 2, 128, list(lens), paged=True, page_size=16, seed=51)
    _check(x)


def test_one_million_keys():
    """One request of 2^20 keys (fp8, GQA 8 on one kv head): sampled rows
    against the oracle."""
    x = synth.generate(1, 8, 1, 128, [1 << 20], kv_dtype="fp8_e4m3", seed=52)
    _check_full(x, path="mma", nrows=4, seed=5)


# ------------------------------------------------------ random shape sweep
def _random_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        dtype = ["bf16", "fp8_e4m3", "int4"][rng.integers(3)]
        d = int(rng.choice([64, 128, 256] if dtype == "bf16" else [128, 256]))
        kv = int(rng.choice([1, 2, 4, 8]))
        q_len = int(rng.choice([1, 1, 1, 2, 3, 4, 8]))
        group = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
        if group * q_len > 32:
            continue
        batch = int(rng.integers(1, 6))
        lens = [int(x) for x in rng.integers(0, 700, size=batch)]
        kw = {"q_len": q_len, "kv_dtype": dtype}
        if rng.random() < 0.5:
            kw.update(paged=True, page_size=int(rng.choice([1, 2, 4, 8, 16, 32, 64, 128, 256])),
                      unused_slot_fill="nan")
        if rng.random() < 0.3:
            kw["window"] = int(rng.integers(1, 400))
        if rng.random() < 0.2:
            kw.update(logit_cap=float(rng.uniform(5, 50)), sm_scale=0.3)
        path = ["auto", "mma", "simt"][rng.integers(3)]
        ctas = int(rng.choice([0, 0, 1, 3, 17]))
        phi = float(rng.uniform(-20, 20)) if rng.random() < 0.2 else None
        cases.append((len(cases), batch, group * kv, kv, d, lens, kw, path, ctas, phi))
    return cases


@pytest.mark.parametrize("case", _random_cases(120, 2026), ids=lambda c: f"r{c[0]}")
def test_random_shapes_match_the_oracle(case):
    """Seeded random decodes over the options' cross product (dtype, head
    size, group, query tokens, paging, window, soft-cap, unified max,
    dataflow, forced split): every supported one matches the oracle; a
    refused one is one the documented limits refuse."""
    idx, B, Hq, Hk, d, lens, kw, path, ctas, phi = case
    if kw.get("paged") and kw["kv_dtype"] == "int4" and d == 128 and kw["page_size"] == 1:
        kw = {**kw, "page_size": 2}  # a one-token int4 page is refused (128-byte copy rule)
    x = synth.generate(B, Hq, Hk, d, lens, seed=1000 + idx, name=f"random{idx}", **kw)
    rows = x.group * x.q_len
    try:
        p = binding.plan(x.batch, x.qo_heads, x.kv_heads, x.head_dim, x.kv_indptr,
                         kv_dtype=x.kv_dtype, paged=x.paged, page_size=x.page_size,
                         window=x.window, sm_scale=x.sm_scale, path=path, num_ctas=ctas,
                         q_len=x.q_len, logit_cap=x.logit_cap, softmax_phi=phi)
    except binding.FadecodeError as e:
        assert e.status == 2, str(e)
        simt_ok = x.kv_dtype != "int4" and rows in (1, 2, 4, 8)
        assert path == "simt" and not simt_ok, f"unexpected refusal: {e}"
        return
    ref_out, ref_lse = oracle.decode_all(x)
    dev = DeviceInputs(x)
    ws = p.new_workspace()
    out, lse = dev.run(p, workspace=ws)
    assert binding.decode_status(ws) == 0
    o, l = to_numpy(out, lse)
    assert_matches(o, l, ref_out, ref_lse, what=f"random{idx} {path} ctas={ctas} phi={phi} {kw}")


@pytest.mark.parametrize("kw", [
    {"lens": [1500, 0, 40, 700, 2000, 17], "paged": True, "page_size": 16},
    {"lens": [3000, 900], "kv_dtype": "fp8_e4m3"},
    {"lens": [2500, 64], "kv_dtype": "int4", "kv": 4},
    {"lens": [1200, 5, 333], "q_len": 4},
], ids=["bf16_paged", "fp8", "int4_head_tiles", "q4_rows16"])
def test_repeated_passes_are_bit_identical(kw):
    """The split depends only on the plan's inputs, and every reduction
    (the tile lanes' merge in a block, the split-segment merge) runs in a
    fixed order, whichever warp or block finishes first: the same inputs give
    the same bits, pass after pass, with the plan reused or made again."""
    import torch
    kw = dict(kw)
    lens, kv = kw.pop("lens"), kw.pop("kv", 2)
    x = synth.generate(len(lens), 4 * kv, kv, 128, lens, seed=41, **kw)
    dev = DeviceInputs(x)
    for n in (0, 9):
        p = dev.plan(num_ctas=n)
        ws = p.new_workspace()
        outs = []
        for rep in range(3):
            q = p if rep < 2 else dev.plan(num_ctas=n)
            out, lse = dev.run(q, workspace=ws)
            torch.cuda.synchronize()
            outs.append((out.view(torch.int16).cpu().clone(), lse.view(torch.int32).cpu().clone()))
        assert binding.decode_status(ws) == 0
        for o, l in outs[1:]:
            assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1]), f"ctas={n}"


@pytest.mark.parametrize("kw", [
    {"lens": [1500, 0, 40, 700, 2000, 17], "paged": True, "page_size": 16},
    {"lens": [3000, 900], "kv_dtype": "fp8_e4m3"},
    {"lens": [1200, 5, 333], "q_len": 4},
], ids=["bf16_paged_split", "fp8", "q4_rows16"])
def test_pass_captured_in_a_cuda_graph(kw):
    """fa_decode_run enqueues kernel launches only (every argument by value,
    no allocation, no synchronisation), so a decode loop can capture it in a
    CUDA graph: the decode kernel and, for split segments, the merge kernel
    as its programmatic dependent.  Replays give the oracle's result, the
    same bits each time, also after the inputs change in place."""
    import torch
    kw = dict(kw)
    lens = kw.pop("lens")
    x = synth.generate(len(lens), 8, 2, 128, lens, seed=43, **kw)
    dev = DeviceInputs(x)
    p = dev.plan(num_ctas=0)
    ws = p.new_workspace()
    out, lse = dev.run(p, workspace=ws)  # warm-up outside the capture
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        dev.run(p, workspace=ws, out=out, lse=lse)
    ref_out, ref_lse = oracle.decode_all(x)
    first = None
    for rep in range(3):
        out.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        o, l = to_numpy(out, lse)
        assert_matches(o, l, ref_out, ref_lse, what=f"graph replay {rep}")
        bits = (out.view(torch.int16).cpu().clone(), lse.view(torch.int32).cpu().clone())
        if first is None:
            first = bits
        else:
            assert torch.equal(bits[0], first[0]) and torch.equal(bits[1], first[1])
    assert binding.decode_status(ws) == 0
    # the graph reads the inputs where they live: new q values, same buffers
    y = synth.generate(len(lens), 8, 2, 128, lens, seed=44, **kw)
    dev.q.copy_(torch.from_numpy(np.ascontiguousarray(y.q).view(np.int16)).to(dev.q.device))
    x.q = y.q
    g.replay()
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_all(x)
    o, l = to_numpy(out, lse)
    assert_matches(o, l, ref_out, ref_lse, what="graph replay, new q")
    # and new lengths: the kernels split the device copy of kv_indptr, so a
    # replay follows requests that shrank (the extents given at capture hold)
    q_len = kw.get("q_len", 1)
    new_lens = [max(q_len, (3 * n) // 4) if n > 0 else 0 for n in lens]
    ind = np.concatenate([[0], np.cumsum(new_lens)]).astype(np.int32)
    dev.kv_indptr.copy_(torch.from_numpy(ind).to(dev.kv_indptr.device))
    x.kv_indptr = ind
    g.replay()
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_all(x)
    o, l = to_numpy(out, lse)
    assert_matches(o, l, ref_out, ref_lse, what="graph replay, shorter requests")
    assert binding.decode_status(ws) == 0
