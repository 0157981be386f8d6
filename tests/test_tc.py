"""GPU parity of the tcgen05 dataflow (bf16 K/V, head_dim 128, 9 to 32 query
rows per segment: several query tokens per request, or GQA groups wider
than 8) against the fp64 oracle, element by element, under the stated
tolerances.  Cases span several 128-token tiles and ragged tails, paged and
contiguous K/V (pages of 8 to 256 tokens, unused slots filled with NaN),
windows, soft-capping, empty and one-key requests, forced splits and the
cost-charged split; repeated passes are bit-identical."""
import zlib

import numpy as np
import pytest

from gqa_decode_attention_split_b200 import binding, synth
from gpu_util import DeviceInputs, assert_matches, run_gpu, to_numpy
from oracle import oracle

pytestmark = pytest.mark.gpu

CASES = [
    # (name, batch, qo, kv, d, lens, kw)
    ("gqa16_rows16", 1, 16, 1, 128, [2000], {}),
    ("gqa12_rows12_pad", 2, 24, 2, 128, [700, 129], {}),
    ("q3_gqa4_rows12", 2, 8, 2, 128, [260, 31], {"q_len": 3}),
    ("q4_gqa4_paged16_rows16", 3, 8, 2, 128, [300, 2, 65], {"q_len": 4, "paged": True,
                                                            "page_size": 16}),
    ("q5_gqa2_rows10_win", 2, 4, 2, 128, [900, 40], {"q_len": 5, "window": 100}),
    ("q8_gqa4_paged16_rows32", 3, 8, 2, 128, [411, 17, 96], {"q_len": 8, "paged": True,
                                                             "page_size": 16}),
    ("q8_gqa4_paged32_rows32", 3, 8, 2, 128, [411, 17, 96], {"q_len": 8, "paged": True,
                                                             "page_size": 32}),
    ("q6_gqa4_rows24", 2, 8, 2, 128, [1000, 300], {"q_len": 6}),
    ("gqa32_paged64_rows32", 2, 32, 1, 128, [700, 130], {"paged": True, "page_size": 64}),
    ("gqa32_paged8_rows32", 2, 32, 1, 128, [300, 17], {"paged": True, "page_size": 8}),
    ("gqa20_paged128_rows20", 2, 40, 2, 128, [1000, 128], {"paged": True, "page_size": 128}),
    ("gqa16_paged256_win", 2, 16, 1, 128, [1500, 257], {"paged": True, "page_size": 256,
                                                         "window": 300}),
    ("q2_gqa8_rows16_cap", 2, 16, 2, 128, [500, 70], {"q_len": 2, "logit_cap": 20.0,
                                                      "sm_scale": 0.5}),
    # a small cap keeps masked keys at weight zero (the cap is applied to
    # visible scores only): window and causal edges, a ragged tail
    ("q4_gqa4_cap1_win", 2, 8, 2, 128, [700, 45], {"q_len": 4, "logit_cap": 1.0,
                                                   "sm_scale": 0.05, "window": 150}),
    ("q8_gqa2_tile_edges", 5, 4, 2, 128, [128, 127, 129, 1, 256], {"q_len": 8}),
    ("q4_gqa4_empty", 4, 8, 2, 128, [0, 300, 0, 3], {"q_len": 4}),
    ("q2_gqa8_short", 2, 16, 2, 128, [1, 2], {"q_len": 2}),
]


def _gen(case):
    name, B, Hq, Hk, d, lens, kw = case
    kw = dict(kw)
    return synth.generate(B, Hq, Hk, d, lens, seed=zlib.crc32(name.encode()) & 0xFFFF, name=name,
                          unused_slot_fill="nan" if kw.get("paged") else None,
                          extra_rows=0 if kw.get("paged") else 40, **kw)


def _check(x, num_ctas=0, piece_cost=0, ref=None, what=""):
    ref_out, ref_lse = ref if ref is not None else oracle.decode_all(x)
    out, lse, flags, info = run_gpu(x, path="tc", num_ctas=num_ctas, piece_cost=piece_cost)
    assert info["path"] == binding.PATH_TC
    assert flags == 0, f"{x.name}: device flags {flags}"
    assert_matches(out, lse, ref_out, ref_lse, what=f"{x.name} tc ctas={num_ctas} {what}")
    return out, lse, info


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_matches_the_oracle(case):
    x = _gen(case)
    _check(x)
    # the planner picks this dataflow by itself for these shapes
    out, lse, flags, info = run_gpu(x)
    assert info["path"] == binding.PATH_TC and flags == 0


SMALL_ROWS = [
    # (batch, qo, kv, lens, kw): 1 to 8 rows, padded to 16 on this dataflow
    (3, 8, 2, [700, 129, 1], {}),
    (2, 8, 2, [500, 70], {"q_len": 2, "paged": True, "page_size": 16}),
    (2, 4, 4, [900, 33], {"q_len": 8}),
    (2, 16, 2, [300, 2000], {"window": 200}),
    (2, 2, 2, [129, 64], {"logit_cap": 10.0}),
]


@pytest.mark.parametrize("case", SMALL_ROWS, ids=["gqa4", "gqa4_q2_paged", "mha_q8", "gqa8_win",
                                                  "mha_cap"])
def test_tc_asked_for_eight_rows_or_fewer(case):
    """Asked for, the dataflow also takes 1 to 8 rows (padded to 16, the
    padding rows' results discarded); the planner does not choose it there
    (the warp-level products measured faster)."""
    B, Hq, Hk, lens, kw = case
    x = synth.generate(B, Hq, Hk, 128, lens, seed=51,
                       unused_slot_fill="nan" if kw.get("paged") else None, **kw)
    ref = oracle.decode_all(x)
    _check(x, ref=ref)
    _check(x, num_ctas=7, ref=ref)
    _, _, _, info = run_gpu(x)
    assert info["path"] != binding.PATH_TC


@pytest.mark.parametrize("q_len", [3, 4, 8])
def test_tc_forced_splits_agree(q_len):
    """Splitting over more blocks, then merging, gives the oracle's result at
    every granularity (one block up to one tile per block)."""
    x = synth.generate(3, 8, 2, 128, [1500, 203, 640], q_len=q_len, seed=41, paged=True,
                       page_size=16)
    ref = oracle.decode_all(x)
    results = []
    total = None
    for n in (1, 2, 7, 64, 0):
        out, lse, info = _check(x, num_ctas=n, ref=ref)
        total = info["total_tiles"]
        results.append((out, lse))
    out, lse, info = _check(x, num_ctas=total, ref=ref)
    results.append((out, lse))
    for o, l in results[1:]:
        assert np.abs(l - results[0][1]).max() <= 2e-5
        assert np.abs(o - results[0][0]).max() <= 4e-3


def test_tc_piece_cost_splits_agree():
    lens = [1500, 0, 40, 1, 0, 700, 127, 128, 129, 0, 2000, 17]
    x = synth.generate(len(lens), 16, 1, 128, lens, seed=43)
    ref = oracle.decode_all(x)
    for cost in (-1, 1, 3, 17, 4096):
        for n in (0, 5, 37):
            _, _, info = _check(x, num_ctas=n, piece_cost=cost, ref=ref, what=f"cost={cost}")
            if cost > 0 and n > 0:
                assert info["piece_cost"] == cost


def test_tc_repeated_passes_are_bit_identical():
    x = synth.generate(4, 8, 2, 128, [3000, 45, 900, 2200], q_len=4, seed=45, paged=True,
                       page_size=16)
    dev = DeviceInputs(x)
    p = dev.plan(path="tc")
    ws = p.new_workspace()
    first = to_numpy(*dev.run(p, workspace=ws))
    for _ in range(3):
        o, l = to_numpy(*dev.run(p, workspace=ws))
        np.testing.assert_array_equal(o, first[0])
        np.testing.assert_array_equal(l, first[1])
    assert binding.decode_status(ws) == 0
    ref_out, ref_lse = oracle.decode_all(x)
    assert_matches(first[0], first[1], ref_out, ref_lse, what="repeated")


def test_tc_bad_page_is_flagged_not_read():
    x = synth.generate(2, 8, 2, 128, [300, 300], q_len=4, paged=True, page_size=16, seed=47)
    x.page_table[1, 3] = x.k.shape[0] + 9  # outside the pool
    out, lse, flags, info = run_gpu(x, path="tc")
    assert info["path"] == binding.PATH_TC and flags & 1
    one = synth.DecodeInputs(**{**x.__dict__, "batch": 1, "q": x.q[:1],
                                "kv_indptr": x.kv_indptr[:2], "page_table": x.page_table[:1]})
    ro, rl = oracle.decode_all(one)
    assert_matches(out[:1], lse[:1], ro, rl, what="unaffected request")


def _random_tc_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        kv = int(rng.choice([1, 2, 4]))
        q_len = int(rng.choice([1, 2, 3, 4, 8]))
        group = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
        if group * q_len > 32:
            continue
        batch = int(rng.integers(1, 6))
        lens = [int(v) for v in rng.integers(0, 1500, size=batch)]
        kw = {"q_len": q_len}
        if rng.random() < 0.5:
            kw.update(paged=True, page_size=int(rng.choice([8, 16, 32, 64, 128, 256])),
                      unused_slot_fill="nan")
        if rng.random() < 0.3:
            kw["window"] = int(rng.integers(1, 600))
        if rng.random() < 0.2:
            kw.update(logit_cap=float(rng.uniform(2, 50)), sm_scale=0.3)
        ctas = int(rng.choice([0, 0, 1, 3, 17]))
        cases.append((len(cases), batch, group * kv, kv, lens, kw, ctas))
    return cases


@pytest.mark.parametrize("case", _random_tc_cases(40, 2027), ids=lambda c: f"r{c[0]}")
def test_tc_random_shapes_match_the_oracle(case):
    """Seeded random decodes on this dataflow over its options' cross
    product (1-32 rows, query tokens, paging, window, soft-cap, forced
    split), each against the oracle."""
    idx, B, Hq, Hk, lens, kw, ctas = case
    x = synth.generate(B, Hq, Hk, 128, lens, seed=3000 + idx, name=f"tc_random{idx}", **kw)
    _check(x, num_ctas=ctas, what=f"random{idx} {kw}")
