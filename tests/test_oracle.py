"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: hand-derived
golden cases, torch's own bf16/e4m3 decoders, closed forms, invariants that
hold for exact attention, the textbook routine
torch.nn.functional.scaled_dot_product_attention in fp64, and an independent
restatement of the tiled online-softmax recurrence ("Forcing Flash Attention
onto a TPU", section "Flash Attention in JAX": running max, running sum and
accumulator per query row, rescaled by exp(m_old - m_new), guarded with
isfinite, normalised at the end).
"""
import glob
import json
import math
import os

import numpy as np
import pytest
import torch

from gqa_decode_attention_split_b200 import synth
from gqa_decode_attention_split_b200.synth import DecodeInputs
from helpers import (bf16_bits, bf16_values, contiguous_inputs, dense_kv, e4m3_values, int4_values,
                     visible)
from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAN_BF16 = np.uint16(0x7FC0)


def _eval(expr):
    return eval(str(expr), {"__builtins__": {}},
                {"e": math.e, "log": math.log, "inf": math.inf})


def _golden_inputs(g, window=None):
    w = g.get("window", -1) if window is None else window
    lens = g["kv_lens"]
    indptr = np.zeros(len(lens) + 1, dtype=np.int32)
    indptr[1:] = np.cumsum(lens)
    q = bf16_bits(np.array(g["q"], dtype=np.float32))
    B, Hq, d = q.shape
    if g["layout"] == "paged":
        def pool(a):
            arr = np.array([[[[np.nan if x is None else x for x in h] for h in s] for s in p]
                            for p in a], dtype=np.float32)
            bits = np.where(np.isnan(arr), NAN_BF16, 0).astype(np.uint16)
            ok = ~np.isnan(arr)
            bits[ok] = bf16_bits(arr[ok])
            return bits
        k, v = pool(g["k_pool"]), pool(g["v_pool"])
        return DecodeInputs(name="golden", batch=B, qo_heads=Hq, kv_heads=k.shape[2], head_dim=d,
                            kv_dtype="bf16", paged=True, page_size=g["page_size"], window=w,
                            sm_scale=g["sm_scale"], q=q, k=k, v=v, kv_indptr=indptr,
                            page_table=np.array(g["page_table"], dtype=np.int32))
    if g["kv_dtype"] == "fp8_e4m3":
        k = np.array(g["k_codes"], dtype=np.uint8)
        v = np.array(g["v_codes"], dtype=np.uint8)
        return DecodeInputs(name="golden", batch=B, qo_heads=Hq, kv_heads=k.shape[1], head_dim=d,
                            kv_dtype="fp8_e4m3", paged=False, page_size=0, window=w,
                            sm_scale=g["sm_scale"], q=q, k=k, v=v, kv_indptr=indptr,
                            k_scale=np.array(g["k_scale"], dtype=np.float32),
                            v_scale=np.array(g["v_scale"], dtype=np.float32))
    return contiguous_inputs(g["q"], g["k"], g["v"], lens, sm_scale=g["sm_scale"], window=w)


def _check_expected(out, lse, exp_out, exp_lse):
    eo = np.vectorize(_eval, otypes=[float])(np.array(exp_out, dtype=object))
    el = np.vectorize(_eval, otypes=[float])(np.array(exp_lse, dtype=object))
    np.testing.assert_allclose(out, eo, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, el, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "*.json"))),
                         ids=lambda p: os.path.basename(p))
def test_golden(path):
    with open(path) as f:
        g = json.load(f)
    if "windows" in g:
        for w, eo, el in zip(g["windows"], g["expected_out_per_window"],
                             g["expected_lse_per_window"]):
            out, lse = oracle.decode_all(_golden_inputs(g, window=w))
            _check_expected(out, lse, eo, el)
    else:
        out, lse = oracle.decode_all(_golden_inputs(g))
        _check_expected(out, lse, g["expected_out"], g["expected_lse"])


def test_bf16_decoder_matches_torch_on_every_code():
    codes = np.arange(65536, dtype=np.uint16)
    ours = oracle.bf16_to_double(codes)
    ref = bf16_values(codes)
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.array_equal(ours[~both_nan], ref[~both_nan])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_e4m3_decoder_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_double(codes)
    ref = e4m3_values(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    # spot values from the format definition
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert ours[0xB8] == -1.0 and np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])


def _sdpa_reference(x: DecodeInputs, b: int):
    """torch's scaled_dot_product_attention (fp64, CPU) on the visible keys of
    request b, with kv heads expanded to query heads in consecutive groups."""
    lo, hi = visible(x, b)
    kf, vf = dense_kv(x, b)
    kf, vf = kf[lo:hi], vf[lo:hi]
    q = torch.from_numpy(bf16_values(x.q[b]))                     # [Hq, d]
    K = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(x.group, dim=0)  # [Hq, n, d]
    V = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(x.group, dim=0)
    out = torch.nn.functional.scaled_dot_product_attention(
        q[None, :, None, :], K[None], V[None], scale=x.sm_scale)[0, :, 0, :]
    scores = torch.einsum("hd,hnd->hn", q, K) * x.sm_scale
    lse = torch.logsumexp(scores, dim=-1)
    return out.numpy(), lse.numpy()


@pytest.mark.parametrize("case", [
    dict(batch=1, qo=8, kv=2, d=64, lens=[53]),
    dict(batch=3, qo=4, kv=4, d=32, lens=[17, 1, 40]),
    dict(batch=2, qo=8, kv=1, d=16, lens=[29, 64], window=5),
    dict(batch=2, qo=4, kv=2, d=16, lens=[33, 7], paged=True, page_size=4),
    dict(batch=2, qo=8, kv=2, d=32, lens=[45, 12], fp8=True),
    dict(batch=2, qo=4, kv=2, d=16, lens=[19, 50], fp8=True, paged=True, page_size=8, window=9),
    dict(batch=2, qo=8, kv=2, d=32, lens=[45, 12], dtype="int4"),
    dict(batch=2, qo=4, kv=2, d=16, lens=[19, 50], dtype="int4", paged=True, page_size=8, window=9),
])
def test_matches_textbook_sdpa(case):
    x = synth.generate(case["batch"], case["qo"], case["kv"], case["d"], case["lens"],
                       kv_dtype=case.get("dtype", "fp8_e4m3" if case.get("fp8") else "bf16"),
                       paged=case.get("paged", False), page_size=case.get("page_size", 16),
                       window=case.get("window", -1), seed=11, unused_slot_fill="nan")
    out, lse = oracle.decode_all(x)
    for b in range(x.batch):
        ro, rl = _sdpa_reference(x, b)
        np.testing.assert_allclose(out[b], ro, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=1e-12, atol=1e-12)


def _online_softmax_restated(q, K, V, scale, block):
    """Tiled single-pass softmax with running (max, sum, acc), restated from
    the recurrence on the TPU flash-attention page; K, V: [n, d] fp64."""
    m, s = -math.inf, 0.0
    acc = np.zeros(V.shape[1])
    for a in range(0, max(1, K.shape[0]), block):
        kt, vt = K[a:a + block], V[a:a + block]
        sc = (kt @ q) * scale if kt.shape[0] else np.zeros(0)
        tmax = sc.max() if sc.size else -math.inf
        mn = max(m, tmax)
        alpha = math.exp(m - mn) if math.isfinite(m) else 0.0
        w = np.exp(sc - mn) if math.isfinite(mn) else np.zeros_like(sc)
        s = alpha * s + w.sum()
        acc = alpha * acc + w @ vt if sc.size else alpha * acc
        m = mn
    out = acc / s if s > 0 else np.zeros_like(acc)
    lse = m + math.log(s) if s > 0 else -math.inf
    return out, lse


@pytest.mark.parametrize("block", [1, 3, 16, 1000])
def test_matches_online_softmax_restatement(block):
    x = synth.generate(2, 4, 2, 16, [37, 0], seed=7)
    out, lse = oracle.decode_all(x)
    for b in range(x.batch):
        lo, hi = visible(x, b)
        kf, vf = dense_kv(x, b)
        for h in range(x.qo_heads):
            g = h // x.group
            ro, rl = _online_softmax_restated(bf16_values(x.q[b, h]), kf[lo:hi, g], vf[lo:hi, g],
                                              x.sm_scale, block)
            np.testing.assert_allclose(out[b, h], ro, rtol=1e-12, atol=1e-13)
            if math.isinf(rl):
                assert lse[b, h] == rl
            else:
                assert abs(lse[b, h] - rl) < 1e-12


def test_constant_keys_give_mean_of_values():
    rng = np.random.default_rng(0)
    L, d = 300, 8
    kvec = rng.integers(-4, 5, size=d)
    qv = rng.integers(-4, 5, size=(1, 2, d))
    k = np.broadcast_to(kvec, (L, 1, d))
    v = rng.integers(-8, 9, size=(L, 1, d))
    for window in (-1, 17):
        x = contiguous_inputs(qv, k, v, [L], sm_scale=0.25, window=window)
        out, lse = oracle.decode_all(x)
        lo = L - window if window > 0 else 0
        for h in range(2):
            np.testing.assert_allclose(out[0, h], v[lo:, 0].mean(axis=0), rtol=0, atol=1e-12)
            assert abs(lse[0, h] - (0.25 * float(qv[0, h] @ kvec) + math.log(L - lo))) < 1e-12


def test_spike_key_returns_its_value_row():
    """One key scores 40, every other key 0: out = V[j*] to within n*e^-40.
    The spike is placed on a page boundary, in the last kv head and at the
    first key of a window, which pins gather, head mapping and window start."""
    d, L, ps = 8, 100, 4
    x = synth.generate(1, 4, 2, d, [L], paged=True, page_size=ps, seed=3)
    q = np.zeros((1, 4, d), np.float32)
    q[0, :, 0] = 8.0
    xq = bf16_bits(q)
    kz = np.zeros_like(x.k)
    for jstar, window in ((ps * 7, -1), (L - 10, 10), (L - 11, 10)):
        k = kz.copy()
        pg = x.page_table[0, jstar // ps]
        k[pg, jstar % ps, 1, 0] = bf16_bits(np.float32(5.0))  # kv head 1 only
        y = DecodeInputs(**{**x.__dict__, "q": xq, "k": k, "window": window, "sm_scale": 1.0})
        out, lse = oracle.decode_all(y)
        _, vf = dense_kv(y, 0)
        lo = L - window if window > 0 else 0
        if jstar >= lo:
            np.testing.assert_allclose(out[0, 2], vf[jstar, 1], atol=1e-12)
            np.testing.assert_allclose(out[0, 3], vf[jstar, 1], atol=1e-12)
            assert abs(lse[0, 2] - (40.0 + math.log1p((L - lo - 1) * math.exp(-40.0)))) < 1e-12
        else:  # spike just outside the window: every visible score is 0
            np.testing.assert_allclose(out[0, 2], vf[lo:, 1].mean(axis=0), atol=1e-12)
            assert abs(lse[0, 2] - math.log(L - lo)) < 1e-12
        # heads 0,1 read kv head 0 where all keys are 0: mean of all visible values
        np.testing.assert_allclose(out[0, 0], vf[lo:, 0].mean(axis=0), atol=1e-12)


def test_degenerate_cases():
    x = synth.generate(3, 4, 2, 16, [1, 50, 50], seed=9)
    out, lse = oracle.decode_all(x)
    kf, vf = dense_kv(x, 0)
    q = bf16_values(x.q[0])
    for h in range(4):   # L = 1: out = V[0], lse = s_0
        np.testing.assert_allclose(out[0, h], vf[0, h // 2], atol=1e-15)
        assert abs(lse[0, h] - x.sm_scale * float(q[h] @ kf[0, h // 2])) < 1e-12
    y = DecodeInputs(**{**x.__dict__, "sm_scale": 0.0})
    out0, lse0 = oracle.decode_all(y)  # sm_scale = 0: uniform weights
    _, vf1 = dense_kv(x, 1)
    np.testing.assert_allclose(out0[1, 3], vf1[:, 1].mean(axis=0), atol=1e-12)
    assert abs(lse0[1, 3] - math.log(50)) < 1e-12
    z = x.with_window(1)  # window 1: the newest key only
    out1, lse1 = oracle.decode_all(z)
    np.testing.assert_allclose(out1[2, 0], dense_kv(x, 2)[1][49, 0], atol=1e-15)


def test_weights_sum_to_one_and_linearity_in_values():
    rng = np.random.default_rng(1)
    L, d = 77, 8
    q = rng.integers(-3, 4, size=(1, 4, d))
    k = rng.integers(-3, 4, size=(L, 2, d))
    v = rng.integers(-8, 9, size=(L, 2, d))
    ones = np.ones_like(v)
    o1, _ = oracle.decode_all(contiguous_inputs(q, k, ones, [L], sm_scale=0.3))
    np.testing.assert_allclose(o1, 1.0, atol=1e-13)
    o, lse = oracle.decode_all(contiguous_inputs(q, k, v, [L], sm_scale=0.3))
    o2, lse2 = oracle.decode_all(contiguous_inputs(q, k, 2 * v + 1, [L], sm_scale=0.3))
    np.testing.assert_allclose(o2, 2 * o + 1, atol=1e-12)
    np.testing.assert_array_equal(lse, lse2)


def test_permutation_and_shift_invariance():
    rng = np.random.default_rng(2)
    L, d = 64, 8
    q = rng.integers(-3, 4, size=(1, 2, d))
    k = rng.integers(-3, 4, size=(L, 1, d))
    v = rng.integers(-8, 9, size=(L, 1, d))
    o, lse = oracle.decode_all(contiguous_inputs(q, k, v, [L], sm_scale=0.2))
    perm = rng.permutation(L)
    op, lsep = oracle.decode_all(contiguous_inputs(q, k[perm], v[perm], [L], sm_scale=0.2))
    np.testing.assert_allclose(op, o, atol=1e-12)
    np.testing.assert_allclose(lsep, lse, atol=1e-12)
    c = rng.integers(-2, 3, size=d)
    os_, lses = oracle.decode_all(contiguous_inputs(q, k + c, v, [L], sm_scale=0.2))
    np.testing.assert_allclose(os_, o, atol=1e-12)
    kappa = 0.2 * (q[0].astype(np.float64) @ c)
    np.testing.assert_allclose(lses[0], lse[0] + kappa, atol=1e-12)


def test_paged_layout_equals_contiguous_layout():
    x = synth.generate(3, 8, 2, 32, [40, 3, 65], seed=5)
    ps = 8
    npages = [(int(L) + ps - 1) // ps for L in x.kv_lens]
    total = sum(npages)
    perm = np.random.default_rng(4).permutation(total)
    kp = np.full((total, ps, 2, 32), NAN_BF16, np.uint16)
    vp = kp.copy()
    pt = np.full((3, max(npages)), -1, np.int32)
    off = 0
    for b in range(3):
        a = int(x.kv_indptr[b])
        for t in range(int(x.kv_lens[b])):
            pg = perm[off + t // ps]
            kp[pg, t % ps] = x.k[a + t]
            vp[pg, t % ps] = x.v[a + t]
        pt[b, :npages[b]] = perm[off:off + npages[b]]
        off += npages[b]
    y = DecodeInputs(**{**x.__dict__, "paged": True, "page_size": ps, "k": kp, "v": vp,
                        "page_table": pt})
    o1, l1 = oracle.decode_all(x)
    o2, l2 = oracle.decode_all(y)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_split_then_merge_equals_unsplit():
    """Cutting one request's keys into consecutive parts (as separate
    requests over the same rows), then merging the parts' states, reproduces
    the unsplit result; an empty part carries no weight."""
    whole = synth.generate(1, 8, 2, 16, [37], seed=6)
    o, lse = oracle.decode_all(whole)
    cuts = [0, 10, 10, 11, 37]
    n = len(cuts) - 1
    parts = DecodeInputs(**{**whole.__dict__, "batch": n,
                            "q": np.repeat(whole.q, n, axis=0),
                            "kv_indptr": np.array(cuts, np.int32)})
    op, lp = oracle.decode_all(parts)
    assert np.isneginf(lp[1]).all() and (op[1] == 0).all()
    om, lm = oracle.merge(op[:, None], lp[:, None])
    np.testing.assert_allclose(om[0], o[0], atol=1e-13)
    np.testing.assert_allclose(lm[0], lse[0], atol=1e-13)


def test_merge_closed_forms_and_algebra():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((3, 2, 4, 16))
    l = rng.standard_normal((3, 2, 4))
    # two states with equal lse: plain average, lse + ln 2
    om, lm = oracle.merge(o[:2], np.stack([l[0], l[0]]))
    np.testing.assert_allclose(om, 0.5 * (o[0] + o[1]), atol=1e-14)
    np.testing.assert_allclose(lm, l[0] + math.log(2.0), atol=1e-14)
    # single state is the identity
    om, lm = oracle.merge(o[:1], l[:1])
    np.testing.assert_allclose(om, o[0], atol=1e-15)
    np.testing.assert_allclose(lm, l[0], atol=1e-15)
    # associativity
    ab_o, ab_l = oracle.merge(o[:2], l[:2])
    left = oracle.merge(np.stack([ab_o, o[2]]), np.stack([ab_l, l[2]]))
    bc_o, bc_l = oracle.merge(o[1:], l[1:])
    right = oracle.merge(np.stack([o[0], bc_o]), np.stack([l[0], bc_l]))
    allm = oracle.merge(o, l)
    for a, b in ((left, right), (left, allm)):
        np.testing.assert_allclose(a[0], b[0], atol=1e-13)
        np.testing.assert_allclose(a[1], b[1], atol=1e-13)
    # a -inf state is the identity; all -inf gives zeros and -inf
    ninf = np.full_like(l[0], -np.inf)
    om, lm = oracle.merge(np.stack([o[0], o[1]]), np.stack([l[0], ninf]))
    np.testing.assert_allclose(om, o[0], atol=1e-15)
    np.testing.assert_allclose(lm, l[0], atol=1e-15)
    om, lm = oracle.merge(o[:2], np.stack([ninf, ninf]))
    assert (om == 0).all() and np.isneginf(lm).all()


# ------------------------------------------------------ several query tokens
# A request's q_len newest keys are its query tokens; token i sits at position
# L - q_len + i and sees keys up to and including itself (the causal mask of
# "Standard causal attention" restricted to the new rows), or the last
# `window` of those.

def _brute_multi(x):
    """Plain numpy two-pass softmax with an explicit causal mask, written
    apart from the oracle: out [B, Q, Hq, d], lse [B, Q, Hq]."""
    B, Q, Hq, d = x.batch, x.q_len, x.qo_heads, x.head_dim
    G = Hq // x.kv_heads
    qf = bf16_values(x.q).reshape(B, Q, Hq, d)
    out = np.zeros((B, Q, Hq, d))
    lse = np.full((B, Q, Hq), -np.inf)
    for b in range(B):
        kf, vf = dense_kv(x, b)
        L = kf.shape[0]
        pos = np.arange(L)
        for i in range(Q):
            me = L - Q + i
            mask = pos <= me
            if x.window > 0:
                mask &= pos > me - x.window
            if not mask.any():
                continue
            for h in range(Hq):
                s = x.sm_scale * (kf[mask, h // G] @ qf[b, i, h])
                m = s.max()
                z = np.exp(s - m).sum()
                out[b, i, h] = (np.exp(s - m) / z) @ vf[mask, h // G]
                lse[b, i, h] = m + math.log(z)
    return out, lse


@pytest.mark.parametrize("window", [-1, 1, 4, 6])
def test_multi_token_matches_brute_force(window):
    x = synth.generate(3, 4, 2, 8, [9, 3, 17], q_len=3, paged=True, page_size=4, seed=40,
                       window=window)
    out, lse = oracle.decode_all(x)
    assert out.shape == (3, 3, 4, 8) and lse.shape == (3, 3, 4)
    ref_out, ref_lse = _brute_multi(x)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [-1, 5])
def test_multi_token_rows_are_single_token_decodes(window):
    """Row (b, i, h) of a q_len problem is the one-token decode of request b
    truncated to L - q_len + i + 1 keys, with token i's query: the same pool,
    only the token counts change."""
    Q = 4
    lens = [33, 4, 18]
    x = synth.generate(3, 8, 2, 16, lens, q_len=Q, paged=True, page_size=8, seed=41,
                       window=window)
    out, lse = oracle.decode_all(x)
    for i in range(Q):
        short = np.array([L - Q + i + 1 for L in lens])
        ind = np.concatenate([[0], np.cumsum(short)]).astype(np.int32)
        y = DecodeInputs(**{**x.__dict__, "q": np.ascontiguousarray(x.q[:, i]), "kv_indptr": ind,
                            "q_len": 1})
        o1, l1 = oracle.decode_all(y)
        np.testing.assert_allclose(out[:, i], o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, i], l1, rtol=0, atol=1e-12)


def test_multi_token_causal_boundary_with_a_spike_key():
    """A spike key at position p is seen by the query tokens at or after p
    (they return its value row) and by none before it."""
    d, L, Q = 8, 40, 5
    x = synth.generate(1, 2, 1, d, [L], q_len=Q, seed=42)
    q = np.zeros((1, Q, 2, d), np.float32)
    q[..., 0] = 8.0
    k = np.zeros_like(x.k)
    p = L - 3  # the position of query token Q - 3
    k[p, 0, 0] = bf16_bits(np.float32(5.0))
    y = DecodeInputs(**{**x.__dict__, "q": bf16_bits(q), "k": k, "sm_scale": 1.0})
    out, lse = oracle.decode_all(y)
    _, vf = dense_kv(y, 0)
    for i in range(Q):
        me = L - Q + i
        if me >= p:
            np.testing.assert_allclose(out[0, i, 0], vf[p, 0], atol=1e-12)
        else:
            np.testing.assert_allclose(out[0, i, 0], vf[:me + 1, 0].mean(axis=0), atol=1e-12)
            assert abs(lse[0, i, 0] - math.log(me + 1)) < 1e-12


def test_multi_token_shorter_request_than_query_block():
    """A query token whose position would be negative (L < q_len) sees no key:
    out = 0, lse = -inf; the others behave as usual."""
    x = synth.generate(1, 2, 1, 8, [2], q_len=4, seed=43)
    out, lse = oracle.decode_all(x)
    assert np.isneginf(lse[0, :2]).all() and (out[0, :2] == 0).all()
    assert np.isfinite(lse[0, 2:]).all()


# ------------------------------------------------------------ logit soft-cap
# Each scaled score s becomes cap * tanh(s / cap) before the softmax (Gemma
# 2's soft-capping; the pages name the variant without the formula).

def test_softcap_two_keys_closed_form():
    """Two keys with scaled scores a, b: weights follow the capped scores."""
    a_, b_, cap = 3.0, -1.5, 2.0
    q = [[[1.0, 0.0]]]
    k = [[[a_, 0.0]], [[b_, 0.0]]]
    v = [[[1.0, 2.0]], [[-3.0, 0.5]]]
    x = contiguous_inputs(q, k, v, [2], sm_scale=1.0)
    x = DecodeInputs(**{**x.__dict__, "logit_cap": cap})
    out, lse = oracle.decode_all(x)
    ca, cb = cap * math.tanh(a_ / cap), cap * math.tanh(b_ / cap)
    wa = math.exp(ca) / (math.exp(ca) + math.exp(cb))
    np.testing.assert_allclose(out[0, 0], [wa * 1.0 + (1 - wa) * -3.0, wa * 2.0 + (1 - wa) * 0.5],
                               rtol=0, atol=1e-14)
    assert abs(lse[0, 0] - math.log(math.exp(ca) + math.exp(cb))) < 1e-14


def test_softcap_limits_and_brute_force():
    x = synth.generate(2, 4, 2, 16, [40, 7], seed=44, sm_scale=0.9)
    plain_out, plain_lse = oracle.decode_all(x)
    # a cap far above every score changes nothing (tanh(s/c)*c = s - s^3/(3c^2) ...)
    big = DecodeInputs(**{**x.__dict__, "logit_cap": 1e7})
    o, l = oracle.decode_all(big)
    np.testing.assert_allclose(o, plain_out, rtol=0, atol=1e-10)
    np.testing.assert_allclose(l, plain_lse, rtol=0, atol=1e-10)
    # a small cap: numpy restatement of the capped softmax
    cap = 1.5
    y = DecodeInputs(**{**x.__dict__, "logit_cap": cap})
    o, l = oracle.decode_all(y)
    qf = bf16_values(x.q)
    for b in range(2):
        kf, vf = dense_kv(x, b)
        for h in range(4):
            s = cap * np.tanh(x.sm_scale * (kf[:, h // 2] @ qf[b, h]) / cap)
            w = np.exp(s - s.max())
            np.testing.assert_allclose(o[b, h], (w / w.sum()) @ vf[:, h // 2], rtol=0, atol=1e-12)
            assert abs(l[b, h] - (s.max() + math.log(w.sum()))) < 1e-12


# ---------------------------------------------------------------- int4 KV
def test_int4_nibble_decoding_by_hand():
    """Two's-complement nibbles, the even element in the low nibble (the
    reading of INT4 KV on "Beyond the Memory Wall", section "2. FlashInfer",
    which names the format without its layout)."""
    table = {0x00: (0, 0), 0x7F: (-1, 7), 0x80: (0, -8), 0x19: (-7, 1), 0xF8: (-8, -1),
             0x07: (7, 0), 0x88: (-8, -8), 0x21: (1, 2)}
    got = oracle.int4_codes(np.array([list(table)], np.uint8))[0]
    assert list(got) == [c for pair in table.values() for c in pair]
    assert np.array_equal(int4_values(np.array(list(table), np.uint8)), got.astype(np.float64))


def _int4_pack_by_hand(codes):
    """[..., d] ints in [-8, 7] -> bytes, element 2i low nibble of byte i."""
    c = np.asarray(codes, np.int64) % 16
    return (c[..., 0::2] + 16 * c[..., 1::2]).astype(np.uint8)


def _int4_inputs(qv, kc, vc, lens, k_scale, v_scale, sm_scale=1.0, window=-1):
    x = contiguous_inputs(qv, np.zeros(kc.shape, np.float32), np.zeros(vc.shape, np.float32), lens,
                          sm_scale=sm_scale, window=window)
    return DecodeInputs(**{**x.__dict__, "kv_dtype": "int4", "k": _int4_pack_by_hand(kc),
                           "v": _int4_pack_by_hand(vc),
                           "k_scale": np.asarray(k_scale, np.float32),
                           "v_scale": np.asarray(v_scale, np.float32)})


def test_int4_constant_keys_and_scales():
    """All K codes equal: every score equal, out = mean of the dequantised V
    rows (codes x the head's V scale), lse = score + ln |J|; the scales are
    per kv head and separate for K and V."""
    rng = np.random.default_rng(4)
    L, d = 77, 8
    qv = rng.integers(-4, 5, size=(1, 4, d)).astype(np.float32)
    kc = np.empty((L, 2, d), np.int64)
    kc[:, 0], kc[:, 1] = 3, -5
    vc = rng.integers(-8, 8, size=(L, 2, d))
    ks, vs = [0.5, 0.25], [0.125, 2.0]
    for window in (-1, 9):
        out, lse = oracle.decode_all(_int4_inputs(qv, kc, vc, [L], ks, vs, 0.5, window))
        lo = L - window if window > 0 else 0
        for h in range(4):
            g = h // 2
            np.testing.assert_allclose(out[0, h], vc[lo:, g].mean(axis=0) * vs[g], atol=1e-12)
            s = 0.5 * float(qv[0, h] @ np.full(d, kc[0, g, 0])) * ks[g]
            assert abs(lse[0, h] - (s + math.log(L - lo))) < 1e-12


def test_int4_spike_pins_the_nibble_and_head():
    """One key holds code 7 at an odd dimension (a high nibble) of kv head 1;
    q is one-hot there, the K scale makes that score 40 and every other 0:
    out = that key's V row to within n e^-40.  The same code placed at the
    neighbouring even dimension (the low nibble of the same byte) scores 0."""
    L, d = 64, 8
    q = np.zeros((1, 4, d), np.float32)
    q[0, :, 3] = 1.0
    vc = np.random.default_rng(5).integers(-8, 8, size=(L, 2, d))
    for dim, hit in ((3, True), (2, False)):
        kc = np.zeros((L, 2, d), np.int64)
        kc[41, 1, dim] = 7
        out, lse = oracle.decode_all(_int4_inputs(q, kc, vc, [L], [1.0, 40.0 / 7.0], [1.0, 0.5]))
        if hit:
            np.testing.assert_allclose(out[0, 2], vc[41, 1] * 0.5, atol=1e-12)
            s = 7.0 * float(np.float32(40.0 / 7.0))  # the stored fp32 scale
            assert abs(lse[0, 3] - (s + math.log1p((L - 1) * math.exp(-s)))) < 1e-12
        else:
            np.testing.assert_allclose(out[0, 2], vc[:, 1].mean(axis=0) * 0.5, atol=1e-12)
            assert abs(lse[0, 3] - math.log(L)) < 1e-12
        np.testing.assert_allclose(out[0, 0], vc[:, 0].mean(axis=0), atol=1e-12)  # kv head 0


def test_int4_quantised_inputs_follow_the_recipe():
    """synth's INT4 inputs decode (by the independent numpy decoder) to
    integers in [-7, 7] times a per-head scale of amax / 7: the largest code
    of every head has magnitude 7."""
    x = synth.generate(1, 4, 2, 16, [300], kv_dtype="int4", seed=12)
    for arr in (x.k, x.v):
        codes = int4_values(arr)
        assert codes.min() >= -7 and codes.max() <= 7
        assert (np.abs(codes).max(axis=(0, 2)) == 7).all()

