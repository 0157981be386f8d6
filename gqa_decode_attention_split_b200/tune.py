"""Measure the dataflow-choice table on the current GPU.

"FlashDecoding++" explainer, section "Hardware-aware heuristic dataflow":
which implementation runs a decode shape is decided from measurements of the
shapes on the target GPU rather than from a fixed rule.  This script times a
grid of decode shapes (head_dim x kv dtype x rows per segment x visible K/V
bytes) with both dataflows and a few caps on the blocks per segment, keeps
for every shape the fastest configuration (the fixed rule unless another is
at least MARGIN faster), merges neighbouring byte ranges with the same
choice, and writes

  csrc/fa_tuning_b200.inc   rows of the built-in table (rebuild the library),
                            under --inc-dir (default: this package)
  tuning_b200.json          every measurement behind them, under --record-dir
                            (default: the working directory, outside the package)

Usage (one GPU):  python -m gqa_decode_attention_split_b200.tune [--quick]
The table can also be installed at run time with binding.set_tuning(rows).
Inputs are seeded synthetic values generated on the device; only timing is
measured here (parity of both dataflows is covered by the GPU tests).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys

_PKG = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(_PKG))

from gqa_decode_attention_split_b200 import binding  # noqa: E402

MARGIN = 0.03                    # an alternative must be this much faster,
MARGIN_US = 1.0                  # and by at least this many microseconds
PIECES = (0, 8, 2)               # 0: the planner's default (64)
BYTES = [1 << 18, 1 << 21, 1 << 24, 1 << 27, 1 << 30]
SHAPES = [(64, "bf16"), (128, "bf16"), (256, "bf16"), (128, "fp8_e4m3"), (256, "fp8_e4m3")]
KV_HEADS = 8
FLUSH_BELOW = 256 << 20          # smaller inputs: L2 flushed before every launch


def simt_rows(dtype):
    return (1, 2, 4) if dtype == "fp8_e4m3" else (1, 2, 4, 8)


def make_inputs(torch, d, dtype, rows, nbytes, seed):
    """Batch 1, contiguous, KV_HEADS kv heads with `rows` query heads each,
    as many keys as give `nbytes` of K and V."""
    es = 1 if dtype == "fp8_e4m3" else 2
    L = max(1, nbytes // (KV_HEADS * 2 * d * es))
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    q = torch.randn((1, rows * KV_HEADS, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((L, KV_HEADS, d), generator=g, device="cuda")
    v = torch.randn((L, KV_HEADS, d), generator=g, device="cuda")
    if dtype == "fp8_e4m3":
        k = k.to(torch.float8_e4m3fn).view(torch.uint8)
        v = v.to(torch.float8_e4m3fn).view(torch.uint8)
        ks = torch.ones(KV_HEADS, device="cuda")
        vs = torch.ones(KV_HEADS, device="cuda")
    else:
        k, v, ks, vs = k.to(torch.bfloat16), v.to(torch.bfloat16), None, None
    indptr = torch.tensor([0, L], dtype=torch.int32)
    return q, k, v, ks, vs, indptr, L


def time_config(torch, x, d, dtype, rows, path, pieces, flush, reps):
    q, k, v, ks, vs, indptr, L = x
    nbytes = L * KV_HEADS * 2 * d * (1 if dtype == "fp8_e4m3" else 2)
    kvd = binding.KV_FP8_E4M3 if dtype == "fp8_e4m3" else binding.KV_BF16
    binding.set_tuning([dict(head_dim=d, kv_dtype=kvd, rows_min=rows, rows_max=rows, bytes_min=0,
                             bytes_max=1 << 62, path=path, max_pieces=pieces)])
    try:
        p = binding.plan(1, rows * KV_HEADS, KV_HEADS, d, indptr, kv_dtype=dtype)
    finally:
        binding.set_tuning([])
    info = p.info()
    if info["path"] != path:
        return None  # no kernel for this dataflow
    ind_dev = indptr.cuda()
    ws = p.new_workspace()
    out = torch.empty((1, rows * KV_HEADS, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, rows * KV_HEADS), dtype=torch.float32, device="cuda")
    run = lambda: binding.run(p, q, k, v, ind_dev, k_scale=ks, v_scale=vs, out=out, lse=lse,
                              workspace=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    if binding.decode_status(ws) != 0:
        raise RuntimeError(f"device check bits set for {d} {dtype} rows {rows} path {path}")
    # CUDA events tick in steps of about 2 us: a trimmed mean over many
    # launches resolves differences finer than one step
    ts.sort()
    cut = len(ts) // 10
    kept = ts[cut:len(ts) - cut] or ts
    return {"us": round(statistics.fmean(kept), 2), "median_us": round(statistics.median(ts), 2),
            "ctas": info["num_ctas"], "bytes": nbytes}


def choose(configs):
    """The fixed rule's configuration unless another is faster by MARGIN and
    by MARGIN_US."""
    base = configs.get((binding.PATH_MMA, 0)) or configs.get((binding.PATH_SIMT, 0))
    best_key = min(configs, key=lambda c: configs[c]["us"])
    if configs[best_key]["us"] < min(base["us"] * (1 - MARGIN), base["us"] - MARGIN_US):
        return best_key
    return (binding.PATH_MMA, 0) if (binding.PATH_MMA, 0) in configs else (binding.PATH_SIMT, 0)


def table_rows(results):
    """Byte ranges split at the geometric midpoints of the measured sizes;
    neighbouring ranges with the same choice merged; rows only where the
    choice differs from the fixed rule."""
    rows = []
    for (d, dtype, r), per in sorted(results.items()):
        sizes = sorted(per)
        edges = [0] + [int(math.sqrt(a * b)) for a, b in zip(sizes, sizes[1:])] + [1 << 62]
        spans = []
        for i, s in enumerate(sizes):
            ch = tuple(per[s]["choice"])
            lo, hi = edges[i], edges[i + 1] - (0 if i + 1 == len(sizes) else 1)
            if spans and spans[-1][2] == ch:
                spans[-1][1] = hi
            else:
                spans.append([lo, hi, ch])
        for lo, hi, (path, pieces) in spans:
            if (path, pieces) == (binding.PATH_MMA, 0):
                continue
            rows.append(dict(head_dim=d, kv_dtype=1 if dtype == "fp8_e4m3" else 0, rows_min=r,
                             rows_max=r, bytes_min=lo, bytes_max=hi, path=path, max_pieces=pieces))
    return rows


def write_inc(rows, path):
    lines = ["// Built-in dataflow-choice table (rows of fa_tuning_entry), written by",
             "// gqa_decode_attention_split_b200/tune.py from measurements on a B200.",
             "// FA_TUNING_ROW(head_dim, kv_dtype, rows_min, rows_max, bytes_min, bytes_max, path, max_pieces)"]
    for r in rows:
        lines.append("FA_TUNING_ROW({head_dim}, {dt}, {rows_min}, {rows_max}, {bytes_min}LL, {bytes_max}LL, "
                     "{p}, {max_pieces})".format(dt="FA_KV_FP8_E4M3" if r["kv_dtype"] else "FA_KV_BF16",
                                                 p="FA_PATH_SIMT" if r["path"] == binding.PATH_SIMT
                                                 else "FA_PATH_MMA", **r))
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--quick", action="store_true", help="head_dim 128 bf16 only (a smoke run)")
    ap.add_argument("--reps", type=int, default=40)
    ap.add_argument("--inc-dir", default=_PKG,
                    help="where csrc/fa_tuning_b200.inc is written (default: this package)")
    ap.add_argument("--record-dir", default=".",
                    help="where the raw measurements (tuning_b200.json) are written")
    args = ap.parse_args()
    import torch
    flush = torch.empty(FLUSH_BELOW, dtype=torch.uint8, device="cuda")
    shapes = [(128, "bf16")] if args.quick else SHAPES
    results, record = {}, []
    seed = 11
    for d, dtype in shapes:
        for r in simt_rows(dtype):
            per = {}
            for nb in BYTES:
                seed += 1
                x = make_inputs(torch, d, dtype, r, nb, seed)
                configs = {}
                for path in (binding.PATH_MMA, binding.PATH_SIMT):
                    for pieces in PIECES:
                        t = time_config(torch, x, d, dtype, r, path, pieces,
                                        flush if nb < FLUSH_BELOW else None, args.reps)
                        if t is not None:
                            configs[(path, pieces)] = t
                ch = choose(configs)
                per[nb] = {"choice": ch}
                base = configs.get((binding.PATH_MMA, 0)) or configs[(binding.PATH_SIMT, 0)]
                rec = {"head_dim": d, "kv_dtype": dtype, "rows": r, "bytes": x[6] * KV_HEADS * 2 * d *
                       (1 if dtype == "fp8_e4m3" else 2), "configs": {
                           f"{'mma' if p == binding.PATH_MMA else 'simt'}/pieces={k or 64}": v
                           for (p, k), v in configs.items()},
                       "choice": f"{'mma' if ch[0] == binding.PATH_MMA else 'simt'}/pieces={ch[1] or 64}",
                       "speedup_vs_fixed_rule": round(base["us"] / configs[ch]["us"], 3)}
                record.append(rec)
                print(json.dumps(rec), flush=True)
                del x
                torch.cuda.empty_cache()
            results[(d, dtype, r)] = per
    rows = table_rows(results)
    os.makedirs(args.record_dir, exist_ok=True)
    with open(os.path.join(args.record_dir, "tuning_b200.json"), "w") as f:
        json.dump({"margin": MARGIN, "margin_us": MARGIN_US, "kv_heads": KV_HEADS, "flush_below_bytes": FLUSH_BELOW,
                   "gpu": torch.cuda.get_device_name(), "measurements": record, "table": rows}, f,
                  indent=1)
    os.makedirs(os.path.join(args.inc_dir, "csrc"), exist_ok=True)
    write_inc(rows, os.path.join(args.inc_dir, "csrc", "fa_tuning_b200.inc"))
    print(f"{len(rows)} table rows written", flush=True)


if __name__ == "__main__":
    main()
