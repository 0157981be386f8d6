"""Host logic of the N > 1 benchmark path, run as two gloo ranks on the CPU.

With more than one GPU every rank decodes its own batch (replicas, no
data-path collective); the only cross-rank steps are the barrier around the
timed region and the max over ranks of each measured time.  These tests run
those steps, as bench.py calls them, in two processes.
"""
import argparse
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    try:
        dist.barrier()
        # rank r "measured" a different device time; every rank must see the max
        ms_total = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        ms_launch = bench.max_over_ranks(0.3 - 0.1 * rank, world, "cpu")
        agg = bench.aggregate(kv_bytes=2_000_000_000, batch=64, ms_total=ms_total, steps=10,
                              world=world)
        dist.barrier()
        # the reference arm: only rank 0 runs and prints; other ranks return at once
        ref_out = ""
        if rank != 0:
            buf = io.StringIO()
            args = argparse.Namespace(workload="gqa4_d64_L512", steps=1, warmup=0)
            with redirect_stdout(buf):
                bench.run_reference(args, rank, world)
            ref_out = buf.getvalue()
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_total": ms_total, "ms_launch": ms_launch, "agg": agg,
                       "ref_out": ref_out}, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_aggregate_weakly(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms_total"] == 15.0      # the slower rank's time, on every rank
        assert r["ms_launch"] == pytest.approx(0.3)
        # weak scaling: both ranks' bytes over the slowest rank's time
        assert r["agg"]["ms_per_step"] == pytest.approx(1.5)
        assert r["agg"]["value"] == pytest.approx(2 * 2e9 / 1.5e-3 / 1e9)
        assert r["agg"]["tokens_per_s"] == pytest.approx(2 * 64 / 1.5e-3)
    assert res[1]["ref_out"] == ""        # rank 1 printed nothing and did no work


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    agg = bench.aggregate(kv_bytes=1_000_000, batch=1, ms_total=2.0, steps=4, world=1)
    assert agg["ms_per_step"] == 0.5
    assert agg["value"] == pytest.approx(1e6 / 0.5e-3 / 1e9)
