"""Full-size parity of every launch the benchmark times.

For each (workload, mode) of the benchmark's sweep -- the headline batched
paged decode, the long-context fp8 and int4 decodes, the MHA, Gemma- and
Llama-3-shaped decodes, several query tokens, soft-capping, the forced
dataflows and the unified max -- the pass is built by the benchmark's own
runner (same plan, grid, split and launch), run once, and EVERY output row
and lse is compared with the fp64 oracle under the stated tolerances
(out: max-abs 1e-2, max-rel 1e-2 over |ref| >= 1e-3; lse: max-abs 1e-3).
The oracle is the plain definition ("Forcing Flash Attention onto a TPU",
section "Standard causal attention").  A mode whose dataflow has no kernel
for the workload's rows is skipped, as the sweep reports it as an error.
"""
import numpy as np
import pytest

import bench
from gqa_decode_attention_split_b200 import synth
from gpu_util import assert_matches, to_numpy
from oracle import oracle

# the headline pass itself, then the sweep; grouped by workload so that each
# full-size workload is generated and run through the oracle once
JOBS = sorted({(bench.HEADLINE, "auto"), *bench.sweep_jobs()})

_cache = {}


def _workload(name):
    if name not in _cache:
        _cache.clear()  # keep one full-size workload in host memory at a time
        x = synth.workload(name)
        _cache[name] = (x, oracle.decode_all(x))
    return _cache[name]


def test_every_sweep_workload_is_covered():
    names = {n for n, _ in JOBS}
    assert set(bench.SWEEP) <= names and bench.HEADLINE in names


@pytest.mark.gpu
@pytest.mark.parametrize("job", JOBS, ids=[bench.sweep_key(n, m) for n, m in JOBS])
def test_sweep_launch_matches_the_oracle(job):
    import torch
    name, mode = job
    x, (ref_o, ref_l) = _workload(name)
    r = bench.make_runner(x, mode)
    r.step()
    torch.cuda.synchronize()
    r.check_status()
    o, l = to_numpy(r.out, r.lse)
    assert o.shape == ref_o.shape
    assert_matches(o, l, ref_o, ref_l, what=f"{bench.sweep_key(name, mode)} all rows")
    # a second pass in the same runner (as the timed loop runs it) is identical
    r.step()
    torch.cuda.synchronize()
    r.check_status()
    o2, l2 = to_numpy(r.out, r.lse)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(l2, l)
    del r
    torch.cuda.empty_cache()
