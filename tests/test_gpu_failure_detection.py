"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait in the library's kernels is bounded by a wall-clock limit; when it
runs out the kernel records code 1 in the device error word and returns, and
the context stays usable.  Here a dedicated kernel waits on a barrier nothing
ever completes, with the limit shortened to 1 ms: the call must come back, the
word must read 1, and the next decode on the same context must still match the
oracle.  No kernel here faults, traps or waits without a bound.
"""
import time

import pytest
import torch

import oracle
from covariance_corrected_softmax_b200 import plx, workloads as W
from parity_util import check_out, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_wait_that_runs_out_is_reported_and_context_survives():
    assert plx.device_error(clear=True) == 0
    plx.set_wait_limit_ns(1_000_000)  # 1 ms
    try:
        t0 = time.perf_counter()
        plx.selftest_wait()
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        code = plx.device_error(clear=True)
    finally:
        plx.set_wait_limit_ns(0)  # back to the default
    assert code == 1, f"device error word {code}, expected 1 (wait timed out)"
    assert elapsed < 1.0, f"the timed-out wait took {elapsed:.3f} s"
    assert plx.device_error() == 0

    # the context is intact: a decode right after still matches the oracle
    shape = W.DecodeShape(B=3, Hq=16, Hkv=8, d=128, S_max=500, ctx=500, ragged=True)
    inp = W.make_decode(shape, seed=5, device=DEV)
    out = plx.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                     softmax_scale=1.0)
    torch.cuda.synchronize()
    ref, _ = oracle.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"],
                           inp["seqlens"], 1.0)
    check_out(to_np(out), ref, bf16=True, what="decode after a timed-out wait",
              output_rounding=True)
    assert plx.device_error() == 0


def test_default_limit_is_restored():
    """With the default limit (2 s) the same wait also ends, after about 2 s."""
    plx.set_wait_limit_ns(0)
    t0 = time.perf_counter()
    plx.selftest_wait()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert plx.device_error(clear=True) == 1
    assert 1.5 < elapsed < 10.0, elapsed
