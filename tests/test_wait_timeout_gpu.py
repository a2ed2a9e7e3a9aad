"""Failure detection on the GPU without a fault: a bounded device wait that nothing completes
gives up after its limit, reports EOT_ERR_TIMEOUT through the status word, and leaves the
context usable.  The self-test kernel runs the library's own wait routines (the mbarrier wait
of every tensor-core kernel, the grid-wide barrier of the fused half-steps) with a 1 ms limit.
The host polls the stream with a deadline, so a wait that did not end would fail the test
instead of blocking it."""
import time

import numpy as np
import pytest

import eot_inputs
from harness import TOL, compare, gpu_run, oracle_run

LIMIT_NS = 1_000_000   # 1 ms


def _run_selftest(which):
    import torch
    from entropic_ot_attention_b200 import _abi
    scratch = torch.zeros(256, dtype=torch.uint8, device="cuda:0")
    stream = torch.cuda.current_stream()
    ev = torch.cuda.Event()
    t0 = time.monotonic()
    _abi.eot_wait_selftest(which, LIMIT_NS, scratch.data_ptr(), stream.cuda_stream)
    ev.record(stream)
    while not ev.query():
        assert time.monotonic() - t0 < 30.0, "the bounded wait did not end"
        time.sleep(0.001)
    word = int(scratch.view(torch.int32)[2].item())
    status = _abi.eot_last_device_status(scratch.data_ptr(), stream.cuda_stream)
    return status, word, time.monotonic() - t0


@pytest.mark.gpu
@pytest.mark.parametrize("which,name", [(0, "mbarrier"), (1, "grid barrier")])
def test_wait_that_nothing_completes_times_out(which, name):
    from entropic_ot_attention_b200 import _abi
    status, word, dt = _run_selftest(which)
    assert word == 2, f"{name} wait did not give up"
    assert status == _abi.EOT_ERR_TIMEOUT
    assert dt >= LIMIT_NS * 1e-9


@pytest.mark.gpu
def test_wait_that_completes_does_not_time_out():
    from entropic_ot_attention_b200 import _abi
    status, word, _ = _run_selftest(2)
    assert word == 1 and status == _abi.EOT_OK


@pytest.mark.gpu
def test_context_usable_after_a_timeout():
    """After a wait ran out, a forward + backward on the same context is exact to tolerance and
    leaves a clean status word."""
    from entropic_ot_attention_b200 import _abi
    status, _, _ = _run_selftest(0)
    assert status == _abi.EOT_ERR_TIMEOUT
    case = eot_inputs.dense_case(1, 2, 384, 64, 100, 6, 2, "bf16", seed=7, name="after_timeout")
    errs = compare(gpu_run(case), oracle_run(case))
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
    status, _, _ = _run_selftest(2)
    assert status == _abi.EOT_OK


def test_selftest_rejects_bad_arguments():
    """Host-side argument checks (nothing is enqueued; no GPU needed)."""
    from entropic_ot_attention_b200 import _abi
    aligned = 1 << 20
    assert _abi.lib.eot_wait_selftest(5, LIMIT_NS, aligned, None) == _abi.EOT_ERR_INVALID_ARGUMENT
    assert _abi.lib.eot_wait_selftest(0, LIMIT_NS, None, None) == _abi.EOT_ERR_INVALID_ARGUMENT
    assert _abi.lib.eot_wait_selftest(0, LIMIT_NS, aligned + 8, None) == _abi.EOT_ERR_INVALID_ARGUMENT
    assert _abi.lib.eot_wait_selftest(0, 0, aligned, None) == _abi.EOT_ERR_INVALID_ARGUMENT
    assert _abi.lib.eot_wait_selftest(0, 2_000_000_000, aligned, None) == _abi.EOT_ERR_INVALID_ARGUMENT
