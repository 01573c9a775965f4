"""Device-side bounded waits: a wait that can never complete ends with GDR_ERR_TIMEOUT after its
bound, releases the CTA's other waiting roles through the abort flag, and leaves the stream usable.

gdr_selftest_bounded_wait runs a kernel laid out like the state pass (a copy role waiting on a ring
flag that nothing sets, an issue role waiting on the copy role, epilogue warps waiting on the issue
role). The copy role's bound is the one given; the others' are 100 times longer, so a run that ends
near the short bound shows the abort flag at work. Nothing faults, traps or spins without a bound.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200 import _lib
from gated_delta_rule_143_b200.inputs import make_chunk_inputs
from gpu_util import TOL, rel_err, run_chunk

GDR_ERR_TIMEOUT = -6


def test_selftest_rejects_bad_bound_on_host():
    el = ctypes.c_ulonglong(0)
    assert _lib.lib().gdr_selftest_bounded_wait(0, ctypes.byref(el), None) == -1
    assert _lib.lib().gdr_selftest_bounded_wait(2000000, ctypes.byref(el), None) == -1


@pytest.mark.gpu
def test_bounded_wait_times_out_then_stream_is_usable():
    stream = torch.cuda.current_stream()
    for limit_us in (1000, 5000):
        el = ctypes.c_ulonglong(0)
        t0 = time.perf_counter()
        rc = _lib.lib().gdr_selftest_bounded_wait(limit_us, ctypes.byref(el), stream.cuda_stream)
        wall = time.perf_counter() - t0
        assert rc == GDR_ERR_TIMEOUT, (rc, _lib.lib().gdr_last_error())
        # at least the short bound; far below the issue / epilogue roles' own (100x) bound
        assert limit_us * 1e3 <= el.value < 20 * limit_us * 1e3, el.value
        assert wall < 5.0
    gdr.sync_status()  # the status word was read and cleared: nothing pending
    # the same stream runs a normal forward correctly afterwards
    x = make_chunk_inputs(1, 200, 2, 128, 128, "scalar", "bf16", 303, s0_std=0.05)
    o, st = run_chunk(x, "scalar")
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], "scalar", S0=x["S0"])
    assert rel_err(o, o_ref)[0] <= TOL["bf16"]
    assert rel_err(st, s_ref)[0] <= TOL["bf16"]
