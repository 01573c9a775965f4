"""The allocation-free chunked forward, gdr_chunk_fwd_noalloc.

It exists for callers that cannot allocate device memory (a plugin whose host owns all device
memory, a loop where an allocation is not allowed, a program with a fixed device footprint): it
takes its scratch from a fixed area built into the library instead of a caller workspace.
The GPU test calls it through the C ABI twice in a row and checks each result against the
workspace entry point, gdr_chunk_fwd, on the same inputs, within the tolerance the parity tests
use. This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
from gated_delta_rule_143_b200 import _lib
from gated_delta_rule_143_b200.inputs import make_chunk_inputs

MODES = {"none": 0, "scalar": 1, "channel": 2}
BF16, F32 = 1, 0
TOL_BF16 = 2e-2  # the parity bar for bf16 inputs, max |diff| <= tol * rms


def _noalloc(q, k, v, g, beta, S0, o, S_T, B, T, H, mode, stream=None):
    p = lambda t: None if t is None else t.data_ptr()
    return _lib.lib().gdr_chunk_fwd_noalloc(p(q), p(k), p(v), p(g), p(beta), p(S0), p(o), p(S_T), B, T, H, 128, 128,
                                            64, MODES[mode], BF16, F32, stream)


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.abs(a - b).max() / np.sqrt(np.mean(b * b)))


def test_noalloc_rejects_oversized_problem_on_host():
    """B * H = 128 heads take the two-pass path, whose scratch holds one block per chunk:
    B * H * ceil(T / 64) = 8192 chunks needs far more than the built-in area, so the call is
    rejected before anything is enqueued (fake, widely spaced addresses; never dereferenced)."""
    M = 1 << 30
    need = _lib.lib().gdr_chunk_fwd_workspace_bytes(8, 4096, 16, 128, 128, 64, 1, BF16, F32)
    assert need > (32 << 20)
    rc = _lib.lib().gdr_chunk_fwd_noalloc(1 * M, 2 * M, 3 * M, 4 * M, 5 * M, None, 6 * M, None, 8, 4096, 16, 128, 128,
                                          64, 1, BF16, F32, None)
    assert rc == -2
    assert b"built-in area" in _lib.lib().gdr_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    cases = [("scalar", 2, 500, 4, 71), ("channel", 1, 1024, 8, 72)]  # 64 and 128 chunks
    for mode, B, T, H, seed in cases:
        x = make_chunk_inputs(B, T, H, 128, 128, mode, "bf16", seed, s0_std=0.05)
        d = {n: (None if t is None else t.cuda()) for n, t in x.items()}
        o_ref, s_ref = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode=mode)
        o = torch.full((B, T, H, 128), float("nan"), device="cuda")
        st = torch.full((B, H, 128, 128), float("nan"), device="cuda")
        rc = _noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, st, B, T, H, mode,
                      torch.cuda.current_stream().cuda_stream)
        assert rc == 0, _lib.lib().gdr_last_error()
        gdr.sync_status()
        assert not torch.isnan(o).any() and not torch.isnan(st).any()
        assert _rel(o, o_ref) <= TOL_BF16
        assert _rel(st, s_ref) <= TOL_BF16
