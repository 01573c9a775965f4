"""The allocation-free chunked forward, gdr_chunk_fwd_noalloc.

It exists for callers that cannot allocate device memory (a plugin whose host owns all device
memory, a loop where an allocation is not allowed, a program with a fixed device footprint): it
takes its scratch from a fixed area built into the library instead of a caller workspace.
The GPU test calls it through the C ABI twice in a row per case, on an area left dirty by the
previous call, and requires each result to equal the workspace entry point's, gdr_chunk_fwd, on
the same inputs: the two run the same plan and kernels, so the outputs must agree to the bit.
This file is named to be collected last.
"""
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
from gated_delta_rule_143_b200 import _lib
from gated_delta_rule_143_b200.inputs import make_chunk_inputs

MODES = {"none": 0, "scalar": 1, "channel": 2}
BF16, F32 = 1, 0


def _noalloc(q, k, v, g, beta, S0, o, S_T, B, T, H, mode, stream=None):
    p = lambda t: None if t is None else t.data_ptr()
    return _lib.lib().gdr_chunk_fwd_noalloc(p(q), p(k), p(v), p(g), p(beta), p(S0), p(o), p(S_T), B, T, H, 128, 128,
                                            64, MODES[mode], BF16, F32, stream)


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
    cases = [("scalar", 2, 500, 4, 71), ("channel", 1, 1024, 8, 72), ("none", 7, 300, 8, 73)]
    for mode, B, T, H, seed in cases:
        x = make_chunk_inputs(B, T, H, 128, 128, mode, "bf16", seed, s0_std=0.05)
        d = {n: (None if t is None else t.cuda()) for n, t in x.items()}
        o_ref, s_ref = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode=mode)
        for call in range(2):  # the second call runs on the area the first one left behind
            o = torch.full((B, T, H, 128), float("nan"), device="cuda")
            st = torch.full((B, H, 128, 128), float("nan"), device="cuda")
            rc = _noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, st, B, T, H, mode,
                          torch.cuda.current_stream().cuda_stream)
            assert rc == 0, _lib.lib().gdr_last_error()
            gdr.sync_status()
            assert torch.equal(o, o_ref), f"{mode}: o differs from the workspace entry point (call {call})"
            assert torch.equal(st, s_ref), f"{mode}: S_T differs from the workspace entry point (call {call})"


@pytest.mark.gpu
def test_noalloc_long_few_heads_keeps_the_ring():
    """A shape gdr_chunk_fwd runs as a segment scan (2 heads, 512 chunks) still fits the built-in area
    through the fused kernel's 8-slot ring: the allocation-free entry point never takes the scan.
    Whole output against the oracle."""
    import oracle
    from gpu_util import TOL, rel_err
    B, T, H = 1, 32768, 2
    x = make_chunk_inputs(B, T, H, 128, 128, "scalar", "bf16", 74, s0_std=0.05)
    d = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    o = torch.full((B, T, H, 128), float("nan"), device="cuda")
    st = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    rc = _noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, st, B, T, H, "scalar",
                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    gdr.sync_status()
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], "scalar", S0=x["S0"])
    assert rel_err(o.double().cpu().numpy(), o_ref)[0] <= TOL["bf16"]
    assert rel_err(st.double().cpu().numpy(), s_ref)[0] <= TOL["bf16"]
