"""GPU parity of Gated DeltaNet-2 (gdr_chunk_fwd_gdn2, gdr_decode_step_gdn2) against the fp64
oracle's Gated DeltaNet-2 recurrence (pinned in test_oracle.py), element by element, with the
forward's bars (1e-4 * rms for fp32 inputs, 2e-2 * rms for bf16)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200.inputs import make_chunk_inputs, make_gdn2_gates
from gpu_util import TOL, guard_ok, guarded_empty, rel_err

pytestmark = pytest.mark.gpu

MODES = ("none", "scalar", "channel")


def run_gdn2(x, e, w, mode, out_dtype=torch.float32):
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o, obuf = guarded_empty((B, T, H, dv), out_dtype, "cuda")
    st, sbuf = guarded_empty((B, H, dv, dk), torch.float32, "cuda")
    gdr.chunk_fwd_gdn2(d["q"], d["k"], d["v"], d["g"], e.cuda(), w.cuda(), d["S0"], mode=mode, out=o, state_out=st)
    gdr.sync_status()
    assert guard_ok(obuf, o.numel()) and guard_ok(sbuf, st.numel())
    return o.double().cpu().numpy(), st.double().cpu().numpy()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,dk,dv", [("f32", 64, 64), ("f32", 32, 32), ("bf16", 128, 128), ("f32", 64, 32),
                                         ("bf16", 32, 128)])
@pytest.mark.parametrize("T", [1, 63, 200, 300])
def test_gdn2_chunk(mode, dtype, dk, dv, T):
    """T <= 256 runs the token recurrence, T = 300 the chunk form (ragged last chunk); with S0."""
    seed = 11000 + 100 * MODES.index(mode) + dk + dv + T + (3 if dtype == "bf16" else 0)
    x = make_chunk_inputs(2, T, 3, dk, dv, mode, dtype, seed, s0_std=0.1)
    gw = make_gdn2_gates(2, T, 3, dk, dv, seed + 1)
    o, st = run_gdn2(x, gw["erase"], gw["write"], mode)
    o_ref, s_ref = oracle.recurrent_gdn2(x["q"], x["k"], x["v"], x["g"], gw["erase"], gw["write"], mode, S0=x["S0"])
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


@pytest.mark.parametrize("mode", MODES)
def test_gdn2_equal_gates_match_chunk_fwd(mode):
    """e = w = beta 1 gives gdr_chunk_fwd's result (fp32, the same CUDA-core arithmetic up to rounding)."""
    x = make_chunk_inputs(2, 300, 2, 64, 64, mode, "f32", 11500 + MODES.index(mode), s0_std=0.1)
    e = x["beta"][..., None].expand(-1, -1, -1, 64).contiguous()
    w = x["beta"][..., None].expand(-1, -1, -1, 64).contiguous()
    o2, s2 = run_gdn2(x, e, w, mode)
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    o1, s1 = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode=mode)
    o1 = o1.double().cpu().numpy()
    s1 = s1.double().cpu().numpy()
    assert rel_err(o2, o1)[0] <= 1e-5 and rel_err(s2, s1)[0] <= 1e-5


def test_gdn2_bf16_output_and_strong_decay():
    """Channel decays from -1e-3 to -1e4 and a bf16 output (bar plus each element's own rounding)."""
    x = make_chunk_inputs(1, 300, 2, 128, 128, "channel", "bf16", 11600, s0_std=0.1)
    gen = torch.Generator().manual_seed(11601)
    x["g"] = (-(10.0 ** (torch.rand(x["g"].shape, generator=gen) * 7.0 - 3.0))).contiguous()
    gw = make_gdn2_gates(1, 300, 2, 128, 128, 11602)
    o, st = run_gdn2(x, gw["erase"], gw["write"], "channel", out_dtype=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent_gdn2(x["q"], x["k"], x["v"], x["g"], gw["erase"], gw["write"], "channel",
                                         S0=x["S0"])
    rms = np.sqrt(np.mean(o_ref ** 2))
    assert (np.abs(o - o_ref) - (TOL["bf16"] * rms + 2.0 ** -8 * np.abs(o_ref))).max() <= 0
    assert rel_err(st, s_ref)[0] <= TOL["bf16"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 40), ("bf16", 256, 96)])
def test_gdn2_decode_steps(mode, dtype, dk, dv):
    B, H, steps = 4, 3, 4
    gen = torch.Generator().manual_seed(11700 + dk + dv + MODES.index(mode))
    S = (0.02 * torch.randn(B, H, dv, dk, generator=gen)).contiguous()
    S_ref = S.double().numpy()
    Sd = S.cuda()
    for step in range(steps):
        x = make_chunk_inputs(B, 1, H, dk, dv, mode, dtype, 11800 + 31 * step + dk)
        gw = make_gdn2_gates(B, 1, H, dk, dv, 11900 + step)
        tok = lambda t: None if t is None else t[:, 0].contiguous()
        o = gdr.decode_step_gdn2(tok(x["q"]).cuda(), tok(x["k"]).cuda(), tok(x["v"]).cuda(),
                                 None if x["g"] is None else tok(x["g"]).cuda(), tok(gw["erase"]).cuda(),
                                 tok(gw["write"]).cuda(), Sd, mode=mode)
        gdr.sync_status()
        o_ref, S_ref = oracle.recurrent_gdn2(x["q"], x["k"], x["v"], x["g"], gw["erase"], gw["write"], mode, S0=S_ref)
        assert rel_err(o.double().cpu().numpy(), o_ref[:, 0])[0] <= TOL[dtype], step
    assert rel_err(Sd.double().cpu().numpy(), S_ref)[0] <= TOL[dtype]


def test_gdn2_tensor_core_kda_workload_shape():
    """The channel decay at the tensor-core shapes runs the channel gate's tensor-core passes: the
    Kimi Delta Attention workload's shape (B = 4, H = 16, d = 128) at T = 2048, with 16 channels
    decaying strongly (their terms on the CUDA cores), whole output against the oracle."""
    x = make_chunk_inputs(4, 2048, 16, 128, 128, "channel", "bf16", 11950, s0_std=0.05)
    x["g"][..., :16] *= 400.0  # spread far past the factored range on channels 0-15
    gw = make_gdn2_gates(4, 2048, 16, 128, 128, 11951)
    assert gdr._lib.lib().gdr_chunk_fwd_gdn2_workspace_bytes(4, 2048, 16, 128, 128, 64, 2, 1, 0) > 0
    o, st = run_gdn2(x, gw["erase"], gw["write"], "channel")
    o_ref, s_ref = oracle.recurrent_gdn2(x["q"], x["k"], x["v"], x["g"], gw["erase"], gw["write"], "channel",
                                         S0=x["S0"])
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    print(f"gdn2 tensor cores: o {eo:.3e}, S_T {es:.3e}")
    assert eo <= TOL["bf16"] and es <= TOL["bf16"]


@pytest.mark.parametrize("B,H,T", [(13, 8, 130), (1, 8, 700)])
def test_gdn2_tensor_core_plans(B, H, T):
    """Gated DeltaNet-2 on the channel gate's tensor-core plans: 104 heads (two passes) and 8 heads
    (fused, 11 chunks through the ring, ragged tail), with S0, whole output against the oracle."""
    x = make_chunk_inputs(B, T, H, 128, 128, "channel", "bf16", 12000 + B * H + T, s0_std=0.05)
    gw = make_gdn2_gates(B, T, H, 128, 128, 12001 + B * H + T)
    o, st = run_gdn2(x, gw["erase"], gw["write"], "channel")
    o_ref, s_ref = oracle.recurrent_gdn2(x["q"], x["k"], x["v"], x["g"], gw["erase"], gw["write"], "channel",
                                         S0=x["S0"])
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)
