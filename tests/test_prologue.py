"""GPU parity of the fused mixer prologue (gdr_chunk_fwd_ex / gdr_decode_step_ex) against the
fp64 oracle: raw q, k, beta logits and gate logits go to the kernels, and the oracle applies its
own prologue (q/k L2 normalisation, sigmoid, g = -A softplus(a)) in fp64 to the same values
before its recurrence. Bars as in the other parity tests: max |GPU - oracle| <= 1e-4 * rms for
fp32 inputs, 2e-2 * rms for bf16 inputs, for o and S_T.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200.inputs import make_raw_chunk_inputs
from gpu_util import BF16_HALF_ULP, TOL, guard_ok, guarded_empty, rel_err

pytestmark = pytest.mark.gpu

MODES = ("none", "scalar", "channel")


def _flags(mode, norm=True, sig=True, gate=True):
    return dict(l2norm_qk=norm, beta_sigmoid=sig, gate_softplus=gate and mode != "none")


def run_and_check(x, mode, dtype, flags, label="", out_dtype=torch.float32):
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o, obuf = guarded_empty((B, T, H, dv), out_dtype, "cuda")
    st, sbuf = guarded_empty((B, H, dv, dk), torch.float32, "cuda")
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode=mode, out=o, state_out=st,
                  gate_scale=d["gate_scale"], **flags)
    gdr.sync_status()
    assert guard_ok(obuf, o.numel()) and guard_ok(sbuf, st.numel()), f"{label}: write past an output"
    q, k, b, g = oracle.prologue(x["q"], x["k"], x["beta"], x["g"], mode, gate_scale=x["gate_scale"], **flags)
    o_ref, s_ref = oracle.recurrent(q, k, x["v"].double(), g, b, mode, S0=x["S0"], f64_inputs=True)
    og, sg = o.double().cpu().numpy(), st.double().cpu().numpy()
    assert not np.isnan(og).any() and not np.isnan(sg).any(), f"{label}: NaN or unwritten output"
    eo, rms = rel_err(og, o_ref)
    es, _ = rel_err(sg, s_ref)
    if out_dtype == torch.bfloat16:  # plus each element's own bf16 rounding, 2^-8 |o_ref|
        excess = np.abs(og - o_ref) - (TOL[dtype] * rms + BF16_HALF_ULP * np.abs(o_ref))
        assert excess.max() <= 0, f"{label}: bf16 o exceeds its bound by {excess.max():.3e}"
    else:
        assert eo <= TOL[dtype], f"{label}: o max err {eo:.3e} * rms > {TOL[dtype]}"
    assert es <= TOL[dtype], f"{label}: S_T max err {es:.3e} * rms > {TOL[dtype]}"
    return eo, es


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,d,T,B,H,plan", [
    ("bf16", 128, 200, 2, 3, None),     # tensor cores: fused
    ("bf16", 128, 130, 8, 8, None),     # tensor cores: prep + fused (channel: fused)
    ("bf16", 128, 70, 13, 8, "two_pass"),
    ("f32", 64, 200, 2, 3, "cuda_core"),   # token recurrence, ragged last block
    ("f32", 64, 300, 1, 2, "cuda_core"),   # CUDA-core chunk form, ragged last chunk
    ("bf16", 64, 300, 1, 2, "cuda_core"),
    ("f32", 32, 1, 1, 2, "cuda_core"),
])
def test_prologue_chunk_all_steps(mode, dtype, d, T, B, H, plan):
    got, _ = gdr.chunk_fwd_plan(B, T, H, d, d, 64, mode, torch.bfloat16 if dtype == "bf16" else torch.float32)
    if plan is not None:
        assert got == plan
    seed = 7000 + 10 * MODES.index(mode) + d + T + B * H
    x = make_raw_chunk_inputs(B, T, H, d, d, mode, dtype, seed, s0_std=0.05)
    run_and_check(x, mode, dtype, _flags(mode), label=f"{mode}/{dtype}/d{d}/T{T}/B{B}H{H}")


@pytest.mark.parametrize("mode", ["scalar", "channel"])
@pytest.mark.parametrize("which", ["norm", "sig", "gate"])
def test_prologue_chunk_each_step_alone(mode, which):
    """One prologue step at a time on the tensor-core path; the other inputs are given in their
    final form (unit vectors, beta in (0, 1), g <= 0), read by both sides as they are."""
    x = make_raw_chunk_inputs(2, 150, 2, 128, 128, mode, "bf16", 7400 + len(which), s0_std=0.05)
    flags = dict(l2norm_qk=which == "norm", beta_sigmoid=which == "sig", gate_softplus=which == "gate")
    if which != "norm":
        for name in ("q", "k"):
            t = x[name].float()
            x[name] = (t / t.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    if which != "sig":
        x["beta"] = torch.rand(x["beta"].shape, generator=torch.Generator().manual_seed(1))
    if which != "gate":
        x["g"] = -0.05 * torch.rand(x["g"].shape, generator=torch.Generator().manual_seed(2))
    run_and_check(x, mode, "bf16", flags, label=f"{mode}/{which}")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_prologue_zero_vectors_stay_zero(dtype, d):
    """All-zero q and k vectors normalise to zero (no NaN): a zero key writes nothing, a zero query
    reads zero."""
    x = make_raw_chunk_inputs(1, 140, 2, d, d, "scalar", dtype, 7500 + d, s0_std=0.05)
    x["q"][0, 5] = 0
    x["k"][0, 7] = 0
    x["k"][0, 64:66] = 0  # a chunk boundary
    x["q"][0, 139, 1] = 0  # the last token
    run_and_check(x, "scalar", dtype, _flags("scalar"), label=f"zero vectors {dtype}")


def test_prologue_channel_strong_decays():
    """Gate scales large enough that many key channels' cumulative decay spreads past the channel
    gate's factored range inside a chunk (their terms go to the CUDA cores), with normalisation."""
    x = make_raw_chunk_inputs(2, 200, 3, 128, 128, "channel", "bf16", 7600, s0_std=0.05)
    x["gate_scale"] = torch.tensor([0.05, 2.0, 12.0])
    run_and_check(x, "channel", "bf16", _flags("channel"), label="channel strong")


def test_prologue_bf16_output():
    x = make_raw_chunk_inputs(2, 200, 2, 128, 128, "scalar", "bf16", 7700, s0_std=0.05)
    run_and_check(x, "scalar", "bf16", _flags("scalar"), label="bf16 out", out_dtype=torch.bfloat16)


def test_prologue_flags_off_is_plain_call():
    """No flag set: the binding calls gdr_chunk_fwd; gdr_chunk_fwd_ex with prologue 0 gives the
    same bits."""
    x = make_raw_chunk_inputs(2, 150, 2, 128, 128, "scalar", "bf16", 7800, s0_std=0.05)
    for name in ("q", "k"):
        t = x[name].float()
        x[name] = (t / t.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    x["beta"] = torch.rand(x["beta"].shape, generator=torch.Generator().manual_seed(3))
    x["g"] = -0.05 * torch.rand(x["g"].shape, generator=torch.Generator().manual_seed(4))
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    o1, s1 = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode="scalar")
    B, T, H, dk = d["q"].shape
    o2 = torch.empty_like(o1)
    s2 = torch.empty_like(s1)
    lib = gdr.lib()
    ws = torch.empty(max(1, gdr.workspace_bytes(B, T, H, dk, dk, 64, "scalar", torch.bfloat16)), dtype=torch.uint8,
                     device="cuda")
    rc = lib.gdr_chunk_fwd_ex(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(),
                              d["beta"].data_ptr(), d["S0"].data_ptr(), o2.data_ptr(), s2.data_ptr(), B, T, H, dk, dk,
                              64, 1, 1, 0, 0, None, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    gdr.sync_status()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("f32", 64, 40), ("bf16", 256, 96)])
def test_prologue_decode_steps(mode, dtype, dk, dv):
    """Four decode steps with the prologue on raw tokens, against the oracle's prologue and
    recurrence step by step (outputs of every step and the final states)."""
    B, H, steps = 4, 3, 4
    gen = torch.Generator().manual_seed(7900 + dk + dv + MODES.index(mode))
    S = (0.02 * torch.randn(B, H, dv, dk, generator=gen)).contiguous()
    S_ref = S.double().numpy()
    Sd = S.cuda()
    flags = _flags(mode)
    for step in range(steps):
        x = make_raw_chunk_inputs(B, 1, H, dk, dv, mode, dtype, 8000 + 31 * step + dk + MODES.index(mode))
        tok = {n: (None if t is None else (t[:, 0].contiguous() if n != "gate_scale" else t)) for n, t in x.items()}
        dd = {n: (None if t is None else t.cuda()) for n, t in tok.items()}
        o = gdr.decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], Sd, mode=mode, gate_scale=dd["gate_scale"],
                            **flags)
        gdr.sync_status()
        q, k, b, g = oracle.prologue(x["q"], x["k"], x["beta"], x["g"], mode, gate_scale=x["gate_scale"], **flags)
        o_ref, S_ref_new = oracle.recurrent(q, k, x["v"].double(), g, b, mode, S0=S_ref, f64_inputs=True)
        S_ref = S_ref_new
        eo, _ = rel_err(o.double().cpu().numpy(), o_ref[:, 0])
        assert eo <= TOL[dtype], f"step {step}: o err {eo:.3e}"
    es, _ = rel_err(Sd.double().cpu().numpy(), S_ref)
    assert es <= TOL[dtype], f"final state err {es:.3e}"


@pytest.mark.parametrize("mode,T", [("scalar", 1024), ("channel", 2048)])
def test_prologue_prep_fused_more_precomputed_chunks(mode, T):
    """64 heads: with the prologue the fused plan pre-computes more leading chunks than the plain call
    (scalar gate, 16 chunks: 11 against 9; channel gate, 32 chunks: 28 against 27) inside the plain
    call's workspace; every step against the oracle."""
    NC = T // 64
    plan, c1 = gdr.chunk_fwd_plan(8, T, 8, 128, 128, 64, mode, torch.bfloat16)
    assert plan == "prep_fused" and 0 < c1 < NC
    x = make_raw_chunk_inputs(8, T, 8, 128, 128, mode, "bf16", 7900 + MODES.index(mode), s0_std=0.05)
    run_and_check(x, mode, "bf16", _flags(mode), label=f"{mode} 64 heads T={T}")
