"""GPU parity of the backward pass (gdr_chunk_bwd) against the fp64 oracle's reverse-mode gradients
(pinned by central finite differences in test_oracle.py), element by element on the same seeded
inputs: dq, dk, dv, dg, dbeta, dS0. Bar: max |GPU - oracle| <= tol * rms(oracle) per gradient, with
the forward's tolerances (1e-4 for fp32 inputs, 2e-2 for bf16 inputs; the arithmetic is fp32 in
both cases).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200.inputs import make_chunk_inputs
from gpu_util import TOL, rel_err

pytestmark = pytest.mark.gpu

MODES = ("none", "scalar", "channel")


def upstream(B, T, H, dk, dv, dtype, seed, with_dst=True):
    gen = torch.Generator().manual_seed(seed)
    dO = torch.randn(B, T, H, dv, generator=gen).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    dST = torch.randn(B, H, dv, dk, generator=gen) if with_dst else None
    return dO.contiguous(), (None if dST is None else dST.contiguous())


def check_bwd(x, mode, dtype, dO, dST, label="", want_dS0=True):
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    got = gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dO.cuda(), S0=d["S0"],
                        dS_T=None if dST is None else dST.cuda(), mode=mode, want_dS0=want_dS0)
    gdr.sync_status()
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, dO, S0=x["S0"], dS_T=dST)
    errs = {}
    for name in ("dq", "dk", "dv", "dbeta", "dg", "dS0"):
        if ref[name] is None or (name == "dS0" and not want_dS0):
            assert got[name] is None
            continue
        g = got[name].double().cpu().numpy()
        assert not np.isnan(g).any(), f"{label}: NaN in {name}"
        e, rms = rel_err(g, ref[name])
        errs[name] = e
        assert e <= TOL[dtype], f"{label}: {name} max err {e:.3e} * rms (rms {rms:.3e}) > {TOL[dtype]}"
    return errs


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,dk,dv", [("f32", 64, 64), ("f32", 32, 32), ("bf16", 128, 128), ("f32", 64, 32),
                                         ("bf16", 32, 128)])
@pytest.mark.parametrize("T", [1, 63, 200])
def test_backward_small(mode, dtype, dk, dv, T):
    seed = 9000 + 100 * MODES.index(mode) + dk + dv + T + (3 if dtype == "bf16" else 0)
    x = make_chunk_inputs(2, T, 3, dk, dv, mode, dtype, seed, s0_std=0.1)
    dO, dST = upstream(2, T, 3, dk, dv, dtype, seed + 1)
    check_bwd(x, mode, dtype, dO, dST, label=f"{mode}/{dtype}/dk{dk}/dv{dv}/T{T}")


@pytest.mark.parametrize("mode", MODES)
def test_backward_optional_arguments(mode):
    """No S0, no dS_T, no dS0 output."""
    x = make_chunk_inputs(1, 100, 2, 64, 64, mode, "f32", 9500 + MODES.index(mode))
    dO, _ = upstream(1, 100, 2, 64, 64, "f32", 9510, with_dst=False)
    check_bwd(x, mode, "f32", dO, None, label=f"{mode} optional", want_dS0=False)


@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_backward_strong_decay(mode):
    """Log-decays from -1e-3 down to -1e4 (alpha = 0 resets the state): the gradients stay finite and
    match the oracle."""
    x = make_chunk_inputs(1, 150, 2, 64, 64, mode, "f32", 9600 + MODES.index(mode), s0_std=0.1)
    gen = torch.Generator().manual_seed(9601)
    mag = 10.0 ** (torch.rand(x["g"].shape, generator=gen) * 7.0 - 3.0)
    x["g"] = (-mag).contiguous()
    dO, dST = upstream(1, 150, 2, 64, 64, "f32", 9602)
    check_bwd(x, mode, "f32", dO, dST, label=f"{mode} strong decay")


@pytest.mark.parametrize("name,mode,B,H", [
    ("deltanet_bf16_b8_h8_d128", "none", 8, 8),
    ("gdn_bf16_b8_h8_d128", "scalar", 8, 8),
    ("kda_bf16_b4_h16_d128", "channel", 4, 16),
])
def test_backward_workload_shapes_reduced_T(name, mode, B, H):
    """The DeltaNet, Gated DeltaNet and Kimi Delta Attention workloads' shapes at T = 256."""
    T = 256
    x = make_chunk_inputs(B, T, H, 128, 128, mode, "bf16", 9700 + MODES.index(mode))
    dO, _ = upstream(B, T, H, 128, 128, "bf16", 9710, with_dst=False)
    errs = check_bwd(x, mode, "bf16", dO, None, label=name)
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})


def test_backward_rejects_bad_arguments():
    x = make_chunk_inputs(1, 8, 1, 64, 64, "scalar", "f32", 1)
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    dO = torch.zeros(1, 8, 1, 64, device="cuda")
    with pytest.raises(gdr.GdrError) as e:
        gdr.chunk_bwd(d["q"], d["k"], d["v"], None, d["beta"], dO, mode="scalar")
    assert e.value.status == "GDR_ERR_INVALID_ARG"
    with pytest.raises(gdr.GdrError) as e:
        gdr.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dO, mode="scalar",
                      workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == "GDR_ERR_WORKSPACE"
