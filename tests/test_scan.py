"""GPU parity of the segment scan (gdr_chunk_fwd_scan) against the fp64 oracle: segments run in
parallel from a zero state, the incoming states are carried across and the outputs corrected. The
result must match the oracle's token recurrence with the bf16 bar (2e-2 * rms), for o and S_T."""
import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200.inputs import CHUNK_WORKLOADS, make_chunk_inputs, workload_inputs
from gpu_util import BF16_HALF_ULP, TOL, guard_ok, guarded_empty, rel_err

pytestmark = pytest.mark.gpu

MODES = ("none", "scalar", "channel")


def run_scan(x, mode, n_seg, out_dtype=torch.float32, inplace=False):
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o, obuf = guarded_empty((B, T, H, dv), out_dtype, "cuda")
    if inplace and d["S0"] is not None:
        st = d["S0"]
        sbuf = None
    else:
        st, sbuf = guarded_empty((B, H, dv, dk), torch.float32, "cuda")
    gdr.chunk_fwd_scan(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], n_seg=n_seg, mode=mode, out=o,
                       state_out=st)
    gdr.sync_status()
    assert guard_ok(obuf, o.numel())
    if sbuf is not None:
        assert guard_ok(sbuf, st.numel())
    return o.double().cpu().numpy(), st.double().cpu().numpy()


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("n_seg", [2, 4, 8])
@pytest.mark.parametrize("with_s0", [False, True])
def test_scan_small(mode, n_seg, with_s0):
    """B = 2, H = 3, T = 512 (8 chunks): segments of 4, 2 and 1 chunks; with and without S0."""
    seed = 12000 + 10 * MODES.index(mode) + n_seg + (5 if with_s0 else 0)
    x = make_chunk_inputs(2, 512, 3, 128, 128, mode, "bf16", seed, s0_std=0.05 if with_s0 else None)
    o, st = run_scan(x, mode, n_seg)
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=x["S0"])
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_scan_bf16_output_inplace_state_and_strong_decay(mode):
    """bf16 o (bar plus each element's own rounding), S_T written over S0, and log-decays spread
    from -1e-3 to -30 so that the segments' transitions range from nearly the identity to zero."""
    x = make_chunk_inputs(1, 768, 2, 128, 128, mode, "bf16", 12100 + MODES.index(mode), s0_std=0.05)
    gen = torch.Generator().manual_seed(12101)
    x["g"] = (-(10.0 ** (torch.rand(x["g"].shape, generator=gen) * 4.5 - 3.0))).contiguous()
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=x["S0"])
    o, st = run_scan(x, mode, 3, out_dtype=torch.bfloat16, inplace=True)
    rms = np.sqrt(np.mean(o_ref ** 2))
    assert (np.abs(o - o_ref) - (TOL["bf16"] * rms + BF16_HALF_ULP * np.abs(o_ref))).max() <= 0
    assert rel_err(st, s_ref)[0] <= TOL["bf16"]


def test_scan_long_sequence_workload():
    """The long-sequence workload (Gated DeltaNet, B = 1, H = 16, T = 65536) in 8 segments, whole
    output against the oracle."""
    w = CHUNK_WORKLOADS["gdn_bf16_b1_h16_t65536_d128"]
    x = workload_inputs(w)
    o, st = run_scan(x, w.mode, 8)
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], w.mode, S0=x["S0"])
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    print(f"scan n_seg=8: max|do|/rms = {eo:.3e}, max|dS|/rms = {es:.3e}")
    assert eo <= TOL["bf16"] and es <= TOL["bf16"]


def test_scan_rejects_unsupported():
    x = make_chunk_inputs(1, 200, 1, 128, 128, "scalar", "bf16", 1)
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    with pytest.raises(gdr.GdrError) as e:  # T not a multiple of 64 * n_seg
        gdr.chunk_fwd_scan(d["q"], d["k"], d["v"], d["g"], d["beta"], n_seg=2, mode="scalar")
    assert e.value.status == "GDR_ERR_UNSUPPORTED"
    with pytest.raises(gdr.GdrError) as e:
        gdr.chunk_fwd_scan(d["q"], d["k"], d["v"], d["g"], d["beta"], n_seg=1, mode="scalar")
    assert e.value.status == "GDR_ERR_INVALID_ARG"


@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_scan_chosen_by_chunk_fwd_with_prologue(mode):
    """gdr_chunk_fwd picks the segment scan by itself for 2 heads of 32768 tokens (16 segments of 32
    chunks); with S0 and the fused prologue (raw q/k, beta and gate logits) against the oracle's
    prologue and recurrence."""
    from gated_delta_rule_143_b200.inputs import make_raw_chunk_inputs
    B, T, H = 1, 32768, 2
    assert gdr.chunk_fwd_plan(B, T, H, 128, 128, 64, mode, torch.bfloat16) == ("scan", 16)
    x = make_raw_chunk_inputs(B, T, H, 128, 128, mode, "bf16", 12300 + len(mode), s0_std=0.05)
    d = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    flags = dict(l2norm_qk=True, beta_sigmoid=True, gate_softplus=True)
    o, st = gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], mode=mode, gate_scale=d["gate_scale"],
                          **flags)
    gdr.sync_status()
    q, k, b, g = oracle.prologue(x["q"], x["k"], x["beta"], x["g"], mode, gate_scale=x["gate_scale"], **flags)
    o_ref, s_ref = oracle.recurrent(q, k, x["v"].double(), g, b, mode, S0=x["S0"], f64_inputs=True)
    eo, _ = rel_err(o.double().cpu().numpy(), o_ref)
    es, _ = rel_err(st.double().cpu().numpy(), s_ref)
    print(f"auto scan + prologue {mode}: o {eo:.3e}, S_T {es:.3e}")
    assert eo <= TOL["bf16"] and es <= TOL["bf16"]
