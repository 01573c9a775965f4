"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element, at small ragged sizes and at the full
workload sizes the bench times.

Bar: max |GPU - oracle| <= 1e-4 * rms(oracle) for fp32 inputs and
<= 2e-2 * rms(oracle) for bf16 inputs, for o and for the final state S_T.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_143_b200 as gdr
import oracle
from gated_delta_rule_143_b200.inputs import (CHUNK_WORKLOADS, DECODE_WORKLOADS, WORKLOAD_SEEDS,
                                              make_chunk_inputs, make_decode_state, make_decode_step,
                                              workload_inputs)
from gpu_util import BF16_HALF_ULP, TOL, guard_ok, guarded_empty, rel_err, run_chunk, to_dev

pytestmark = pytest.mark.gpu

MODES = ("none", "scalar", "channel")


def check_chunk(x, mode, dtype, S0=None, label=""):
    o, st = run_chunk(x, mode, S0=S0)
    s0 = x["S0"] if S0 is None else S0
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=s0)
    assert not np.isnan(o).any(), f"{label}: unwritten or NaN output"
    eo, _ = rel_err(o, o_ref)
    es, _ = rel_err(st, s_ref)
    assert eo <= TOL[dtype], f"{label}: o max err {eo:.3e} * rms > {TOL[dtype]}"
    assert es <= TOL[dtype], f"{label}: S_T max err {es:.3e} * rms > {TOL[dtype]}"
    return eo, es


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f32", 128), ("f32", 32), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("T", [1, 63, 200])
@pytest.mark.parametrize("with_s0", [False, True])
def test_chunk_small(mode, dtype, d, T, with_s0):
    """Several chunks plus a ragged tail; T = 1 and T = C - 1 edge cases."""
    seed = 1000 + 100 * MODES.index(mode) + d + T + (7 if with_s0 else 0) + (3 if dtype == "bf16" else 0)
    x = make_chunk_inputs(2, T, 3, d, d, mode, dtype, seed, s0_std=0.1 if with_s0 else None)
    check_chunk(x, mode, dtype, label=f"{mode}/{dtype}/d{d}/T{T}")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f32", 32), ("bf16", 64)])
def test_chunk_cuda_core_chunk_form(mode, dtype, d):
    """Past 256 tokens the CUDA-core path runs the chunk form (shorter sequences run the token
    recurrence): several chunks and a ragged tail, with S0, against the oracle."""
    seed = 5000 + 100 * MODES.index(mode) + d + (3 if dtype == "bf16" else 0)
    x = make_chunk_inputs(1, 300, 2, d, d, mode, dtype, seed, s0_std=0.1)
    check_chunk(x, mode, dtype, label=f"chunk form {mode}/{dtype}/d{d}")


@pytest.mark.parametrize("mode", ["none", "scalar"])
@pytest.mark.parametrize("B,H,T,plan", [
    (1, 1, 5000, "fused"),        # one head, 147 prep CTAs, 79 chunks through the 8-slot ring
    (3, 16, 333, "fused"),        # 48 heads
    (7, 8, 191, "fused"),         # 56 heads: the largest fused-only case
    (8, 8, 200, "prep_fused"),    # 64 heads: the first chunks prepared before the fused kernel
    (8, 8, 1000, "prep_fused"),   # 64 heads, 16 chunks (9 prepared before, 7 ring slots), ragged tail
    (8, 8, 50, "prep_fused"),     # 64 heads, one chunk: every chunk prepared before, no ring slot
    (12, 8, 100, "prep_fused"),   # 96 heads, two chunks, both prepared before
    (13, 8, 130, "two_pass"),     # 104 heads: prep kernel, then state kernel
])
def test_chunk_tensor_core_paths(mode, B, H, T, plan):
    """The bf16 d = 128 path runs fused (one cooperative kernel, hand-off through a ring), prep +
    fused, or as two kernels (hand-off through the workspace), by head count: each against the
    oracle."""
    got, c1 = gdr.chunk_fwd_plan(B, T, H, 128, 128, 64, mode, torch.bfloat16)
    assert got == plan and (c1 > 0) == (plan == "prep_fused")
    seed = 4000 + B * 100 + H + T + (1 if mode == "scalar" else 0)
    x = make_chunk_inputs(B, T, H, 128, 128, mode, "bf16", seed, s0_std=0.05)
    check_chunk(x, mode, "bf16", label=f"{mode}/B{B}/H{H}/T{T}/{plan}")


@pytest.mark.parametrize("B,H,T,plan", [
    (1, 1, 5000, "fused"),        # one head, 10 prep CTAs, 79 chunks through the 8-slot ring
    (1, 16, 64, "fused"),         # 16 heads, one chunk
    (1, 8, 1000, "fused"),        # 8 heads, ragged tail
    (2, 16, 700, "prep_fused"),   # 32 heads: 6 of 11 chunks prepared before the fused kernel
    (4, 16, 1000, "prep_fused"),  # 64 heads: 14 of 16 prepared before, 2 ring slots
    (13, 8, 130, "two_pass"),     # 104 heads
])
def test_chunk_tensor_core_paths_channel_gate(B, H, T, plan):
    """The channel gate's plans (one prep pipeline per fused CTA), with a within-chunk log2-decay
    spread of about 30 on a quarter of the channels (the exact CUDA-core terms) and alpha = 0 on
    four more, against the oracle."""
    got, c1 = gdr.chunk_fwd_plan(B, T, H, 128, 128, 64, "channel", torch.bfloat16)
    assert got == plan and (c1 > 0) == (plan == "prep_fused")
    x = make_chunk_inputs(B, T, H, 128, 128, "channel", "bf16", 4500 + B * 100 + H + T, s0_std=0.05)
    g = x["g"].clone()
    g[..., 96:128] = _g_for_spread(30.0)
    g[..., 40:44] = -1e4
    x["g"] = g
    check_chunk(x, "channel", "bf16", label=f"channel/B{B}/H{H}/T{T}/{plan}")


@pytest.mark.parametrize("mode", MODES)
def test_chunk_unequal_head_dims(mode):
    x = make_chunk_inputs(1, 130, 2, 128, 64, mode, "bf16", 77, s0_std=0.05)
    check_chunk(x, mode, "bf16")
    x = make_chunk_inputs(1, 130, 2, 64, 128, mode, "f32", 78, s0_std=0.05)
    check_chunk(x, mode, "f32")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dk,dv", [(64, 32), (32, 128)])
@pytest.mark.parametrize("T", [200, 300])
def test_chunk_cuda_core_unequal_head_dims(mode, dk, dv, T):
    """d_k != d_v in both directions on the fp32 CUDA-core path: T = 200 runs the token recurrence
    (a ragged last block of 16 tokens), T = 300 the chunk form (ragged last chunk), both with S0."""
    seed = 6000 + 10 * MODES.index(mode) + dk + dv + T
    x = make_chunk_inputs(1, T, 2, dk, dv, mode, "f32", seed, s0_std=0.1)
    check_chunk(x, mode, "f32", label=f"{mode}/dk{dk}/dv{dv}/T{T}")


def test_chunk_cuda_core_chunk_form_gdn_small_workload_shape():
    """The chunk form at the small Gated DeltaNet workload's shape (fp32, B = 1, H = 2, d = 64) with a
    sequence long enough to leave the token recurrence (T = 320, five chunks): the workload itself
    (T = 256) is served by the recurrence, so this keeps the fp32 chunk form covered at that shape."""
    x = make_chunk_inputs(1, 320, 2, 64, 64, "scalar", "f32", 6100)
    check_chunk(x, "scalar", "f32", label="gdn f32 B1 H2 d64 T320")


@pytest.mark.parametrize("name", list(CHUNK_WORKLOADS))
def test_chunk_full_workload(name):
    """Every named workload at full size, whole output against the oracle."""
    w = CHUNK_WORKLOADS[name]
    x = workload_inputs(w)
    eo, es = check_chunk(x, w.mode, w.dtype, label=name)
    print(f"{name}: max|do|/rms(o) = {eo:.3e}, max|dS|/rms(S) = {es:.3e}")


def test_state_carry_split_and_inplace():
    """fwd(T1) then fwd(T2, S0 = S_T(T1)) equals fwd(T1+T2); S_T may alias S0."""
    x = make_chunk_inputs(2, 300, 2, 128, 128, "scalar", "bf16", 91, s0_std=0.05)
    o_all, s_all = run_chunk(x, "scalar")
    d = to_dev(x)
    S = d["S0"].clone()
    outs = []
    for sl in (slice(0, 100), slice(100, 300)):
        part = {k: (None if v is None else v[:, sl].contiguous()) for k, v in d.items() if k != "S0"}
        o, _ = gdr.chunk_fwd(part["q"], part["k"], part["v"], part["g"], part["beta"], S, mode="scalar",
                             state_out=S)  # in place
        outs.append(o)
    gdr.sync_status()
    o_split = torch.cat(outs, dim=1).double().cpu().numpy()
    e1, _ = rel_err(o_split, o_all)
    e2, _ = rel_err(S.double().cpu().numpy(), s_all)
    assert e1 <= TOL["bf16"] and e2 <= TOL["bf16"], (e1, e2)


def test_alpha_zero_resets():
    """g = -1e4 (alpha underflows to 0): o_t = scale beta_t (k_t.q_t) v_t."""
    x = make_chunk_inputs(1, 150, 2, 128, 128, "scalar", "bf16", 92, s0_std=0.1)
    x["g"] = torch.full_like(x["g"], -1e4)
    check_chunk(x, "scalar", "bf16")


def test_scalar_decay_strength_mix():
    """Chunks whose cumulative in-chunk log2-decay stays within 120 units take the factored pairwise
    decays 2^Gamma_r * 2^-Gamma_i, stronger ones the exact 2^(Gamma_r - Gamma_i): both kinds of
    chunk (and one right at the limit) in one call, against the oracle."""
    x = make_chunk_inputs(2, 640, 4, 128, 128, "scalar", "bf16", 96, s0_std=0.05)
    g = x["g"].clone()
    g[:, 128:256] = -3.0   # about 277 log2 units across a chunk
    g[:, 384:448] = -1.3   # 64 * 1.3 * log2(e) = 120.0
    x["g"] = g
    check_chunk(x, "scalar", "bf16")


def test_channel_constant_equals_scalar():
    x = make_chunk_inputs(2, 192, 2, 128, 128, "scalar", "bf16", 93)
    o1, s1 = run_chunk(x, "scalar")
    xc = dict(x)
    xc["g"] = x["g"][..., None].expand(-1, -1, -1, 128).contiguous()
    o2, s2 = run_chunk(xc, "channel")
    assert rel_err(o2, o1)[0] <= TOL["bf16"]
    assert rel_err(s2, s1)[0] <= TOL["bf16"]


# log-decay per token that makes a channel's cumulative log2-decay spread by about `spread` over a
# full chunk of 64 tokens: 63 * |g| * log2(e)
def _g_for_spread(spread):
    return -spread / (63 * 1.4426950408889634)


def test_channel_gate_strong_decays_mixed():
    """Channel gate with a within-chunk log2-decay spread of about 5, 15, 21 and 40 on four groups of
    channels and alpha = 0 (g = -1e4) on a fifth, the rest at the workload's mild decay: channels
    beyond the factored operands' range take the exact CUDA-core terms, the others the tensor-core
    product; several chunks, a ragged tail and S0, against the oracle."""
    x = make_chunk_inputs(2, 300, 3, 128, 128, "channel", "bf16", 201, s0_std=0.05)
    g = x["g"].clone()
    for c0, spread in ((0, 5.0), (8, 15.0), (16, 21.0), (24, 40.0)):
        g[..., c0:c0 + 8] = _g_for_spread(spread)
    g[..., 40:44] = -1e4
    x["g"] = g
    check_chunk(x, "channel", "bf16", label="channel spreads 5/15/21/40 + alpha=0")


@pytest.mark.parametrize("gval", [-1.0, -1e4])
def test_channel_gate_every_channel_strong(gval):
    """Every key channel beyond the factored range (g = -1: a spread of about 91 log2 units per chunk;
    g = -1e4: alpha = 0, the state resets every token)."""
    x = make_chunk_inputs(1, 200, 2, 128, 128, "channel", "bf16", 202, s0_std=0.05)
    x["g"] = torch.full_like(x["g"], gval)
    check_chunk(x, "channel", "bf16", label=f"channel g={gval} everywhere")


def test_channel_gate_strong_decays_full_workload_shape():
    """The channel-gate workload's shape at a quarter of its length (B=4, H=16, T=2048, d=128) with
    strong decays on a quarter of the channels: the prep + fused plan at full width against the oracle."""
    x = make_chunk_inputs(4, 2048, 16, 128, 128, "channel", "bf16", 203)
    g = x["g"].clone()
    g[..., 96:128] = _g_for_spread(30.0)
    x["g"] = g
    check_chunk(x, "channel", "bf16", label="KDA B4 H16 T2048, 32 strong channels")


def test_zero_beta_output_is_decayed_initial_state():
    x = make_chunk_inputs(1, 128, 2, 128, 128, "channel", "bf16", 94, s0_std=0.1)
    x["beta"] = torch.zeros_like(x["beta"])
    check_chunk(x, "channel", "bf16")


@pytest.mark.parametrize("mode", MODES)
def test_bf16_output(mode):
    """bf16 output: each element within the computation bound plus its own bf16 rounding,
    |o - o_ref| <= 2e-2 rms(o_ref) + 2^-8 |o_ref|."""
    x = make_chunk_inputs(2, 333, 3, 128, 128, mode, "bf16", 99 + MODES.index(mode), s0_std=0.05)
    o, st = run_chunk(x, mode, out_dtype=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=x["S0"])
    rms = np.sqrt(np.mean(o_ref ** 2))
    excess = np.abs(o - o_ref) - (TOL["bf16"] * rms + BF16_HALF_ULP * np.abs(o_ref))
    assert excess.max() <= 0, excess.max()
    assert rel_err(st, s_ref)[0] <= TOL["bf16"]


def test_bf16_output_full_headline_workload():
    """The headline workload (Gated DeltaNet bf16, B = 8, H = 8, T = 4096) with o in the input dtype,
    as the bench times it: every element within the bar plus its own bf16 rounding."""
    name = "gdn_bf16_b8_h8_t4096_d128"
    w = CHUNK_WORKLOADS[name]
    x = workload_inputs(w)
    o, st = run_chunk(x, w.mode, out_dtype=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], w.mode, S0=x["S0"])
    rms = np.sqrt(np.mean(o_ref ** 2))
    excess = np.abs(o - o_ref) - (TOL["bf16"] * rms + BF16_HALF_ULP * np.abs(o_ref))
    assert excess.max() <= 0, excess.max()
    assert rel_err(st, s_ref)[0] <= TOL["bf16"]
    print(f"{name} bf16 o: max|do|/rms = {rel_err(o, o_ref)[0]:.3e}")


def test_no_state_output():
    x = make_chunk_inputs(1, 70, 1, 128, 128, "none", "bf16", 95)
    o, st = run_chunk(x, "none", want_state=False)
    o_ref, _ = oracle.recurrent(x["q"], x["k"], x["v"], None, x["beta"], "none")
    assert rel_err(o, o_ref)[0] <= TOL["bf16"]


def test_host_tensors_roundtrip():
    """chunk_fwd on host tensors stages through the device and returns host tensors."""
    x = make_chunk_inputs(1, 100, 2, 128, 128, "scalar", "bf16", 96)
    o, st = gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, mode="scalar")
    torch.cuda.synchronize()
    assert o.device.type == "cpu" and st.device.type == "cpu"
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], "scalar")
    assert rel_err(o.double().numpy(), o_ref)[0] <= TOL["bf16"]
    assert rel_err(st.double().numpy(), s_ref)[0] <= TOL["bf16"]


@pytest.mark.parametrize("B,T,H,d,mode,dtype,with_s0", [
    (5, 130, 2, 128, "scalar", "bf16", True),    # 5 pieces of one sequence, tensor cores
    (11, 70, 2, 128, "channel", "bf16", False),  # pieces of 2, the last one of 1
    (3, 90, 3, 64, "none", "f32", True),         # CUDA-core path
])
def test_host_tensors_in_pieces(B, T, H, d, mode, dtype, with_s0):
    """gdr_chunk_fwd_host: page-locked host inputs, copies overlapped with the pieces' work; every
    piece against the oracle, with S0 carried in and S_T copied back."""
    x = make_chunk_inputs(B, T, H, d, d, mode, dtype, 500 + B + T, s0_std=0.1 if with_s0 else None)
    h = {kk: (None if t is None else t.contiguous().pin_memory()) for kk, t in x.items()}
    o, st = gdr.chunk_fwd(h["q"], h["k"], h["v"], h["g"], h["beta"], h["S0"], mode=mode)
    torch.cuda.synchronize()
    gdr.sync_status()
    o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=x["S0"])
    assert rel_err(o.double().numpy(), o_ref)[0] <= TOL[dtype]
    assert rel_err(st.double().numpy(), s_ref)[0] <= TOL[dtype]


# ------------------------------------------------------------- decode -----
def run_decode_steps(w_B, w_H, dk, dv, mode, dtype, steps, seed, s_std=0.02, out_dtype=torch.float32):
    from gated_delta_rule_143_b200.inputs import DecodeWorkload
    w = DecodeWorkload("t", mode, dtype, w_B, w_H, dk, dv, steps, s_std)
    S0 = make_decode_state(w, seed)
    S_dev = S0.cuda()
    S_ref = S0.double().numpy()
    worst = 0.0
    for st in range(steps):
        x = make_decode_step(w, seed, st)
        d = to_dev(x)
        o, obuf = guarded_empty((w_B, w_H, dv), out_dtype, "cuda")
        gdr.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S_dev, mode=mode, out=o)
        gdr.sync_status()
        assert guard_ok(obuf, o.numel())
        o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref, mode)
        og = o.double().cpu().numpy()
        e, rms = rel_err(og, o_ref)
        worst = max(worst, e)
        if out_dtype == torch.bfloat16:
            assert (np.abs(og - o_ref) - TOL[dtype] * rms - BF16_HALF_ULP * np.abs(o_ref)).max() <= 0
        else:
            assert e <= TOL[dtype], f"step {st}: o err {e:.3e}"
    es, _ = rel_err(S_dev.double().cpu().numpy(), S_ref)
    assert es <= TOL[dtype], f"final state err {es:.3e}"
    return worst, es


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (32, 40), (256, 96)])
def test_decode_small(mode, dtype, dk, dv):
    run_decode_steps(3, 5, dk, dv, mode, dtype, 6, 300 + dk + dv)


def test_decode_bf16_output():
    run_decode_steps(4, 8, 128, 128, "scalar", "bf16", 4, 555, out_dtype=torch.bfloat16)


def test_decode_full_workload():
    """The full decode workload: 256 steps at B=256, H=16 from random fp32 states; o checked at
    every step and the final states at the end."""
    w = DECODE_WORKLOADS["gdn_decode_bf16_b256_h16_d128"]
    worst, es = run_decode_steps(w.B, w.H, w.dk, w.dv, w.mode, w.dtype, w.steps, WORKLOAD_SEEDS[w.name], w.s_std)
    print(f"decode: worst per-step max|do|/rms = {worst:.3e}, final state {es:.3e}")


def test_decode_steps_equal_chunked_forward():
    """T decode steps from S0 reproduce the chunked forward over the same T tokens."""
    x = make_chunk_inputs(2, 40, 2, 128, 128, "channel", "bf16", 97, s0_std=0.05)
    o_fwd, s_fwd = run_chunk(x, "channel")
    d = to_dev(x)
    S = d["S0"].clone()
    outs = []
    for t in range(40):
        outs.append(gdr.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                    d["g"][:, t].contiguous(), d["beta"][:, t].contiguous(), S, mode="channel"))
    gdr.sync_status()
    o_dec = torch.stack(outs, dim=1).double().cpu().numpy()
    assert rel_err(o_dec, o_fwd)[0] <= TOL["bf16"]
    assert rel_err(S.double().cpu().numpy(), s_fwd)[0] <= TOL["bf16"]


# ------------------------------------------------------------- errors -----
def test_device_errors_are_codes_not_faults():
    x = to_dev(make_chunk_inputs(1, 64, 1, 128, 128, "scalar", "bf16", 98))
    with pytest.raises(gdr.GdrError) as e:  # misaligned view of a real buffer
        q2 = torch.empty(x["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + x["q"].numel()]
        gdr.chunk_fwd(q2.view_as(x["q"]), x["k"], x["v"], x["g"], x["beta"], None, mode="scalar")
    assert e.value.code == -3
    with pytest.raises(gdr.GdrError) as e:
        gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, mode="scalar", chunk=48)
    assert e.value.code == -2
    gdr.sync_status()


def test_host_tensors_two_threads():
    """gdr_chunk_fwd_host from two host threads at once, each with its own stream and staging: the
    calls share the device's copy streams and events (serialised while enqueueing); every result
    matches the oracle."""
    import threading

    cases = [make_chunk_inputs(3, 150, 2, 128, 128, "scalar", "bf16", 700 + i, s0_std=0.05) for i in range(2)]
    pinned = [{kk: (None if t is None else t.contiguous().pin_memory()) for kk, t in x.items()} for x in cases]
    results, errors = [None, None], []
    dev = torch.cuda.current_device()

    def worker(i):
        try:
            torch.cuda.set_device(dev)
            s = torch.cuda.Stream()
            outs = []
            with torch.cuda.stream(s):
                for _ in range(3):
                    h = pinned[i]
                    outs.append(gdr.chunk_fwd(h["q"], h["k"], h["v"], h["g"], h["beta"], h["S0"], mode="scalar"))
            s.synchronize()
            results[i] = outs
        except Exception as e:  # reported on the main thread
            errors.append(e)

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    gdr.sync_status()
    for i, x in enumerate(cases):
        o_ref, s_ref = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], "scalar", S0=x["S0"])
        for o, st in results[i]:
            assert rel_err(o.double().numpy(), o_ref)[0] <= TOL["bf16"]
            assert rel_err(st.double().numpy(), s_ref)[0] <= TOL["bf16"]
