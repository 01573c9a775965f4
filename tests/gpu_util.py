"""Helpers for the GPU parity tests: device staging with NaN-filled, guarded
outputs, and the tolerance rule (max |GPU - oracle| <= tol * rms(oracle),
tol = 1e-4 for fp32 inputs and 2e-2 for bf16 inputs, fp32 accumulation and
fp32 state)."""
import numpy as np
import torch

import gated_delta_rule_143_b200 as gdr

TOL = {"f32": 1e-4, "bf16": 2e-2}
BF16_HALF_ULP = 2.0 ** -8  # relative rounding bound of a bf16 output element
GUARD = 4096  # elements of canary after each output


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.abs(got - ref).max()) / max(rms, 1e-30), rms


def guarded_empty(shape, dtype, device):
    """A NaN-filled tensor followed by a canary region (to catch unwritten
    elements and writes past the end)."""
    n = int(np.prod(shape))
    buf = torch.full((n + GUARD,), float("nan"), dtype=dtype, device=device)
    buf[n:] = 12345.0
    return buf[:n].view(shape), buf


def guard_ok(buf, n):
    return bool(torch.all(buf[n:] == 12345.0).item())


def to_dev(x):
    return {k: (None if t is None else t.cuda()) for k, t in x.items()}


def run_chunk(x, mode, chunk=64, S0=None, want_state=True, out_dtype=torch.float32):
    """Run the CUDA chunked forward through the C ABI; returns (o, S_T) as CPU float64 numpy."""
    d = to_dev(x)
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o, obuf = guarded_empty((B, T, H, dv), out_dtype, "cuda")
    st, sbuf = guarded_empty((B, H, dv, dk), torch.float32, "cuda")
    s0 = d["S0"] if S0 is None else S0.cuda()
    gdr.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], s0, mode=mode, chunk=chunk, out=o,
                  state_out=st if want_state else None, return_state=want_state)
    gdr.sync_status()
    assert guard_ok(obuf, o.numel()), "write past the end of o"
    assert guard_ok(sbuf, st.numel()), "write past the end of S_T"
    return o.double().cpu().numpy(), (st.double().cpu().numpy() if want_state else None)
