"""Gated delta-rule mixer for NVIDIA B200 (sm_100a): Python binding of libgdr.so.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels; PyTorch provides device memory and streams. The two operations:

* ``chunk_fwd``   -- chunkwise-parallel forward over whole sequences (prefill /
  training form) for DeltaNet (mode "none"), Gated DeltaNet ("scalar") and
  Kimi Delta Attention ("channel");
* ``decode_step`` -- one recurrent token step on a batch of fp32 states, in place.

Both can apply the mixer layer's input steps inside their kernels (keyword
arguments ``l2norm_qk``, ``beta_sigmoid``, ``gate_softplus`` / ``gate_scale``):
q and k then hold raw vectors, ``beta`` logits and ``g`` gate logits.

Both take device tensors. ``chunk_fwd`` also accepts host (CPU) tensors: it
then copies them to the current device on the current stream, runs, and copies
the outputs back (the end-to-end path a host-resident caller uses).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import (DECAY_MODES, DTYPE_BF16, DTYPE_F32, PLANS, PRO_BETA_SIGMOID, PRO_GATE_SOFTPLUS, PRO_L2NORM_QK,
                   GdrError, check, lib)

__all__ = ["chunk_fwd", "chunk_bwd", "chunk_fwd_gdn2", "chunk_fwd_scan", "decode_step", "decode_step_gdn2", "sync_status", "workspace_bytes", "launches_per_chunk_fwd", "chunk_fwd_plan",
           "profile_next_call",
           "GdrError", "DECAY_MODES"]


def _mode(mode) -> int:
    if isinstance(mode, str):
        if mode not in DECAY_MODES:
            raise ValueError(f"unknown decay mode {mode!r}")
        return DECAY_MODES[mode]
    return int(mode)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return DTYPE_BF16
    if dt == torch.float32:
        return DTYPE_F32
    raise TypeError(f"tensors must be bfloat16 or float32, got {dt}")


def _dtype(t: torch.Tensor) -> int:
    return _dtype_code(t.dtype)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _prologue(l2norm_qk: bool, beta_sigmoid: bool, gate_softplus: bool) -> int:
    return ((PRO_L2NORM_QK if l2norm_qk else 0) | (PRO_BETA_SIGMOID if beta_sigmoid else 0)
            | (PRO_GATE_SOFTPLUS if gate_softplus else 0))


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def workspace_bytes(B: int, T: int, H: int, dk: int, dv: int, chunk: int, mode, dtype: torch.dtype,
                    out_dtype: torch.dtype = torch.float32) -> int:
    """Device scratch ``chunk_fwd`` needs for this problem (bytes)."""
    return int(lib().gdr_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, _mode(mode), _dtype_code(dtype),
                                                   _dtype_code(out_dtype)))


def launches_per_chunk_fwd(B: int, T: int, H: int, dk: int, dv: int, chunk: int, mode, dtype: torch.dtype,
                           out_dtype: torch.dtype = torch.float32) -> int:
    """Kernel launches one ``chunk_fwd`` makes for this problem (as the library reports)."""
    return int(lib().gdr_chunk_fwd_launches(B, T, H, dk, dv, chunk, _mode(mode), _dtype_code(dtype),
                                            _dtype_code(out_dtype)))


def chunk_fwd_plan(B: int, T: int, H: int, dk: int, dv: int, chunk: int, mode, dtype: torch.dtype,
                   out_dtype: torch.dtype = torch.float32) -> Tuple[str, int]:
    """How ``chunk_fwd`` runs this problem: ("cuda_core" | "two_pass" | "fused" | "prep_fused" |
    "invalid", chunks per head prepared before the fused kernel)."""
    import ctypes
    c1 = ctypes.c_int(0)
    code = lib().gdr_chunk_fwd_plan(B, T, H, dk, dv, chunk, _mode(mode), _dtype_code(dtype), _dtype_code(out_dtype),
                                    ctypes.byref(c1))
    return PLANS[int(code)], int(c1.value)


_ws_cache = {}


def _workspace(nbytes: int, device: torch.device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor],
              beta: torch.Tensor, S0: Optional[torch.Tensor] = None, *, mode="scalar", chunk: int = 64,
              return_state: bool = True, out: Optional[torch.Tensor] = None,
              out_dtype: torch.dtype = torch.float32,
              state_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None, l2norm_qk: bool = False, beta_sigmoid: bool = False,
              gate_softplus: bool = False,
              gate_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked forward. q, k [B,T,H,dk]; v [B,T,H,dv] (bf16 or fp32, same dtype);
    g fp32 [B,T,H] ("scalar") / [B,T,H,dk] ("channel") / None ("none"); beta fp32
    [B,T,H]; S0 fp32 [B,H,dv,dk] or None. Returns (o [B,T,H,dv], S_T or None).
    o is fp32 by default (``out_dtype``, or the dtype of ``out``; bf16 allowed for bf16
    inputs). ``state_out`` may be ``S0`` itself (in-place carry).
    Prologue (device tensors only, gdr_chunk_fwd_ex): ``l2norm_qk`` divides every q and k
    vector by its norm, ``beta_sigmoid`` reads ``beta`` as logits, ``gate_softplus`` reads
    ``g`` as gate logits a with g = -gate_scale[h] * softplus(a) (``gate_scale`` fp32 [H] or None = 1)."""
    pro = _prologue(l2norm_qk, beta_sigmoid, gate_softplus)
    if q.device.type == "cpu":
        if pro:
            raise ValueError("the fused prologue takes device tensors")
        return _chunk_fwd_host(q, k, v, g, beta, S0, mode=mode, chunk=chunk, return_state=return_state,
                               out=out, out_dtype=out_dtype, state_out=state_out, stream=stream)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype(q)
    m = _mode(mode)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, device=q.device)
    odt = _dtype(out)
    if return_state and state_out is None:
        state_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(lib().gdr_chunk_fwd_workspace_bytes(B, T, H, dk, dv, chunk, m, dt, odt), q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if pro:
        rc = lib().gdr_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out),
                                    _ptr(state_out) if return_state else None, B, T, H, dk, dv, chunk, m, dt, odt,
                                    pro, _ptr(gate_scale), _ptr(workspace), ws_bytes, _stream_handle(stream))
    else:
        rc = lib().gdr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out),
                                 _ptr(state_out) if return_state else None, B, T, H, dk, dv, chunk, m, dt, odt,
                                 _ptr(workspace), ws_bytes, _stream_handle(stream))
    check(rc)
    return out, (state_out if return_state else None)


def _chunk_fwd_host(q, k, v, g, beta, S0, *, mode, chunk, return_state, out, out_dtype, state_out, stream):
    """Host-resident tensors: gdr_chunk_fwd_host copies them in, computes and copies the outputs
    back piece by piece, the copies overlapping the work (device staging from a per-stream cache;
    outputs in page-locked memory unless given)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype(q)
    m = _mode(mode)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, pin_memory=True)
    odt = _dtype(out)
    if return_state and state_out is None:
        state_out = torch.empty((B, H, dv, dk), dtype=torch.float32, pin_memory=True)
    for t in (q, k, v, g, beta, S0, out, state_out):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError("host path: every tensor must be a contiguous CPU tensor")
    nbytes = int(lib().gdr_chunk_fwd_host_staging_bytes(B, T, H, dk, dv, chunk, m, dt, odt))
    key = ("staging", dev.index, s.cuda_stream)
    staging = _ws_cache.get(key)
    if staging is None or staging.numel() < nbytes:
        staging = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _ws_cache[key] = staging
    rc = lib().gdr_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out),
                                  _ptr(state_out) if return_state else None, B, T, H, dk, dv, chunk, m, dt, odt,
                                  _ptr(staging), staging.numel(), s.cuda_stream)
    check(rc)
    return out, (state_out if return_state else None)


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor],
                beta: torch.Tensor, S: torch.Tensor, *, mode="scalar", out: Optional[torch.Tensor] = None,
                out_dtype: torch.dtype = torch.float32,
                stream: Optional[torch.cuda.Stream] = None, l2norm_qk: bool = False, beta_sigmoid: bool = False,
                gate_softplus: bool = False, gate_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One recurrent step: q, k [B,H,dk], v [B,H,dv], g [B,H] / [B,H,dk] / None,
    beta [B,H], S fp32 [B,H,dv,dk] updated in place. Returns o [B,H,dv] (fp32 by default).
    The prologue keywords are those of ``chunk_fwd`` (gdr_decode_step_ex)."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype, device=q.device)
    pro = _prologue(l2norm_qk, beta_sigmoid, gate_softplus)
    if pro:
        rc = lib().gdr_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(out), B, H, dk,
                                      dv, _mode(mode), _dtype(q), _dtype(out), pro, _ptr(gate_scale),
                                      _stream_handle(stream))
    else:
        rc = lib().gdr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(out), B, H, dk,
                                   dv, _mode(mode), _dtype(q), _dtype(out), _stream_handle(stream))
    check(rc)
    return out


def chunk_fwd_scan(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor],
                   beta: torch.Tensor, S0: Optional[torch.Tensor] = None, *, n_seg: int, mode="scalar",
                   chunk: int = 64, return_state: bool = True, out: Optional[torch.Tensor] = None,
                   out_dtype: torch.dtype = torch.float32, state_out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``chunk_fwd`` with every sequence split into ``n_seg`` segments run in parallel
    (gdr_chunk_fwd_scan); bf16 q/k/v with d_k = d_v = 128 and T a multiple of 64 * n_seg."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    m = _mode(mode)
    dt = _dtype(q)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, device=q.device)
    odt = _dtype(out)
    if return_state and state_out is None:
        state_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(lib().gdr_chunk_fwd_scan_workspace_bytes(B, T, H, dk, dv, chunk, m, dt, odt, n_seg),
                               q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().gdr_chunk_fwd_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out),
                                  _ptr(state_out) if return_state else None, B, T, H, dk, dv, chunk, m, dt, odt, n_seg,
                                  _ptr(workspace), ws_bytes, _stream_handle(stream))
    check(rc)
    return out, (state_out if return_state else None)


def chunk_fwd_gdn2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor],
                   erase: torch.Tensor, write: torch.Tensor, S0: Optional[torch.Tensor] = None, *, mode="channel",
                   chunk: int = 64, return_state: bool = True, out: Optional[torch.Tensor] = None,
                   out_dtype: torch.dtype = torch.float32, state_out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated DeltaNet-2 forward (gdr_chunk_fwd_gdn2): ``erase`` fp32 [B,T,H,dk] and ``write`` fp32
    [B,T,H,dv] gates in place of beta; other arguments as ``chunk_fwd``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, device=q.device)
    if return_state and state_out is None:
        state_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device)
    m, dt, odt = _mode(mode), _dtype(q), _dtype(out)
    if workspace is None:
        workspace = _workspace(lib().gdr_chunk_fwd_gdn2_workspace_bytes(B, T, H, dk, dv, chunk, m, dt, odt), q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().gdr_chunk_fwd_gdn2(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(erase), _ptr(write), _ptr(S0), _ptr(out),
                                  _ptr(state_out) if return_state else None, B, T, H, dk, dv, chunk, m, dt, odt,
                                  _ptr(workspace), ws_bytes, _stream_handle(stream))
    check(rc)
    return out, (state_out if return_state else None)


def decode_step_gdn2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor],
                     erase: torch.Tensor, write: torch.Tensor, S: torch.Tensor, *, mode="channel",
                     out: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.float32,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One Gated DeltaNet-2 decode step (gdr_decode_step_gdn2): erase [B,H,dk], write [B,H,dv] fp32;
    S updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=out_dtype, device=q.device)
    rc = lib().gdr_decode_step_gdn2(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(erase), _ptr(write), _ptr(S), _ptr(out),
                                    B, H, dk, dv, _mode(mode), _dtype(q), _dtype(out), _stream_handle(stream))
    check(rc)
    return out


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor], beta: torch.Tensor,
              dO: torch.Tensor, S0: Optional[torch.Tensor] = None, dS_T: Optional[torch.Tensor] = None, *,
              mode="scalar", want_dS0: bool = True, workspace: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of ``chunk_fwd`` (gdr_chunk_bwd) for upstream gradients dO [B,T,H,dv] (the dtype of
    q) and dS_T [B,H,dv,dk] fp32 (None: zero). Returns fp32 device tensors ``dq``, ``dk`` [B,T,H,dk],
    ``dv`` [B,T,H,dv], ``dbeta`` [B,T,H], ``dg`` (shape of g, None for "none"), ``dS0`` (or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    m = _mode(mode)
    dt = _dtype(q)
    f32 = dict(dtype=torch.float32, device=q.device)
    out = {"dq": torch.empty((B, T, H, dk), **f32), "dk": torch.empty((B, T, H, dk), **f32),
           "dv": torch.empty((B, T, H, dv), **f32), "dbeta": torch.empty((B, T, H), **f32),
           "dg": None if g is None or m == 0 else torch.empty(g.shape, **f32),
           "dS0": torch.empty((B, H, dv, dk), **f32) if want_dS0 else None}
    if workspace is None:
        workspace = _workspace(lib().gdr_chunk_bwd_workspace_bytes(B, T, H, dk, dv, m, dt), q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().gdr_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dS_T),
                             _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                             _ptr(out["dS0"]), B, T, H, dk, dv, m, dt, _ptr(workspace), ws_bytes,
                             _stream_handle(stream))
    check(rc)
    return out


def sync_status(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Wait for the stream and raise if a kernel recorded a device-side error."""
    check(lib().gdr_sync_status(_stream_handle(stream)))


def profile_next_call(events) -> None:
    """Per-kernel timing: the next ``chunk_fwd`` on this thread records ``events[i]`` (created
    ``torch.cuda.Event`` objects) right after enqueuing its i-th kernel, on its stream."""
    import ctypes
    handles = [int(e.cuda_event) for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each event once before passing it (torch creates events lazily)")
    arr = (ctypes.c_void_p * max(len(handles), 1))(*handles)
    check(lib().gdr_profile_next_call(arr, len(handles)))
