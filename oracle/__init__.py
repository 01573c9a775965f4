"""fp64 CPU oracle for the gated delta-rule recurrence -- TEST INFRASTRUCTURE.

Only the test-suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package. It shares no code with the CUDA library and never
imports it; the product path never imports this.

The arithmetic lives in ``gdr_oracle.c`` (plain token-by-token recurrence in
float64, see its header for the sources it follows). This module compiles it
with gcc on first use, loads it with ctypes and marshals numpy / torch CPU
arrays. Parity of every function here is pinned by ``tests/test_oracle.py``
against closed forms, brute-force transition products, exact-recall and
limiting cases; no function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_MODES = {"none": 0, "scalar": 1, "channel": 2}
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile ``gdr_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, -O2, IEEE fp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.gdr_oracle_recurrent.restype = ctypes.c_int
            lib.gdr_oracle_recurrent.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + [
                ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            lib.gdr_oracle_max_threads.restype = ctypes.c_int
            lib.gdr_oracle_recurrent_gdn2.restype = ctypes.c_int
            lib.gdr_oracle_recurrent_gdn2.argtypes = lib.gdr_oracle_recurrent.argtypes
            lib.gdr_oracle_backward.restype = ctypes.c_int
            lib.gdr_oracle_backward.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 4 + [
                ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_double] + [
                ctypes.c_void_p] * 8 + [ctypes.c_int]
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().gdr_oracle_max_threads())


def _arr(x, f64: bool) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU); bf16 widens exactly to fp32
        x = x.detach().to("cpu").float().numpy() if not f64 else x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x), dtype=np.float64 if f64 else np.float32)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def recurrent(q, k, v, g, beta, mode: str, S0=None, *, erase=None, write=None,
              scale: Optional[float] = None, f64_inputs: bool = False,
              threads: int = 0, want_state: bool = True) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """Token-by-token recurrence over q, k [B,T,H,dk], v [B,T,H,dv].

    ``g`` is the log-decay ([B,T,H] for "scalar", [B,T,H,dk] for "channel",
    ignored for "none"); ``beta`` [B,T,H]. ``erase``/``write`` override the
    erase and write coefficients (both default to ``beta``). ``scale``
    defaults to 1/sqrt(dk). Inputs are read as float32 (exact for bf16 and
    fp32 data) unless ``f64_inputs``. Returns ``(o [B,T,H,dv], S_T [B,H,dv,dk])``
    in float64.
    """
    lib = _load()
    if mode not in _MODES:
        raise ValueError(f"unknown decay mode {mode!r}")
    qa, ka, va = _arr(q, f64_inputs), _arr(k, f64_inputs), _arr(v, f64_inputs)
    B, T, H, dk = qa.shape
    dv = va.shape[-1]
    if ka.shape != (B, T, H, dk) or va.shape != (B, T, H, dv):
        raise ValueError("q, k, v shapes disagree")
    ba = _arr(beta, f64_inputs)
    ea = ba if erase is None else _arr(erase, f64_inputs)
    wa = ba if write is None else _arr(write, f64_inputs)
    for name, a in (("erase", ea), ("write", wa)):
        if a.shape != (B, T, H):
            raise ValueError(f"{name} must be [B,T,H]")
    ga = None
    if mode != "none":
        ga = _arr(g, f64_inputs)
        want = (B, T, H) if mode == "scalar" else (B, T, H, dk)
        if ga.shape != want:
            raise ValueError(f"g must be {want} for mode {mode}")
    s0 = None
    if S0 is not None:
        s0 = _arr(S0, True)
        if s0.shape != (B, H, dv, dk):
            raise ValueError("S0 must be [B,H,dv,dk]")
    o = np.empty((B, T, H, dv), dtype=np.float64)
    st = np.empty((B, H, dv, dk), dtype=np.float64) if want_state else None
    sc = (1.0 / np.sqrt(dk)) if scale is None else float(scale)
    rc = lib.gdr_oracle_recurrent(B, T, H, dk, dv, _ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _MODES[mode],
                                  _ptr(ea), _ptr(wa), int(bool(f64_inputs)), _ptr(s0), sc,
                                  _ptr(o), _ptr(st), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle failed with status {rc}")
    return o, st


def recurrent_gdn2(q, k, v, g, erase, write, mode: str, S0=None, *, scale: Optional[float] = None,
                   f64_inputs: bool = False, threads: int = 0,
                   want_state: bool = True) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """Gated DeltaNet-2 token recurrence (``gdr_oracle_recurrent_gdn2``): channel-wise erase gate
    ``erase`` [B,T,H,dk] on the key side and write gate ``write`` [B,T,H,dv] on the value side,
    decay g as in ``recurrent``. Returns ``(o, S_T)`` in float64."""
    lib = _load()
    if mode not in _MODES:
        raise ValueError(f"unknown decay mode {mode!r}")
    qa, ka, va = _arr(q, f64_inputs), _arr(k, f64_inputs), _arr(v, f64_inputs)
    B, T, H, dk = qa.shape
    dv = va.shape[-1]
    if ka.shape != (B, T, H, dk) or va.shape != (B, T, H, dv):
        raise ValueError("q, k, v shapes disagree")
    ea, wa = _arr(erase, f64_inputs), _arr(write, f64_inputs)
    if ea.shape != (B, T, H, dk) or wa.shape != (B, T, H, dv):
        raise ValueError("erase must be [B,T,H,dk] and write [B,T,H,dv]")
    ga = None
    if mode != "none":
        ga = _arr(g, f64_inputs)
        want = (B, T, H) if mode == "scalar" else (B, T, H, dk)
        if ga.shape != want:
            raise ValueError(f"g must be {want} for mode {mode}")
    s0 = None if S0 is None else _arr(S0, True)
    if s0 is not None and s0.shape != (B, H, dv, dk):
        raise ValueError("S0 must be [B,H,dv,dk]")
    o = np.empty((B, T, H, dv), dtype=np.float64)
    st = np.empty((B, H, dv, dk), dtype=np.float64) if want_state else None
    sc = (1.0 / np.sqrt(dk)) if scale is None else float(scale)
    rc = lib.gdr_oracle_recurrent_gdn2(B, T, H, dk, dv, _ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _MODES[mode],
                                       _ptr(ea), _ptr(wa), int(bool(f64_inputs)), _ptr(s0), sc, _ptr(o), _ptr(st),
                                       int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle failed with status {rc}")
    return o, st


def backward(q, k, v, g, beta, mode: str, dO, S0=None, dS_T=None, *, scale: Optional[float] = None,
             f64_inputs: bool = False, threads: int = 0):
    """Gradients of the mixer recurrence (``recurrent`` with erase = write = beta) for a loss
    whose gradients with respect to o [B,T,H,dv] and S_T [B,H,dv,dk] are ``dO`` and ``dS_T``
    (None: zero). Reverse-mode differentiation of the token recurrence in float64 (see
    ``gdr_oracle_backward`` in ``gdr_oracle.c``). Returns a dict of float64 arrays: ``dq``, ``dk``
    [B,T,H,dk], ``dv`` [B,T,H,dv], ``dbeta`` [B,T,H], ``dg`` (shape of g; None for "none") and
    ``dS0`` [B,H,dv,dk]."""
    lib = _load()
    if mode not in _MODES:
        raise ValueError(f"unknown decay mode {mode!r}")
    qa, ka, va = _arr(q, f64_inputs), _arr(k, f64_inputs), _arr(v, f64_inputs)
    B, T, H, dk = qa.shape
    dv = va.shape[-1]
    if ka.shape != (B, T, H, dk) or va.shape != (B, T, H, dv):
        raise ValueError("q, k, v shapes disagree")
    ba = _arr(beta, f64_inputs)
    if ba.shape != (B, T, H):
        raise ValueError("beta must be [B,T,H]")
    ga = None
    if mode != "none":
        ga = _arr(g, f64_inputs)
        want = (B, T, H) if mode == "scalar" else (B, T, H, dk)
        if ga.shape != want:
            raise ValueError(f"g must be {want} for mode {mode}")
    s0 = None if S0 is None else _arr(S0, True)
    do = _arr(dO, True)
    if do.shape != (B, T, H, dv):
        raise ValueError("dO must be [B,T,H,dv]")
    dst = None if dS_T is None else _arr(dS_T, True)
    for name, a in (("S0", s0), ("dS_T", dst)):
        if a is not None and a.shape != (B, H, dv, dk):
            raise ValueError(f"{name} must be [B,H,dv,dk]")
    out = {"dq": np.empty((B, T, H, dk)), "dk": np.empty((B, T, H, dk)), "dv": np.empty((B, T, H, dv)),
           "dbeta": np.empty((B, T, H)), "dg": None if ga is None else np.empty(ga.shape),
           "dS0": np.empty((B, H, dv, dk))}
    sc = (1.0 / np.sqrt(dk)) if scale is None else float(scale)
    rc = lib.gdr_oracle_backward(B, T, H, dk, dv, _ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _MODES[mode], _ptr(ba),
                                 int(bool(f64_inputs)), _ptr(s0), sc, _ptr(do), _ptr(dst), _ptr(out["dq"]),
                                 _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                                 _ptr(out["dS0"]), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle backward failed with status {rc}")
    return out


def decode_step(q, k, v, g, beta, S, mode: str, *, scale: Optional[float] = None,
                f64_inputs: bool = False, threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """One recurrent step for a batch of states: q, k [B,H,dk], v [B,H,dv],
    beta [B,H], g [B,H] / [B,H,dk] / None, S [B,H,dv,dk]. It is the same
    recurrence with T = 1. Returns ``(o [B,H,dv], S_new [B,H,dv,dk])`` (fp64)."""
    def tok(x):
        if x is None:
            return None
        a = _arr(x, f64_inputs)
        return a.reshape((a.shape[0], 1) + a.shape[1:])
    o, st = recurrent(tok(q), tok(k), tok(v), tok(g), tok(beta), mode, S0=S, scale=scale,
                      f64_inputs=f64_inputs, threads=threads)
    return o[:, 0], st


def _sigmoid(x: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + e^-x) in float64, evaluated on the side where the
    exponential cannot overflow (e^x / (1 + e^x) for negative x)."""
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def _softplus(x: np.ndarray) -> np.ndarray:
    """softplus(x) = log(1 + e^x) in float64, written as max(x, 0) + log1p(e^-|x|)."""
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def prologue(q, k, beta, g, mode: str, *, l2norm_qk: bool = False, beta_sigmoid: bool = False,
             gate_softplus: bool = False, gate_scale=None):
    """The mixer layer's steps in front of the recurrence, in float64.

    Follows the pages' recurrent reference form ("Linear Attention & DeltaNet",
    minimal pseudocode): q and k pass through a feature map, the write strength is
    beta = sigmoid(logit) and the decay gate is a squashed logit. The three steps, each
    applied only when its flag is set, are:

    - ``l2norm_qk``: every (b, t, h) vector of q and of k is divided by its Euclidean
      norm (no epsilon; an all-zero vector stays zero).
    - ``beta_sigmoid``: ``beta`` holds logits; the write strength is their sigmoid.
    - ``gate_softplus``: ``g`` holds gate logits a ([B,T,H] or [B,T,H,dk]); the
      log-decay is g = -A_h * softplus(a) with A = ``gate_scale`` [H] (1 if None).
      With A_h = 0.05 this is the decay exp(-0.05 softplus(.)) of the small
      Gated DeltaNet workload; with A_h = 1 and a = -x it is alpha = sigmoid(x), the
      pseudocode's gate, since log sigmoid(x) = -softplus(-x).

    Inputs are read as float32 (exact for bf16 / fp32 data). Returns float64
    ``(q, k, beta, g)`` to hand to ``recurrent(..., f64_inputs=True)``; arguments
    whose step is off come back unchanged (widened).
    """
    # widen through float32, as the library reads them
    qa, ka = _arr(_arr(q, False), True), _arr(_arr(k, False), True)
    ba = _arr(_arr(beta, False), True)
    ga = None if g is None else _arr(_arr(g, False), True)
    if l2norm_qk:
        out = []
        for a in (qa, ka):
            n = np.sqrt(np.sum(a * a, axis=-1, keepdims=True))
            out.append(np.divide(a, n, out=np.zeros_like(a), where=n > 0))
        qa, ka = out
    if beta_sigmoid:
        ba = _sigmoid(ba)
    if gate_softplus:
        if mode == "none" or ga is None:
            raise ValueError("gate_softplus needs a decay mode and gate logits")
        H = ba.shape[2]
        A = np.ones(H) if gate_scale is None else _arr(_arr(gate_scale, False), True).reshape(H)
        Ab = A.reshape((1, 1, H)) if mode == "scalar" else A.reshape((1, 1, H, 1))
        ga = -Ab * _softplus(ga)
    return qa, ka, ba, ga
