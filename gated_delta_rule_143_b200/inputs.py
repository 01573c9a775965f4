"""Seeded synthetic inputs for the gated delta-rule mixer.

This module serves both the CUDA path (tests, bench) and the CPU oracle. It
holds none of the recurrence's arithmetic: only random draws, the input recipe
and dtype casts.

Input recipe (the pages train 350M-3B models; no dataset is used here, these
synthetic tensors stand in for a layer's projected activations):

* q, k ~ N(0, 1), each (b, t, h) vector L2-normalised in fp32 *before* any
  bf16 cast (no epsilon, no re-normalisation after rounding);
* v ~ N(0, 1);
* beta = sigmoid(N(0, 1)) in fp32, shape [B, T, H];
* log-decay g = -0.05 * softplus(N(0, 1)) in fp32, shape [B, T, H] for the
  scalar gate (Gated DeltaNet), [B, T, H, d_k] for the channel gate (Kimi
  Delta Attention), absent for DeltaNet (alpha = 1);
* optional initial state S0 ~ N(0, s0_std) fp32, shape [B, H, d_v, d_k].

Draw order from one ``torch.Generator`` seeded with ``seed``: q, k, v,
beta-logit, g-logit, S0. Decode steps draw their per-step tokens from a
generator seeded by ``(seed, step)`` so any single step can be regenerated.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch
import torch.nn.functional as F

DECAY_MODES = ("none", "scalar", "channel")
DTYPES = ("f32", "bf16")


@dataclasses.dataclass(frozen=True)
class ChunkWorkload:
    """One chunked-forward problem: shapes, gate kind and input dtype."""

    name: str
    mode: str
    dtype: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int = 64
    s0_std: Optional[float] = None  # None: S0 = 0 (passed as a null pointer)
    returns_state: bool = True

    @property
    def tokens(self) -> int:
        return self.B * self.T


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """A run of single-token recurrent steps over a batch of fp32 states."""

    name: str
    mode: str
    dtype: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    s_std: float = 0.02


# The workloads, named by what they are. Shapes and distributions follow the
# pages' model sizes (350M-3B, head dim 128, chunk 64) and their 4k-32k+
# sequence-length sweeps.
CHUNK_WORKLOADS: Dict[str, ChunkWorkload] = {
    w.name: w
    for w in (
        ChunkWorkload("gdn_f32_b1_h2_t256_d64", "scalar", "f32", 1, 256, 2, 64, 64),
        ChunkWorkload("deltanet_bf16_b8_h8_t4096_d128", "none", "bf16", 8, 4096, 8, 128, 128),
        ChunkWorkload("gdn_bf16_b8_h8_t4096_d128", "scalar", "bf16", 8, 4096, 8, 128, 128),
        ChunkWorkload("kda_bf16_b4_h16_t8192_d128", "channel", "bf16", 4, 8192, 16, 128, 128),
        ChunkWorkload("gdn_bf16_b1_h16_t65536_d128", "scalar", "bf16", 1, 65536, 16, 128, 128),
    )
}

DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    w.name: w
    for w in (DecodeWorkload("gdn_decode_bf16_b256_h16_d128", "scalar", "bf16", 256, 16, 128, 128, 256),)
}

# Seeds: one per workload, fixed, so every test and bench run sees the same data.
WORKLOAD_SEEDS = {
    "gdn_f32_b1_h2_t256_d64": 1,
    "deltanet_bf16_b8_h8_t4096_d128": 2,
    "gdn_bf16_b8_h8_t4096_d128": 3,
    "kda_bf16_b4_h16_t8192_d128": 4,
    "gdn_bf16_b1_h16_t65536_d128": 5,
    "gdn_decode_bf16_b256_h16_d128": 5,
}


def _torch_dtype(dtype: str) -> torch.dtype:
    if dtype == "f32":
        return torch.float32
    if dtype == "bf16":
        return torch.bfloat16
    raise ValueError(f"unknown dtype {dtype!r}")


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def make_chunk_inputs(
    B: int,
    T: int,
    H: int,
    dk: int,
    dv: int,
    mode: str,
    dtype: str,
    seed: int,
    s0_std: Optional[float] = None,
    g_scale: float = 0.05,
) -> Dict[str, Optional[torch.Tensor]]:
    """Seeded CPU tensors for one chunked forward.

    Returns ``q, k`` [B,T,H,dk] and ``v`` [B,T,H,dv] in ``dtype``; ``beta``
    [B,T,H] fp32; ``g`` fp32 ([B,T,H] scalar, [B,T,H,dk] channel, None for
    mode "none"); ``S0`` [B,H,dv,dk] fp32 or None. All contiguous.
    """
    if mode not in DECAY_MODES:
        raise ValueError(f"unknown decay mode {mode!r}")
    gen = torch.Generator().manual_seed(int(seed))
    q = torch.randn(B, T, H, dk, generator=gen)
    k = torch.randn(B, T, H, dk, generator=gen)
    v = torch.randn(B, T, H, dv, generator=gen)
    beta_logit = torch.randn(B, T, H, generator=gen)
    g = None
    if mode == "scalar":
        g = -g_scale * F.softplus(torch.randn(B, T, H, generator=gen))
    elif mode == "channel":
        g = -g_scale * F.softplus(torch.randn(B, T, H, dk, generator=gen))
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(B, H, dv, dk, generator=gen)
    td = _torch_dtype(dtype)
    return {
        "q": _unit(q).to(td).contiguous(),
        "k": _unit(k).to(td).contiguous(),
        "v": v.to(td).contiguous(),
        "beta": torch.sigmoid(beta_logit).contiguous(),
        "g": None if g is None else g.contiguous(),
        "S0": None if S0 is None else S0.contiguous(),
    }


def make_raw_chunk_inputs(
    B: int,
    T: int,
    H: int,
    dk: int,
    dv: int,
    mode: str,
    dtype: str,
    seed: int,
    s0_std: Optional[float] = None,
) -> Dict[str, Optional[torch.Tensor]]:
    """Seeded CPU tensors for a chunked forward whose prologue runs in the kernels: the draws
    before any squashing or normalisation.

    ``q, k`` [B,T,H,dk]: N(0, 1) vectors, each times a length drawn from U(0.25, 4) (so that
    their norms differ); ``v`` [B,T,H,dv] N(0, 1); ``beta`` [B,T,H] fp32 logits N(0, 1);
    ``g`` fp32 gate logits N(0, 1) ([B,T,H] scalar, [B,T,H,dk] channel, None for "none");
    ``gate_scale`` [H] fp32 from U(0.02, 1); ``S0`` as in ``make_chunk_inputs``. Draw order:
    q, k, v, beta-logit, g-logit, S0, the q lengths, the k lengths, gate_scale.
    """
    if mode not in DECAY_MODES:
        raise ValueError(f"unknown decay mode {mode!r}")
    gen = torch.Generator().manual_seed(int(seed))
    q = torch.randn(B, T, H, dk, generator=gen)
    k = torch.randn(B, T, H, dk, generator=gen)
    v = torch.randn(B, T, H, dv, generator=gen)
    beta_logit = torch.randn(B, T, H, generator=gen)
    a = None
    if mode == "scalar":
        a = torch.randn(B, T, H, generator=gen)
    elif mode == "channel":
        a = torch.randn(B, T, H, dk, generator=gen)
    S0 = None
    if s0_std is not None:
        S0 = s0_std * torch.randn(B, H, dv, dk, generator=gen)
    q = q * (0.25 + 3.75 * torch.rand(B, T, H, 1, generator=gen))
    k = k * (0.25 + 3.75 * torch.rand(B, T, H, 1, generator=gen))
    gate_scale = 0.02 + 0.98 * torch.rand(H, generator=gen)
    td = _torch_dtype(dtype)
    return {
        "q": q.to(td).contiguous(),
        "k": k.to(td).contiguous(),
        "v": v.to(td).contiguous(),
        "beta": beta_logit.contiguous(),
        "g": None if a is None else a.contiguous(),
        "S0": None if S0 is None else S0.contiguous(),
        "gate_scale": gate_scale.contiguous(),
    }


def make_gdn2_gates(B: int, T: int, H: int, dk: int, dv: int, seed: int) -> Dict[str, torch.Tensor]:
    """Seeded Gated DeltaNet-2 gates: ``erase`` [B,T,H,dk] and ``write`` [B,T,H,dv], fp32 draws
    from U(0, 1) (the range of a sigmoid gate). Draw order: erase, write."""
    gen = torch.Generator().manual_seed(int(seed))
    return {"erase": torch.rand(B, T, H, dk, generator=gen).contiguous(),
            "write": torch.rand(B, T, H, dv, generator=gen).contiguous()}


def workload_inputs(w: ChunkWorkload, seed: Optional[int] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of a named chunked workload (its fixed seed unless overridden)."""
    s = WORKLOAD_SEEDS.get(w.name, 0) if seed is None else seed
    return make_chunk_inputs(w.B, w.T, w.H, w.dk, w.dv, w.mode, w.dtype, s, w.s0_std)


def make_decode_state(w: DecodeWorkload, seed: int) -> torch.Tensor:
    """Initial fp32 states S ~ N(0, s_std), shape [B, H, dv, dk]."""
    gen = torch.Generator().manual_seed(int(seed))
    return (w.s_std * torch.randn(w.B, w.H, w.dv, w.dk, generator=gen)).contiguous()


def make_decode_step(w: DecodeWorkload, seed: int, step: int) -> Dict[str, Optional[torch.Tensor]]:
    """Fresh tokens for one decode step: q,k [B,H,dk], v [B,H,dv] (dtype),
    beta [B,H] fp32, g [B,H] or [B,H,dk] fp32 (None for mode "none")."""
    x = make_chunk_inputs(w.B, 1, w.H, w.dk, w.dv, w.mode, w.dtype, seed * 1_000_003 + 7919 * (step + 1))
    out = {}
    for name, t in x.items():
        if t is None or name == "S0":
            out[name] = None if name != "S0" else None
            continue
        out[name] = t.reshape((w.B,) + tuple(t.shape[2:])).contiguous()
    out.pop("S0")
    return out
