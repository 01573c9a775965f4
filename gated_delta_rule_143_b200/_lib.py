"""ctypes loader for libgdr.so (the C ABI in include/gdr.h).

There is no fallback: if the shared library is missing or cannot be loaded,
every call raises. Build it with ``python -m gated_delta_rule_143_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

# Mirrors of the C enums (include/gdr.h).
GDR_OK = 0
STATUS_NAMES = {
    0: "GDR_OK", -1: "GDR_ERR_INVALID_ARG", -2: "GDR_ERR_UNSUPPORTED", -3: "GDR_ERR_MISALIGNED",
    -4: "GDR_ERR_WORKSPACE", -5: "GDR_ERR_CUDA", -6: "GDR_ERR_TIMEOUT", -7: "GDR_ERR_DEVICE",
    -8: "GDR_ERR_RANGE",
}
DECAY_MODES = {"none": 0, "scalar": 1, "channel": 2}
DTYPE_F32, DTYPE_BF16 = 0, 1
PLANS = {0: "invalid", 1: "cuda_core", 2: "two_pass", 3: "fused", 4: "prep_fused", 5: "scan"}
PRO_L2NORM_QK, PRO_BETA_SIGMOID, PRO_GATE_SOFTPLUS = 1, 2, 4  # gdr_prologue flags

# Every symbol the header declares: name -> (restype, argtypes).
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "gdr_chunk_fwd": (_i, [_vp] * 8 + [_i] * 9 + [_vp, _sz, _vp]),
    "gdr_chunk_fwd_workspace_bytes": (_sz, [_i] * 9),
    "gdr_chunk_fwd_launches": (_i, [_i] * 9),
    "gdr_chunk_fwd_plan": (_i, [_i] * 9 + [_vp]),
    "gdr_chunk_fwd_ex": (_i, [_vp] * 8 + [_i] * 10 + [_vp, _vp, _sz, _vp]),
    "gdr_decode_step": (_i, [_vp] * 7 + [_i] * 7 + [_vp]),
    "gdr_chunk_bwd": (_i, [_vp] * 14 + [_i] * 7 + [_vp, _sz, _vp]),
    "gdr_chunk_fwd_gdn2": (_i, [_vp] * 9 + [_i] * 9 + [_vp, _sz, _vp]),
    "gdr_chunk_fwd_gdn2_workspace_bytes": (_sz, [_i] * 9),
    "gdr_chunk_fwd_scan": (_i, [_vp] * 8 + [_i] * 10 + [_vp, _sz, _vp]),
    "gdr_chunk_fwd_scan_workspace_bytes": (_sz, [_i] * 10),
    "gdr_decode_step_gdn2": (_i, [_vp] * 8 + [_i] * 7 + [_vp]),
    "gdr_chunk_bwd_workspace_bytes": (_sz, [_i] * 7),
    "gdr_decode_step_ex": (_i, [_vp] * 7 + [_i] * 8 + [_vp, _vp]),
    "gdr_chunk_fwd_noalloc": (_i, [_vp] * 8 + [_i] * 9 + [_vp]),
    "gdr_chunk_fwd_host": (_i, [_vp] * 8 + [_i] * 9 + [_vp, _sz, _vp]),
    "gdr_chunk_fwd_host_staging_bytes": (_sz, [_i] * 9),
    "gdr_profile_next_call": (_i, [_vp, _i]),
    "gdr_sync_status": (_i, [_vp]),
    "gdr_selftest_bounded_wait": (_i, [ctypes.c_uint, _vp, _vp]),
    "gdr_last_error": (ctypes.c_char_p, []),
    "gdr_version": (_i, []),
}

_lib = None
_lock = threading.Lock()


class GdrError(RuntimeError):
    """A non-zero gdr_status from the library."""

    def __init__(self, code: int, message: str):
        self.code = code
        self.status = STATUS_NAMES.get(code, str(code))
        super().__init__(f"{self.status}: {message}")


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing; build it with `python -m gated_delta_rule_143_b200.build` "
                    "(there is no non-CUDA fallback)")
            l = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(l, name)
                fn.restype = res
                fn.argtypes = args
            _lib = l
    return _lib


def check(rc: int) -> None:
    if rc != GDR_OK:
        msg = lib().gdr_last_error()
        raise GdrError(rc, msg.decode() if msg else "")
