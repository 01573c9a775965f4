"""Host-side checks of the C ABI (CPU only: nothing here launches a kernel).

The library must load, export every function include/gdr.h declares, and turn
bad arguments into error codes before touching the device.
"""
import ctypes
import os
import re

import pytest

from gated_delta_rule_143_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gdr_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for want in ("gdr_chunk_fwd", "gdr_chunk_fwd_workspace_bytes", "gdr_decode_step", "gdr_sync_status",
                 "gdr_last_error", "gdr_version"):
        assert want in names
    assert set(names) == set(_lib.SIGNATURES), "binding signatures and header disagree"


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.gdr_version() >= 100


def test_library_links_no_oracle_code():
    """The product library and the oracle share nothing: no oracle symbol in libgdr.so."""
    data = open(_lib.LIB_PATH, "rb").read()
    assert b"gdr_oracle" not in data


def _chunk(**kw):
    """Calls gdr_chunk_fwd with fake addresses. Only ever used with an argument error."""
    M = 1 << 24  # fake, widely spaced addresses: every case below fails validation on the host
    a = dict(q=1 * M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, S0=None, o=6 * M, S_T=None, B=1, T=64, H=1, dk=128, dv=128,
             chunk=64, mode=1, dtype=1, odt=0, ws=None, wsb=0, stream=None)
    a.update(kw)
    lib = _lib.lib()
    return lib.gdr_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["o"], a["S_T"], a["B"], a["T"],
                             a["H"], a["dk"], a["dv"], a["chunk"], a["mode"], a["dtype"], a["odt"], a["ws"],
                             a["wsb"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -1), (dict(T=0), -1), (dict(H=-1), -1), (dict(dk=0), -1),
    (dict(mode=7), -1), (dict(dtype=3), -1), (dict(odt=5), -1), (dict(dtype=0, odt=1), -2),
    (dict(dk=96), -2), (dict(dv=256), -2), (dict(chunk=32), -2),
    (dict(q=None), -1), (dict(beta=None), -1), (dict(o=None), -1), (dict(g=None), -1),
    (dict(q=(1 << 24) + 2), -3), (dict(o=(6 << 24) + 4), -3),
])
def test_chunk_fwd_rejects_bad_arguments_on_host(kw, code):
    assert _chunk(**kw) == code
    assert len(_lib.lib().gdr_last_error()) > 0


def test_chunk_fwd_rejects_output_aliasing_an_input():
    # o overlapping q is an error (addresses are never dereferenced: it fails on the host)
    assert _chunk(o=1 << 24) == -1
    assert b"overlaps" in _lib.lib().gdr_last_error()


def test_workspace_query_is_host_only():
    lib = _lib.lib()
    assert lib.gdr_chunk_fwd_workspace_bytes(0, 64, 1, 128, 128, 64, 1, 1, 0) == 0  # invalid -> 0
    n = lib.gdr_chunk_fwd_workspace_bytes(8, 4096, 8, 128, 128, 64, 1, 1, 0)
    assert n >= 0 and n < (1 << 34)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -1), (dict(dk=48), -2), (dict(mode=5), -1), (dict(S=None), -1), (dict(S=20), -3),
])
def test_decode_rejects_bad_arguments_on_host(kw, code):
    a = dict(q=16, k=32, v=48, g=64, beta=80, S=1 << 20, o=1 << 21, B=2, H=2, dk=128, dv=128, mode=1, dtype=1, odt=0)
    a.update(kw)
    rc = _lib.lib().gdr_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S"], a["o"], a["B"], a["H"],
                                    a["dk"], a["dv"], a["mode"], a["dtype"], a["odt"], None)
    assert rc == code


def test_error_object_carries_status_name():
    e = _lib.GdrError(-3, "x")
    assert e.status == "GDR_ERR_MISALIGNED" and "x" in str(e)


def test_profile_next_call_validates_on_host():
    L = _lib.lib()
    assert L.gdr_profile_next_call(None, 9) == -1
    assert L.gdr_profile_next_call(None, -1) == -1
    assert L.gdr_profile_next_call(None, 1) == -1
    assert L.gdr_profile_next_call(None, 0) == 0  # clears; enqueues nothing


def test_plan_query_is_host_only():
    import torch
    import gated_delta_rule_143_b200 as gdr
    bf = torch.bfloat16
    assert gdr.chunk_fwd_plan(1, 4096, 8, 128, 128, 64, "scalar", bf) == ("fused", 0)
    assert gdr.chunk_fwd_plan(7, 4096, 8, 128, 128, 64, "none", bf) == ("fused", 0)
    plan, c1 = gdr.chunk_fwd_plan(8, 4096, 8, 128, 128, 64, "scalar", bf)
    assert plan == "prep_fused" and 0 < c1 < 64
    assert gdr.chunk_fwd_plan(13, 4096, 8, 128, 128, 64, "scalar", bf) == ("two_pass", 0)
    assert gdr.chunk_fwd_plan(1, 4096, 8, 128, 128, 64, "channel", bf) == ("fused", 0)
    plan_ch, c1_ch = gdr.chunk_fwd_plan(4, 8192, 16, 128, 128, 64, "channel", bf)
    assert plan_ch == "prep_fused" and 64 < c1_ch < 128
    assert gdr.chunk_fwd_plan(13, 4096, 8, 128, 128, 64, "channel", bf) == ("two_pass", 0)
    assert gdr.chunk_fwd_plan(1, 100, 2, 64, 64, 64, "scalar", torch.float32) == ("cuda_core", 0)
    # few heads, long sequences: the segment scan with 4 segments (4 launches)
    assert gdr.chunk_fwd_plan(1, 65536, 16, 128, 128, 64, "scalar", bf) == ("scan", 4)
    assert gdr.chunk_fwd_plan(1, 32768, 2, 128, 128, 64, "channel", bf) == ("scan", 16)
    assert gdr.chunk_fwd_plan(1, 65536, 8, 128, 128, 64, "scalar", bf) == ("scan", 8)
    assert gdr.chunk_fwd_plan(1, 16384, 16, 128, 128, 64, "none", bf) == ("scan", 4)
    assert gdr.chunk_fwd_plan(1, 16384 + 4096, 2, 128, 128, 64, "scalar", bf) == ("scan", 16)
    assert gdr.chunk_fwd_plan(1, 16384 + 64, 2, 128, 128, 64, "scalar", bf) == ("fused", 0)  # no T % 128 == 0
    assert gdr.chunk_fwd_plan(1, 8192, 2, 128, 128, 64, "scalar", bf) == ("fused", 0)  # 128 chunks: too short
    assert gdr.chunk_fwd_plan(2, 32768, 16, 128, 128, 64, "scalar", bf)[0] == "fused"  # 32 heads
    assert gdr.launches_per_chunk_fwd(1, 65536, 16, 128, 128, 64, "scalar", bf) == 4
    assert gdr.workspace_bytes(1, 65536, 16, 128, 128, 64, "scalar", bf) == \
        _lib.lib().gdr_chunk_fwd_scan_workspace_bytes(1, 65536, 16, 128, 128, 64, 1, 1, 0, 4)
    assert gdr.chunk_fwd_plan(0, 100, 2, 64, 64, 64, "scalar", torch.float32) == ("invalid", 0)
    # launches and workspace follow the plan
    assert gdr.launches_per_chunk_fwd(1, 4096, 8, 128, 128, 64, "scalar", bf) == 1
    assert gdr.launches_per_chunk_fwd(8, 4096, 8, 128, 128, 64, "scalar", bf) == 2
    block = 74752  # one hand-off block per chunk of a head

    def flags(heads, slots):  # a ready flag per slot, a consumed counter per head, one task counter
        return (heads * (slots + 1) + 1) * 4 + 255 & ~255

    # fused alone: a ring of eight slots per head
    assert gdr.workspace_bytes(1, 4096, 8, 128, 128, 64, "scalar", bf) == 8 * 8 * block + flags(8, 8)
    # prep + fused: c1 pre-computed blocks and a slot for every later chunk, i.e. one block per chunk
    assert gdr.workspace_bytes(8, 4096, 8, 128, 128, 64, "scalar", bf) == 64 * 64 * block + flags(64, 64 - c1)
    # a short sequence keeps eight slots even when it has fewer chunks
    assert gdr.workspace_bytes(1, 100, 8, 128, 128, 64, "scalar", bf) == 8 * 8 * block + flags(8, 8)
    # the channel gate: the same layouts; Gated DeltaNet-2 (erase / write gates) too, with its own
    # share of pre-computed chunks; two passes (one block per chunk of every head) above 100 heads
    assert gdr.workspace_bytes(1, 4096, 8, 128, 128, 64, "channel", bf) == 8 * 8 * block + flags(8, 8)
    _, c1c = gdr.chunk_fwd_plan(4, 8192, 16, 128, 128, 64, "channel", bf)
    assert gdr.workspace_bytes(4, 8192, 16, 128, 128, 64, "channel", bf) == 64 * 128 * block + flags(64, 128 - c1c)
    L = _lib.lib()
    assert L.gdr_chunk_fwd_gdn2_workspace_bytes(1, 8192, 8, 128, 128, 64, 2, 1, 1) == 8 * 8 * block + flags(8, 8)
    ws2 = L.gdr_chunk_fwd_gdn2_workspace_bytes(4, 8192, 16, 128, 128, 64, 2, 1, 1)
    assert any(ws2 == 64 * 128 * block + flags(64, d) for d in range(1, 128 - c1c))  # more chunks pre-computed
    assert L.gdr_chunk_fwd_gdn2_workspace_bytes(13, 8192, 8, 128, 128, 64, 2, 1, 1) == 104 * 128 * block


def test_host_entry_point_validates_on_host():
    L = _lib.lib()
    need = L.gdr_chunk_fwd_host_staging_bytes(8, 4096, 8, 128, 128, 64, 1, 1, 0)
    assert need > 0
    assert L.gdr_chunk_fwd_host_staging_bytes(0, 4096, 8, 128, 128, 64, 1, 1, 0) == 0
    M = 1 << 24  # fake addresses: the missing staging area is rejected before anything is enqueued
    rc = L.gdr_chunk_fwd_host(1 * M, 2 * M, 3 * M, 4 * M, 5 * M, None, 6 * M, None, 8, 4096, 8, 128, 128, 64, 1, 1, 0,
                              None, 0, None)
    assert rc == -4
    assert b"staging" in L.gdr_last_error()


@pytest.mark.parametrize("pro,mode,gs,code", [
    (8, 1, None, -1),             # unknown prologue bit
    (4, 0, None, -1),             # gate logits without a gated decay mode
    (4, 1, (7 << 24) + 4, -3),    # misaligned gate_scale
    (4, 1, (1 << 24) + 64, -1),   # the output o placed over gate_scale
])
def test_chunk_fwd_ex_validates_prologue_on_host(pro, mode, gs, code):
    M = 1 << 24
    o = 6 * M
    if code == -1 and gs is not None:
        o = gs  # o starts at gate_scale: an output overlapping an input
    rc = _lib.lib().gdr_chunk_fwd_ex(1 * M, 2 * M, 3 * M, 4 * M, 5 * M, None, o, None, 1, 64, 1, 128, 128, 64, mode, 1, 0,
                                     pro, gs, None, 0, None)
    assert rc == code
    assert len(_lib.lib().gdr_last_error()) > 0


@pytest.mark.parametrize("pro,mode,code", [(16, 1, -1), (4, 0, -1), (3, 5, -1)])
def test_decode_ex_validates_prologue_on_host(pro, mode, code):
    rc = _lib.lib().gdr_decode_step_ex(16, 32, 48, 64, 80, 1 << 20, 1 << 21, 2, 2, 128, 128, mode, 1, 0, pro, None, None)
    assert rc == code


def _bwd(**kw):
    """Calls gdr_chunk_bwd with fake, widely spaced addresses; used only with argument errors."""
    M = 1 << 26
    a = dict(q=1 * M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, S0=None, dO=6 * M, dST=None, dq=7 * M, dk=8 * M,
             dv=9 * M, dg=10 * M, dbeta=11 * M, dS0=None, B=1, T=16, H=1, d_k=64, d_v=64, mode=1, dtype=0,
             ws=12 * M, wsb=1 << 26)
    a.update(kw)
    return _lib.lib().gdr_chunk_bwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S0"], a["dO"], a["dST"], a["dq"],
                                    a["dk"], a["dv"], a["dg"], a["dbeta"], a["dS0"], a["B"], a["T"], a["H"], a["d_k"],
                                    a["d_v"], a["mode"], a["dtype"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -1), (dict(mode=9), -1), (dict(dtype=4), -1), (dict(d_k=256), -2), (dict(d_v=40), -2),
    (dict(g=None), -1), (dict(dg=None), -1), (dict(dO=None), -1), (dict(dq=None), -1),
    (dict(dk=(8 << 26) + 8), -3), (dict(wsb=100), -4), (dict(ws=None), -4),
    (dict(dv=(1 << 26) + 256), -1),  # dv (an output) over q
    (dict(dbeta=8 << 26), -1),       # two outputs overlap
])
def test_chunk_bwd_rejects_bad_arguments_on_host(kw, code):
    assert _bwd(**kw) == code
    assert len(_lib.lib().gdr_last_error()) > 0


def test_chunk_bwd_workspace_query():
    lib = _lib.lib()
    assert lib.gdr_chunk_bwd_workspace_bytes(2, 100, 3, 64, 32, 1, 0) == 2 * 3 * 100 * 64 * 32 * 4
    assert lib.gdr_chunk_bwd_workspace_bytes(2, 100, 3, 48, 32, 1, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(erase=None), -1), (dict(write=None), -1), (dict(dk=256), -2), (dict(chunk=32), -2),
    (dict(erase=(4 << 24) + 8), -3), (dict(o=(5 << 24) + 64), -1),
])
def test_chunk_fwd_gdn2_rejects_bad_arguments_on_host(kw, code):
    M = 1 << 24
    a = dict(q=1 * M, k=2 * M, v=3 * M, g=6 * M, erase=4 * M, write=5 * M, o=7 * M, dk=64, chunk=64)
    a.update(kw)
    rc = _lib.lib().gdr_chunk_fwd_gdn2(a["q"], a["k"], a["v"], a["g"], a["erase"], a["write"], None, a["o"], None, 1,
                                       16, 1, a["dk"], 64, a["chunk"], 2, 0, 0, None, 0, None)
    assert rc == code


def test_chunk_fwd_gdn2_workspace_query():
    lib = _lib.lib()
    # the channel decay at the tensor-core shapes runs the channel gate's plans: two heads run fused, a
    # ring of eight blocks per head and the ring's flags
    assert lib.gdr_chunk_fwd_gdn2_workspace_bytes(1, 128, 2, 128, 128, 64, 2, 1, 0) == \
        2 * 8 * 74752 + ((2 * 9 + 1) * 4 + 255 & ~255)
    assert lib.gdr_chunk_fwd_gdn2_workspace_bytes(1, 128, 2, 128, 128, 64, 1, 1, 0) == 0  # scalar: CUDA cores
    assert lib.gdr_chunk_fwd_gdn2_workspace_bytes(1, 128, 2, 64, 64, 64, 2, 0, 0) == 0    # fp32: CUDA cores
    M = 1 << 24  # missing workspace on the tensor-core route: rejected on the host
    rc = lib.gdr_chunk_fwd_gdn2(1 * M, 2 * M, 3 * M, 4 * M, 5 * M, 6 * M, None, 7 * M, None, 1, 128, 2, 128, 128, 64,
                                2, 1, 0, None, 0, None)
    assert rc == -4


def test_library_exports_only_declared_c_symbols():
    """Every unmangled symbol libgdr.so defines is an entry point of include/gdr.h (nothing internal
    leaks out with C linkage)."""
    import shutil
    import subprocess
    if shutil.which("nm") is None:
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True, check=True)
    names = {line.split()[-1] for line in out.stdout.splitlines() if line.strip()}
    c_names = {n for n in names if not n.startswith("_")}
    assert c_names == set(declared_functions()), sorted(c_names ^ set(declared_functions()))
