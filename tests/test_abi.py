"""Host-only tests of the C ABI: the library builds, loads and exports every
symbol include/gdn.h declares, and every argument error is reported by status
code before anything is launched (no GPU needed; nothing here dereferences
the fake device pointers, because validation rejects the call first)."""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
A = 0x10000          # a 16-byte-aligned fake device address (never dereferenced)
MIS = 0x10008        # misaligned


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names.update(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_symbols()
    assert {"gdn_chunk_fwd", "gdn_decode_step"} <= names
    for name in names:
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTED) == names


def test_status_strings_and_version():
    assert gdn.gdn_abi_version() == 1
    assert gdn.gdn_status_string(0) == "GDN_OK"
    assert gdn.gdn_status_string(3) == "GDN_ERR_WORKSPACE"
    assert gdn.gdn_status_string(99) == "GDN_ERR_UNKNOWN"


def test_workspace_bytes():
    lib = _lib.load()
    bad = ctypes.c_size_t(-1).value
    assert lib.gdn_chunk_fwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, 1) != bad
    assert lib.gdn_chunk_fwd_workspace_bytes(4, 2048, 16, 96, 128, 64, 0, 1) == bad
    assert lib.gdn_chunk_fwd_workspace_bytes(4, 2048, 16, 128, 128, 32, 0, 1) == bad
    assert lib.gdn_chunk_fwd_workspace_bytes(-1, 2048, 16, 128, 128, 64, 0, 1) == bad
    assert lib.gdn_chunk_fwd_workspace_min_bytes(4, 2048, 16, 96, 128, 64, 0, 1) == bad
    assert lib.gdn_chunk_fwd_workspace_min_bytes(-1, 2048, 16, 128, 128, 64, 0, 1) == bad


@pytest.mark.parametrize("B,T,H", [(4, 2048, 16), (4, 4096, 16), (1, 65536, 32), (1, 64, 1),
                                   (2, 200, 2), (1, 256, 1024), (3, 4097, 5)])
def test_workspace_min_not_above_full_speed_size(B, T, H):
    """The least workspace the forward accepts is at most the full-speed size;
    both are 0 without tokens and grow with the number of heads."""
    lib = _lib.load()
    for gate in (0, 1, 2):
        full = lib.gdn_chunk_fwd_workspace_bytes(B, T, H, 128, 128, 64, 0, gate)
        least = lib.gdn_chunk_fwd_workspace_min_bytes(B, T, H, 128, 128, 64, 0, gate)
        assert 0 < least <= full
        assert lib.gdn_chunk_fwd_workspace_min_bytes(B, 0, H, 128, 128, 64, 0, gate) == 0
        # the fp32 path needs none
        assert lib.gdn_chunk_fwd_workspace_min_bytes(B, T, H, 128, 128, 64, 1, gate) == 0


def chunk_call(**over):
    args = dict(q=A, k=A, v=A, beta=A, g=A, gate=1, s0=None, o=A * 2, s1=None, B=1, T=64, H=1,
                Dk=64, Dv=64, chunk=64, dtype=0, ws=None, ws_bytes=0, stream=None)
    args.update(over)
    return _lib.load().gdn_chunk_fwd(args["q"], args["k"], args["v"], args["beta"], args["g"],
                                     args["gate"], args["s0"], args["o"], args["s1"], args["B"],
                                     args["T"], args["H"], args["Dk"], args["Dv"], args["chunk"],
                                     args["dtype"], args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(o=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(beta=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(g=None), _lib.GDN_ERR_INVALID_ARG),                 # gate scalar needs g
    (dict(gate=0), _lib.GDN_ERR_INVALID_ARG),                 # gate none forbids g
    (dict(gate=3), _lib.GDN_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.GDN_ERR_INVALID_ARG),
    (dict(B=-1), _lib.GDN_ERR_INVALID_ARG),
    (dict(T=-5), _lib.GDN_ERR_INVALID_ARG),
    (dict(Dk=96), _lib.GDN_ERR_UNSUPPORTED),
    (dict(Dv=32), _lib.GDN_ERR_UNSUPPORTED),
    (dict(chunk=128), _lib.GDN_ERR_UNSUPPORTED),
    (dict(q=MIS), _lib.GDN_ERR_INVALID_ARG),
    (dict(o=MIS), _lib.GDN_ERR_INVALID_ARG),
    (dict(s1=A * 2), _lib.GDN_ERR_INVALID_ARG),               # final state overlaps o
    (dict(s0=A * 4, s1=A * 4 + 4096), _lib.GDN_ERR_INVALID_ARG),  # partial state overlap
    (dict(s0=A * 2), _lib.GDN_ERR_INVALID_ARG),               # o overlaps the initial state
])
def test_chunk_fwd_argument_errors(over, code):
    assert chunk_call(**over) == code


def test_chunk_fwd_noop_sizes():
    assert chunk_call(B=0) == _lib.GDN_OK
    assert chunk_call(H=0, q=None, o=None) == _lib.GDN_OK


def test_chunk_fwd_workspace_errors():
    """The tensor-core path (bf16, d = 128) needs its workspace: a buffer
    smaller than gdn_chunk_fwd_workspace_min_bytes, or none at all, is refused
    with GDN_ERR_WORKSPACE before anything is launched."""
    lib = _lib.load()
    least = lib.gdn_chunk_fwd_workspace_min_bytes(1, 256, 2, 128, 128, 64, 0, 1)
    assert least > 0
    base = dict(B=1, T=256, H=2, Dk=128, Dv=128, o=A * 64)
    assert chunk_call(ws=A * 1024, ws_bytes=least - 16, **base) == _lib.GDN_ERR_WORKSPACE
    assert chunk_call(ws=None, ws_bytes=least, **base) == _lib.GDN_ERR_WORKSPACE


def test_chunk_fwd_index_range():
    """Token and (batch, head) counts past 2^31 - 1 are refused as unsupported
    (the kernels index tokens and heads with 32-bit integers)."""
    assert chunk_call(B=65536, T=65536) == _lib.GDN_ERR_UNSUPPORTED
    assert chunk_call(B=65536, H=65536) == _lib.GDN_ERR_UNSUPPORTED
    assert decode_call(N=65536, H=65536) == _lib.GDN_ERR_UNSUPPORTED


def decode_call(**over):
    args = dict(q=A, k=A, v=A, beta=A, g=A, gate=1, state=A * 8, o=A * 2, N=2, H=2, Dk=64,
                Dv=64, dtype=0, stream=None)
    args.update(over)
    return _lib.load().gdn_decode_step(args["q"], args["k"], args["v"], args["beta"], args["g"],
                                       args["gate"], args["state"], args["o"], args["N"],
                                       args["H"], args["Dk"], args["Dv"], args["dtype"],
                                       args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(state=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(o=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(g=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(gate=2, g=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(N=-1), _lib.GDN_ERR_INVALID_ARG),
    (dict(Dk=256), _lib.GDN_ERR_UNSUPPORTED),
    (dict(state=A * 8 + 4), _lib.GDN_ERR_INVALID_ARG),
    (dict(o=A * 8 + 256), _lib.GDN_ERR_INVALID_ARG),          # o inside the state
])
def test_decode_argument_errors(over, code):
    assert decode_call(**over) == code


def test_decode_noop_sizes():
    assert decode_call(N=0, q=None) == _lib.GDN_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path only")
def test_valid_call_without_a_device_reports_cuda_error():
    assert chunk_call() == _lib.GDN_ERR_CUDA
    assert decode_call() == _lib.GDN_ERR_CUDA


def test_python_binding_rejects_bad_tensors():
    q = torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        gdn.gdn_chunk_fwd(q, q, q, torch.zeros(1, 64, 1), None, 0, None, q, None)
    with pytest.raises(ValueError):
        gdn.gdn_chunk_fwd(q.transpose(1, 3), q, q, None, None, 0, None, q, None)


# ------------------------------------------------ preconditioned delta rule
def wk_call(**over):
    args = dict(q=A, k=A, kw=A * 4, v=A, beta=A, g=A, gate=1, s0=None, o=A * 2, s1=None, B=1,
                T=64, H=1, Dk=128, Dv=128, chunk=64, dtype=0, ws=None, ws_bytes=0, stream=None)
    args.update(over)
    return _lib.load().gdn_chunk_fwd_wk(args["q"], args["k"], args["kw"], args["v"],
                                        args["beta"], args["g"], args["gate"], args["s0"],
                                        args["o"], args["s1"], args["B"], args["T"], args["H"],
                                        args["Dk"], args["Dv"], args["chunk"], args["dtype"],
                                        args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(dtype=1), _lib.GDN_ERR_UNSUPPORTED),                # a write key needs bf16 ...
    (dict(Dk=64, Dv=64), _lib.GDN_ERR_UNSUPPORTED),           # ... and d = 128
    (dict(kw=MIS), _lib.GDN_ERR_INVALID_ARG),
    (dict(q=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(s1=A * 4), _lib.GDN_ERR_INVALID_ARG),               # final state overlaps the write key
    (dict(kw=A * 2), _lib.GDN_ERR_INVALID_ARG),               # the write key overlaps o
    (dict(), _lib.GDN_ERR_WORKSPACE),                         # valid, but no workspace
])
def test_chunk_fwd_wk_argument_errors(over, code):
    assert wk_call(**over) == code


def test_chunk_fwd_wk_without_write_key_is_chunk_fwd():
    """k_write = NULL takes exactly gdn_chunk_fwd's path: the fp32 and d = 64
    shapes it supports are accepted up to the (missing) device."""
    assert wk_call(kw=None, B=0) == _lib.GDN_OK
    assert wk_call(kw=None, dtype=1, Dk=64, Dv=64, B=0) == _lib.GDN_OK


def osdn_call(**over):
    args = dict(k=A, beta=A * 2, r=None, eta=0.5, d0=None, kw=A * 4, d1=None, B=1, T=64, H=1,
                Dk=128, dtype=0, ws=A * 8, ws_bytes=1 << 20, stream=None)
    args.update(over)
    return _lib.load().gdn_osdn_precondition(args["k"], args["beta"], args["r"], args["eta"],
                                             args["d0"], args["kw"], args["d1"], args["B"],
                                             args["T"], args["H"], args["Dk"], args["dtype"],
                                             args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(k=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(kw=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(beta=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(eta=float("nan")), _lib.GDN_ERR_INVALID_ARG),
    (dict(eta=float("inf")), _lib.GDN_ERR_INVALID_ARG),
    (dict(Dk=96), _lib.GDN_ERR_UNSUPPORTED),
    (dict(dtype=5), _lib.GDN_ERR_INVALID_ARG),
    (dict(B=-1), _lib.GDN_ERR_INVALID_ARG),
    (dict(kw=MIS), _lib.GDN_ERR_INVALID_ARG),
    (dict(kw=A), _lib.GDN_ERR_INVALID_ARG),                   # write keys over the keys
    (dict(d1=A * 4), _lib.GDN_ERR_INVALID_ARG),               # final d over the write keys
    (dict(d0=A * 1024, d1=A * 1024 + 16), _lib.GDN_ERR_INVALID_ARG),   # partial d overlap
    (dict(B=65536, T=65536), _lib.GDN_ERR_UNSUPPORTED),
    (dict(ws=None), _lib.GDN_ERR_WORKSPACE),
    (dict(ws_bytes=1024), _lib.GDN_ERR_WORKSPACE),            # below one block's 18 KB
    (dict(ws=A), _lib.GDN_ERR_INVALID_ARG),                   # workspace over the keys
    (dict(ws=A * 8 + 8), _lib.GDN_ERR_INVALID_ARG),           # misaligned workspace
])
def test_osdn_precondition_argument_errors(over, code):
    assert osdn_call(**over) == code


def test_osdn_precondition_noop_sizes():
    assert osdn_call(B=0) == _lib.GDN_OK
    assert osdn_call(H=0, k=None, kw=None) == _lib.GDN_OK
    assert osdn_call(T=0, k=None, kw=None, beta=None) == _lib.GDN_OK   # nothing to write


# -------------------------------------------------------------------- backward
def bwd_call(**over):
    args = dict(q=A, k=A, v=A, beta=A, g=A, gate=1, s0=None, do_=A, ds=None, dq=A * 64,
                dk=A * 128, dv=A * 192, dbeta=A * 256, dg=A * 320, ds0=None, B=1, T=64, H=1,
                Dk=128, Dv=128, chunk=64, dtype=0, ws=None, ws_bytes=0, stream=None)
    args.update(over)
    a = args
    return _lib.load().gdn_chunk_bwd(a["q"], a["k"], a["v"], a["beta"], a["g"], a["gate"], a["s0"],
                                     a["do_"], a["ds"], a["dq"], a["dk"], a["dv"], a["dbeta"],
                                     a["dg"], a["ds0"], a["B"], a["T"], a["H"], a["Dk"], a["Dv"],
                                     a["chunk"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(gate=2), _lib.GDN_ERR_UNSUPPORTED),                 # per-dimension gate: not built
    (dict(dtype=1), _lib.GDN_ERR_UNSUPPORTED),
    (dict(Dk=64, Dv=64), _lib.GDN_ERR_UNSUPPORTED),
    (dict(dq=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(dg=None), _lib.GDN_ERR_INVALID_ARG),                # scalar gate needs dg
    (dict(g=None), _lib.GDN_ERR_INVALID_ARG),
    (dict(dq=MIS), _lib.GDN_ERR_INVALID_ARG),
    (dict(dq=A), _lib.GDN_ERR_INVALID_ARG),                   # output over an input
    (dict(dk=A * 64), _lib.GDN_ERR_INVALID_ARG),              # two outputs overlap
    (dict(), _lib.GDN_ERR_WORKSPACE),
    (dict(gate=3), _lib.GDN_ERR_INVALID_ARG),
])
def test_chunk_bwd_argument_errors(over, code):
    assert bwd_call(**over) == code


def test_chunk_bwd_workspace_bytes():
    lib = _lib.load()
    bad = ctypes.c_size_t(-1).value
    n = lib.gdn_chunk_bwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, 1)
    assert n != bad and n > 2 * 64 * 32 * 128 * 128 * 4
    assert lib.gdn_chunk_bwd_workspace_bytes(4, 2048, 16, 128, 128, 64, 0, 2) == bad
    assert lib.gdn_chunk_bwd_workspace_bytes(4, 2048, 16, 64, 64, 64, 0, 1) == bad
    assert lib.gdn_chunk_bwd_workspace_bytes(4, 0, 16, 128, 128, 64, 0, 1) == 0
