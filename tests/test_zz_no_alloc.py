"""gdn_chunk_fwd_noalloc: the chunk forward for callers that cannot allocate
device memory (the library supplies the workspace from a fixed scratch array).

Collected last on purpose, so that a run stopping at the first failure has
run every other test first.

The GPU tests call the entry point through the C ABI and compare it with the
regular gdn_chunk_fwd given a caller-allocated workspace.  The forward's
result does not depend on the workspace size (only the length of the waves
does), so the two must agree to the bit.  Between two calls with the same
inputs a call with other inputs (another gate kind, sequence length and
initial state) leaves different data in the shared scratch, so a kernel that
read scratch before writing it would not reproduce its first result.  The
host-only tests check the refusals that happen before anything is launched."""
import pytest
import torch

import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import _lib
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import to_dev


def call_noalloc(d, gate, S0, o, S1, B=None, H=None):
    Bx, T, Hx, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    ptr = lambda t: None if t is None else t.data_ptr()
    return _lib.load().gdn_chunk_fwd_noalloc(
        ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["beta"]), ptr(d["g"]), gate, ptr(S0), ptr(o),
        ptr(S1), Bx if B is None else B, T, Hx if H is None else H, Dk, Dv, 64, _lib.GDN_BF16,
        torch.cuda.current_stream().cuda_stream)


def regular(x, d):
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    need = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, torch.bfloat16, x["gate_kind"])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o = torch.empty(B, T, H, Dv, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(B, H, Dk, Dv, device="cuda")
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o, S,
                      workspace=ws)
    torch.cuda.synchronize()
    return o, S


def noalloc(x, d):
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    o = torch.full((B, T, H, Dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, H, Dk, Dv), float("nan"), device="cuda")
    assert call_noalloc(d, x["gate_kind"], d["S0"], o, S) == _lib.GDN_OK
    torch.cuda.synchronize()
    return o, S


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_point_bit_for_bit():
    # X runs several waves through the scratch; Y (another gate kind, twice the
    # length, another initial state) overwrites it in between
    X = gi.make_inputs(4, 2048, 16, 128, 128, dtype=torch.bfloat16, gate="scalar", s0_std=0.02,
                       seed=7)
    Y = gi.make_inputs(4, 4096, 16, 128, 128, dtype=torch.bfloat16, gate="per_dim",
                       gate_scale=0.05, s0_std=0.05, seed=11)
    dX, dY = to_dev(X), to_dev(Y)
    cap = _lib.load().gdn_chunk_fwd_noalloc_scratch_bytes()
    for x in (X, Y):
        B, T, H, Dk = x["q"].shape
        least = gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, Dk, Dk, 64, torch.bfloat16,
                                                      x["gate_kind"])
        assert 0 < least <= cap
    refX, refY = regular(X, dX), regular(Y, dY)
    for x, d, ref in ((X, dX, refX), (Y, dY, refY), (X, dX, refX)):
        o, S = noalloc(x, d)
        assert torch.equal(o, ref[0]), "o differs from the regular entry point"
        assert torch.equal(S, ref[1]), "final state differs from the regular entry point"
    assert gdn.gdn_read_device_status() == 0


@pytest.mark.gpu
def test_noalloc_setup_call_leaves_nothing_to_reserve():
    """After the set-up call (no work: B = 0), a call with work changes the
    device's free memory by far less than the scratch's size."""
    x = gi.make_inputs(2, 512, 4, 128, 128, dtype=torch.bfloat16, gate="scalar", seed=3)
    d = to_dev(x)
    ref = regular(x, d)            # loads the forward's kernels first
    o = torch.empty_like(ref[0])
    S = torch.empty_like(ref[1])
    assert call_noalloc(d, x["gate_kind"], None, o, S, B=0) == _lib.GDN_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert call_noalloc(d, x["gate_kind"], None, o, S) == _lib.GDN_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    cap = _lib.load().gdn_chunk_fwd_noalloc_scratch_bytes()
    assert free0 - free1 < cap // 8, f"free memory dropped by {free0 - free1} bytes"
    assert torch.equal(o, ref[0]) and torch.equal(S, ref[1])


def test_noalloc_rejects_shapes_beyond_the_scratch():
    """1024 heads x 4 chunks need more workspace than the scratch holds: the
    call returns GDN_ERR_WORKSPACE before touching the (fake, never
    dereferenced) device pointers."""
    lib = _lib.load()
    cap = lib.gdn_chunk_fwd_noalloc_scratch_bytes()
    need = lib.gdn_chunk_fwd_workspace_min_bytes(1, 256, 1024, 128, 128, 64, _lib.GDN_BF16, 1)
    assert need > cap
    A = 1 << 40
    rc = lib.gdn_chunk_fwd_noalloc(A, A + (1 << 30), A + (2 << 30), A + (3 << 30), A + (4 << 30), 1,
                                   None, A + (5 << 30), None, 1, 256, 1024, 128, 128, 64,
                                   _lib.GDN_BF16, None)
    assert rc == _lib.GDN_ERR_WORKSPACE


def test_noalloc_setup_call_validates_sizes():
    """The set-up form (B = 0) still refuses sizes the forward does not
    support, before looking at any device."""
    lib = _lib.load()
    rc = lib.gdn_chunk_fwd_noalloc(None, None, None, None, None, 1, None, None, None, 0, 256, 4,
                                   96, 128, 64, _lib.GDN_BF16, None)
    assert rc == _lib.GDN_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path only")
def test_noalloc_setup_call_without_a_device_reports_cuda_error():
    lib = _lib.load()
    rc = lib.gdn_chunk_fwd_noalloc(None, None, None, None, None, 1, None, None, None, 0, 256, 4,
                                   128, 128, 64, _lib.GDN_BF16, None)
    assert rc == _lib.GDN_ERR_CUDA
