"""gdn_chunk_fwd_noalloc: the chunk forward for callers that cannot allocate
device memory (the library supplies the workspace from a fixed scratch array).

Collected last on purpose.  The GPU test calls the entry point through the C
ABI twice in a row (the second call finds the first call's leftovers in the
shared scratch) and checks both outputs and final states against the regular
gdn_chunk_fwd with a caller-allocated workspace, on a shape that runs several
waves through the workspace.  The host-only test checks that a shape needing
more than the scratch is refused before anything is launched."""
import ctypes

import pytest
import torch

import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import _lib
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import TOL, check, to_dev


def call_noalloc(d, gate, S0, o, S1):
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    ptr = lambda t: None if t is None else t.data_ptr()
    return _lib.load().gdn_chunk_fwd_noalloc(
        ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["beta"]), ptr(d["g"]), gate, ptr(S0), ptr(o),
        ptr(S1), B, T, H, Dk, Dv, 64, _lib.GDN_BF16, torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_noalloc_matches_regular_entry_point_twice():
    x = gi.make_inputs(4, 2048, 16, 128, 128, dtype=torch.bfloat16, gate="scalar", s0_std=0.02,
                       seed=7)
    d = to_dev(x)
    B, T, H, D = 4, 2048, 16, 128
    least = gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, D, D, 64, torch.bfloat16,
                                                  x["gate_kind"])
    assert 0 < least <= _lib.load().gdn_chunk_fwd_noalloc_scratch_bytes()
    need = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, D, D, 64, torch.bfloat16, x["gate_kind"])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o_ref = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    S_ref = torch.empty(B, H, D, D, device="cuda")
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o_ref,
                      S_ref, workspace=ws)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full((B, T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, D, D), float("nan"), device="cuda")
        assert call_noalloc(d, x["gate_kind"], d["S0"], o, S) == _lib.GDN_OK
        torch.cuda.synchronize()
        check("o (no-alloc vs regular)", o, o_ref.double().cpu().numpy(), TOL[torch.bfloat16])
        check("S (no-alloc vs regular)", S, S_ref.double().cpu().numpy(), TOL[torch.bfloat16])
    assert gdn.gdn_read_device_status() == 0


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
