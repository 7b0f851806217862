"""GPU parity of the preconditioned delta rule ("OSDN: Improving Delta Rule with
Provable Online Preconditioning in Linear Attention", sec. 2.1-2.3) against the
fp64 oracle, through the C ABI:

  * phase 1 (gdn_osdn_precondition): the write keys and the final
    preconditioner against oracle.osdn_precondition, with and without the
    retention gate and an initial preconditioner, both dtypes and head sizes;
  * phase 2 (gdn_chunk_fwd_wk): o and the final state against
    oracle.recurrent_wk on the same (rounded) write keys, every gate kind,
    ragged tails, several waves, a GDN-sized workload;
  * both phases (osdn_chunk_fwd) against the oracle's two phases in fp64;
  * eta = 0 gives k_write = k and then the plain forward, to the bit.
Tolerance: max|x - x_ref| / max|x_ref| <= 1e-2 for bf16 inputs, 1e-4 for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import TOL, check, to_dev

pytestmark = pytest.mark.gpu


def retention(B, T, H, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.sigmoid(torch.randn(B, T, H, generator=gen) + 2.0).to(dtype)


def gpu_phase1(x, eta, r=None, d0=None):
    d = to_dev(x)
    kw = torch.full_like(d["k"], float("nan"))
    B, T, H, Dk = d["k"].shape
    d1 = torch.full((B, H, Dk), float("nan"), device="cuda")
    gdn.gdn_osdn_precondition(d["k"], d["beta"], None if r is None else r.cuda(), eta,
                              None if d0 is None else d0.cuda(), kw, d1)
    torch.cuda.synchronize()
    return kw, d1


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("Dk", [64, 128])
@pytest.mark.parametrize("with_r", [False, True])
def test_phase1_matches_oracle(dtype, Dk, with_r):
    x = gi.make_inputs(2, 300, 3, Dk, 16, dtype=dtype, gate="none", seed=21)
    r = retention(2, 300, 3, dtype, 22) if with_r else None
    d0 = None if not with_r else 0.5 + torch.rand(2, 3, Dk, generator=torch.Generator().manual_seed(23))
    kw, d1 = gpu_phase1(x, 0.7, r, d0)
    f = gi.to_f64_numpy(x)
    kw_ref, d_ref = oracle.osdn_precondition(
        f["k"], f["beta"], float(np.float32(0.7)),
        r=None if r is None else r.double().numpy(), d0=None if d0 is None else d0.double().numpy())
    check("k_write", kw, kw_ref, TOL[dtype])
    check("d_final", d1, d_ref, 1e-4 if dtype == torch.float32 else 1e-3)


@pytest.mark.parametrize("gate", ["none", "scalar", "per_dim"])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_phase2_matches_oracle(gate, T):
    x = gi.make_inputs(2, T, 3, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=0.05, seed=31)
    kw, _ = gpu_phase1(x, 0.7)
    d = to_dev(x)
    B, H = 2, 3
    o = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, H, 128, 128), float("nan"), device="cuda")
    nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, 128, 128, 64, torch.bfloat16, x["gate_kind"])
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    gdn.gdn_chunk_fwd_wk(d["q"], d["k"], kw, d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o,
                         S, workspace=ws)
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    o_ref, S_ref = oracle.recurrent_wk(f["q"], f["k"], kw.double().cpu().numpy(), f["v"],
                                       f["beta"], f["g"], x["gate_kind"], f["S0"])
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


@pytest.mark.parametrize("gate", ["scalar", "per_dim"])
def test_phase2_several_waves_small_workspace(gate):
    """A workspace of one chunk per wave: the write key is used in every wave."""
    x = gi.make_inputs(2, 700, 4, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=0.02, seed=41)
    kw, _ = gpu_phase1(x, 0.4)
    d = to_dev(x)
    B, T, H = 2, 700, 4
    least = gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, 128, 128, 64, torch.bfloat16,
                                                  x["gate_kind"])
    ws = torch.empty(least, dtype=torch.uint8, device="cuda")
    o = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(B, H, 128, 128, device="cuda")
    gdn.gdn_chunk_fwd_wk(d["q"], d["k"], kw, d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o,
                         S, workspace=ws)
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    o_ref, S_ref = oracle.recurrent_wk(f["q"], f["k"], kw.double().cpu().numpy(), f["v"],
                                       f["beta"], f["g"], x["gate_kind"], f["S0"])
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


def test_both_phases_gdn_workload_shape():
    """B4 H16 T2048 scalar gate (the GDN workload's shape) with the
    preconditioner and a retention gate, against the oracle's two phases in
    fp64 (the oracle's write keys are not rounded)."""
    w = gi.WORKLOADS[1]
    x = gi.workload_inputs(w)
    r = retention(w.B, w.T, w.H, torch.bfloat16, 51)
    d = to_dev(x)
    o, S, d1 = gdn.osdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], eta=0.5, r=r.cuda())
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    kw_ref, d_ref = oracle.osdn_precondition(f["k"], f["beta"], 0.5, r=r.double().numpy())
    o_ref, S_ref = oracle.recurrent_wk(f["q"], f["k"], kw_ref, f["v"], f["beta"], f["g"],
                                       x["gate_kind"], f["S0"])
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])
    check("d_final", d1, d_ref, 1e-3)
    assert gdn.gdn_read_device_status() == 0


@pytest.mark.parametrize("gate", ["none", "scalar", "per_dim"])
def test_eta_zero_is_the_plain_forward_bit_for_bit(gate):
    x = gi.make_inputs(2, 333, 3, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=0.05, seed=61)
    kw, d1 = gpu_phase1(x, 0.0)
    d = to_dev(x)
    assert torch.equal(kw, d["k"])
    assert torch.equal(d1, torch.ones_like(d1))
    B, T, H = 2, 333, 3
    nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, 128, 128, 64, torch.bfloat16, x["gate_kind"])
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    outs = []
    for key in (kw, None):
        o = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
        S = torch.empty(B, H, 128, 128, device="cuda")
        gdn.gdn_chunk_fwd_wk(d["q"], d["k"], key, d["v"], d["beta"], d["g"], x["gate_kind"],
                             d["S0"], o, S, workspace=ws)
        torch.cuda.synchronize()
        outs.append((o, S))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
