"""GPU parity of the backward (gdn_chunk_bwd) against the fp64 oracle: the
gradients of L = sum(o * dO) + sum(S_T * dS) with respect to q, k, v, beta, g
and S0, on the same (bf16-rounded) inputs, computed by reverse-mode autograd
of the plain token loop (oracle.backward).  Tolerance as for the forward's
bf16 path: max|x - x_ref| / max|x_ref| <= 1e-2 per gradient."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import TOL, check, to_dev

pytestmark = pytest.mark.gpu


def run_case(B, T, H, gate, s0, ds, seed):
    x = gi.make_inputs(B, T, H, 128, 128, dtype=torch.bfloat16, gate=gate,
                       s0_std=0.05 if s0 else None, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1)
    dO = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    dS = (torch.randn(B, H, 128, 128, generator=gen) * 0.1) if ds else None
    d = to_dev(x)
    gr = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], dO.cuda(),
                       None if dS is None else dS.cuda())
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    ref = oracle.backward(f["q"], f["k"], f["v"], f["beta"], f["g"], x["gate_kind"], f["S0"],
                          dO.double().numpy(), None if dS is None else dS.double().numpy())
    return gr, ref


@pytest.mark.parametrize("gate", ["none", "scalar"])
@pytest.mark.parametrize("T", [1, 64, 100, 200])
def test_bwd_small_shapes(gate, T):
    gr, ref = run_case(1, T, 2, gate, s0=True, ds=True, seed=81)
    tol = TOL[torch.bfloat16]
    for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dbeta", "dbeta"),
                      ("d_initial_state", "dS0")):
        check(name, gr[name], ref[key], tol)
    if gate == "scalar":
        check("dg", gr["dg"], ref["dg"], tol)
    assert gdn.gdn_read_device_status() == 0


def test_bwd_several_chunks_without_states():
    gr, ref = run_case(2, 700, 3, "scalar", s0=False, ds=False, seed=82)
    tol = TOL[torch.bfloat16]
    for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dbeta", "dbeta"), ("dg", "dg"),
                      ("d_initial_state", "dS0")):
        check(name, gr[name], ref[key], tol)


def test_bwd_deterministic():
    x = gi.make_inputs(1, 300, 2, 128, 128, dtype=torch.bfloat16, gate="scalar", seed=83)
    d = to_dev(x)
    dO = torch.randn(1, 300, 2, 128, generator=torch.Generator().manual_seed(84)).to(
        torch.bfloat16).cuda()
    a = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], None, dO)
    b = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], None, dO)
    torch.cuda.synchronize()
    for key in ("dq", "dk", "dv", "dbeta", "dg", "d_initial_state"):
        # shared-memory atomics inside a chunk may reorder the sums of dG and
        # dbeta: equal to fp32 rounding (relative to the tensor's scale), not to
        # the bit (the first token's dg is a sum over the whole chunk that nearly
        # cancels)
        check(key, a[key], b[key].double().cpu().numpy(), 1e-5)


def test_bwd_gdn_workload_sampled_heads():
    """The bench's backward record, B4 H16 T2048 (scalar gate): every head runs
    on the GPU; two whole (sequence, head) pairs -- heads are independent --
    against the oracle's chunkwise backward (pinned to autograd of the token
    loop in test_backward_oracle)."""
    w = gi.WORKLOADS[1]
    x = gi.workload_inputs(w)
    gen = torch.Generator().manual_seed(11)
    dO = torch.randn(w.B, w.T, w.H, 128, generator=gen).to(torch.bfloat16)
    dS = 0.02 * torch.randn(w.B, w.H, 128, 128, generator=gen)
    d = to_dev(x)
    gr = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], dO.cuda(), dS.cuda())
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    tol = TOL[torch.bfloat16]
    for b, h in ((0, 0), (3, 15)):
        sl = lambda a: None if a is None else np.ascontiguousarray(a[b:b + 1, :, h:h + 1])
        ref = oracle.chunk_backward(sl(f["q"]), sl(f["k"]), sl(f["v"]), sl(f["beta"]), sl(f["g"]),
                                    x["gate_kind"], None, dO[b:b + 1, :, h:h + 1].double().numpy(),
                                    dS[b:b + 1, h:h + 1].double().numpy())
        for name, key in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dbeta", "dbeta"),
                          ("dg", "dg")):
            check(f"{name}[{b},{h}]", gr[name][b:b + 1, :, h:h + 1], ref[key], tol)
        check(f"dS0[{b},{h}]", gr["d_initial_state"][b:b + 1, h:h + 1], ref["dS0"], tol)
