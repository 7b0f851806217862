"""Shared helpers of the GPU parity tests: run the library and the oracle on
the same seeded inputs and compare with the operator's tolerance
(max|x - x_ref| / max|x_ref| <= 1e-2 for bf16 inputs, 1e-4 for fp32)."""
import numpy as np
import torch

import oracle
import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import inputs as gi

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def to_dev(x: dict, device="cuda") -> dict:
    return {key: (val.to(device) if isinstance(val, torch.Tensor) else val)
            for key, val in x.items()}


def gpu_chunk(x: dict, *, final=True, alias=False):
    d = to_dev(x)
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    o = torch.full((B, T, H, Dv), float("nan"), dtype=d["q"].dtype, device="cuda")
    S0 = d["S0"]
    if alias:
        S1 = S0
    else:
        S1 = torch.full((B, H, Dk, Dv), float("nan"), device="cuda") if final else None
    nws = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, d["q"].dtype, x["gate_kind"])
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda") if nws else None
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], S0, o, S1,
                      workspace=ws)
    torch.cuda.synchronize()
    return o, S1


def oracle_chunk(x: dict, heads=None):
    """fp64 oracle on the same (rounded) inputs, optionally on a subset of heads."""
    f = gi.to_f64_numpy(x)
    q, k, v, beta, g, S0 = f["q"], f["k"], f["v"], f["beta"], f["g"], f["S0"]
    if heads is not None:
        q, k, v, beta = q[:, :, heads], k[:, :, heads], v[:, :, heads], beta[:, :, heads]
        g = None if g is None else g[:, :, heads]
        S0 = None if S0 is None else S0[:, heads]
    return oracle.recurrent(q, k, v, beta, g, x["gate_kind"], S0)


def check(name, got, ref, tol):
    got = got.detach().to(torch.float64).cpu().numpy() if isinstance(got, torch.Tensor) else got
    err = oracle.rel_err(got, ref)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    assert err <= tol, f"{name}: rel err {err:.3e} > {tol:.0e}"
    return err
