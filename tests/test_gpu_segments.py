"""GPU parity of the segment-parallel state pass: with few (batch, head) pairs
and long sequences, the full-speed workspace splits each wave of every head
into segments -- their offsets and transitions from the chunk maps
h' = (Diag(gamma) + Phi) h + K~^T U, composed in fp32, then every segment run
from its entering state (the chunkwise state recurrence of "Moonshot AI's New
Attention Architecture: Key Innovations Explained", sec. 3, is affine in the
entering state).  Checked against the fp64 oracle for every gate kind, ragged
lengths, initial and final states, the write-key variant, and against the
plain chain (least workspace: one chunk per wave, no segments)."""
import pytest
import torch

import oracle
import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import TOL, check, oracle_chunk, to_dev

pytestmark = pytest.mark.gpu


def run(x, nbytes=None):
    d = to_dev(x)
    B, T, H, Dk = d["q"].shape
    Dv = d["v"].shape[-1]
    full = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, Dk, Dv, 64, d["q"].dtype, x["gate_kind"])
    ws = torch.empty(full if nbytes is None else nbytes, dtype=torch.uint8, device="cuda")
    o = torch.full((B, T, H, Dv), float("nan"), dtype=d["q"].dtype, device="cuda")
    S = torch.full((B, H, Dk, Dv), float("nan"), device="cuda")
    gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o, S,
                      workspace=ws)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("gate", ["none", "scalar", "per_dim"])
@pytest.mark.parametrize("T", [4096, 4000])
def test_segments_match_oracle(gate, T):
    x = gi.make_inputs(1, T, 2, 128, 128, dtype=torch.bfloat16, gate=gate,
                       gate_scale=0.05 if gate == "per_dim" else 0.1, s0_std=0.05, seed=71)
    plan = gdn.gdn_chunk_fwd_plan(1, T, 2, 128, 128, 64, torch.bfloat16, x["gate_kind"])
    assert plan["segments"] > 1        # the case exercises the segment path
    o, S = run(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])
    assert gdn.gdn_read_device_status() == 0


def test_segments_agree_with_the_plain_chain():
    """Full-speed workspace (segments) against the least workspace (one chunk per
    wave, the plain chain): different rounding, same result within tolerance."""
    x = gi.make_inputs(2, 6000, 2, 128, 128, dtype=torch.bfloat16, gate="scalar", s0_std=0.02,
                       seed=72)
    least = gdn.gdn_chunk_fwd_workspace_min_bytes(2, 6000, 2, 128, 128, 64, torch.bfloat16,
                                                  x["gate_kind"])
    assert gdn.gdn_chunk_fwd_plan(2, 6000, 2, 128, 128, 64, torch.bfloat16, x["gate_kind"],
                                  workspace_bytes=least)["segments"] == 1
    o1, S1 = run(x)
    o2, S2 = run(x, least)
    check("o", o1, o2.double().cpu().numpy(), TOL[torch.bfloat16])
    check("S", S1, S2.double().cpu().numpy(), TOL[torch.bfloat16])


def test_segments_with_write_key():
    x = gi.make_inputs(1, 4096, 2, 128, 128, dtype=torch.bfloat16, gate="scalar", s0_std=0.05,
                       seed=73)
    d = to_dev(x)
    o, S, _ = gdn.osdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], eta=0.5)
    torch.cuda.synchronize()
    f = gi.to_f64_numpy(x)
    kw_ref, _ = oracle.osdn_precondition(f["k"], f["beta"], 0.5)
    o_ref, S_ref = oracle.recurrent_wk(f["q"], f["k"], kw_ref, f["v"], f["beta"], f["g"],
                                       x["gate_kind"], f["S0"])
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


def test_segments_few_head_long_sequence_workload():
    """The bench's segment record, B1 H4 T65536 (scalar gate, the long-sequence
    recipe) with the full-speed workspace: three waves of 18 segments; every
    head against the oracle."""
    x = gi.make_inputs(1, 65536, 4, 128, 128, dtype=torch.bfloat16, gate="scalar", seed=0)
    plan = gdn.gdn_chunk_fwd_plan(1, 65536, 4, 128, 128, 64, torch.bfloat16, x["gate_kind"])
    assert plan["segments"] > 1 and plan["waves"] > 1
    o, S = run(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])
    assert gdn.gdn_read_device_status() == 0
