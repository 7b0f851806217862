"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.  Full-size workloads are compared in full where the
oracle finishes in seconds and on whole sampled heads / sequences otherwise;
small cases cover ragged tails, both head sizes, all gate kinds, optional and
aliased states, and the empty sequence."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_94_b200 as gdn
from gated_delta_rule_94_b200 import inputs as gi
from gpu_util import TOL, check, gpu_chunk, oracle_chunk, to_dev

pytestmark = pytest.mark.gpu

GATES = ["none", "scalar", "per_dim"]


# ------------------------------------------------------------ full workloads
def test_workload0_tiny_fp32():
    w = gi.WORKLOADS[0]
    x = gi.workload_inputs(w)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.float32])
    check("S", S, S_ref, TOL[torch.float32])


def test_workload1_gdn_bf16():
    w = gi.WORKLOADS[1]
    x = gi.workload_inputs(w)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


def test_workload2_kda_per_dim_bf16():
    w = gi.WORKLOADS[2]
    x = gi.workload_inputs(w)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


def test_workload3_long_sequence_sampled_heads():
    """All 32 heads run on the GPU; the oracle recomputes 4 whole heads (the
    first, one from each half of the grid, the last), every wave of each."""
    w = gi.WORKLOADS[3]
    x = gi.workload_inputs(w)
    o, S = gpu_chunk(x)
    heads = [0, 16, 29, 31]
    o_ref, S_ref = oracle_chunk(x, heads=heads)
    check("o", o[:, :, heads], o_ref, TOL[torch.bfloat16])
    check("S", S[:, heads], S_ref, TOL[torch.bfloat16])


def run_decode_steps(x, state):
    """Apply gdn_decode_step once per token of x (tokens along dim 1)."""
    d = to_dev(x)
    steps = d["q"].shape[1]
    outs = []
    for t in range(steps):
        g = None if d["g"] is None else d["g"][:, t].contiguous()
        o = gdn.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                            d["v"][:, t].contiguous(), d["beta"][:, t].contiguous(), g, state)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.stack(outs, dim=1)


def test_workload4_decode_128_steps_sampled_sequences():
    """256 sequences x 32 heads, 128 steps in place on the GPU; the oracle
    replays 12 whole sequences (all heads, all steps)."""
    w = gi.WORKLOADS[4]
    x = gi.workload_inputs(w)
    state = x["S0"].cuda()
    o = run_decode_steps(x, state)
    seqs = [0, 1, 77, 128, 200, 255, 3, 64, 99, 150, 180, 254]
    xs = {key: (val[seqs] if isinstance(val, torch.Tensor) else val) for key, val in x.items()}
    o_ref, S_ref = oracle_chunk(xs)
    check("o", o[seqs], o_ref, TOL[torch.bfloat16])
    check("S", state[seqs], S_ref, TOL[torch.bfloat16])


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 100, 200])
@pytest.mark.parametrize("dims", [(64, 64), (128, 128)])
def test_small_shapes(dtype, gate, T, dims):
    Dk, Dv = dims
    x = gi.make_inputs(2, T, 3, Dk, Dv, dtype=dtype, gate=gate, gate_scale=0.1,
                       s0_std=0.5 if T % 2 else None, seed=T + Dk)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[dtype])
    check("S", S, S_ref, TOL[dtype])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dims", [(64, 128), (128, 64)])
@pytest.mark.parametrize("gate", GATES)
def test_mixed_head_sizes(dtype, dims, gate):
    Dk, Dv = dims
    x = gi.make_inputs(1, 130, 2, Dk, Dv, dtype=dtype, gate=gate, s0_std=0.3, seed=5)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[dtype])
    check("S", S, S_ref, TOL[dtype])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_strong_decay_and_large_beta(dtype):
    """Fast forgetting (log a down to about -3 per token) and beta near 1:
    exercises the log-domain cumulation of the gates over a whole chunk."""
    x = gi.make_inputs(1, 192, 2, 128, 128, dtype=dtype, gate="per_dim", gate_scale=1.0,
                       s0_std=1.0, seed=9)
    x["beta"] = (x["beta"].float() * 0.1 + 0.9).to(dtype)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[dtype])
    check("S", S, S_ref, TOL[dtype])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_no_final_state_and_aliased_state(dtype):
    x = gi.make_inputs(2, 150, 2, 128, 128, dtype=dtype, gate="scalar", s0_std=0.5, seed=3)
    o_ref, S_ref = oracle_chunk(x)
    o, S = gpu_chunk(x, final=False)
    assert S is None
    check("o", o, o_ref, TOL[dtype])
    o2, S2 = gpu_chunk(x, alias=True)      # final state written over the initial state
    check("o aliased", o2, o_ref, TOL[dtype])
    check("S aliased", S2, S_ref, TOL[dtype])


def test_empty_sequence_copies_state():
    x = gi.make_inputs(2, 0, 2, 64, 64, dtype=torch.bfloat16, s0_std=0.5, seed=1)
    o, S = gpu_chunk(x)
    assert o.numel() == 0
    assert torch.equal(S.cpu(), x["S0"])
    x["S0"] = None
    o, S = gpu_chunk(x)
    assert torch.count_nonzero(S) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_deterministic(dtype):
    x = gi.make_inputs(2, 300, 4, 128, 128, dtype=dtype, gate="per_dim", s0_std=0.1, seed=4)
    o1, S1 = gpu_chunk(x)
    o2, S2 = gpu_chunk(x)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_steps_match_oracle_and_chunk(dtype, gate, dims):
    Dk, Dv = dims
    x = gi.make_inputs(5, 70, 3, Dk, Dv, dtype=dtype, gate=gate, s0_std=0.2, seed=Dk + Dv)
    state = x["S0"].cuda().clone()
    o = run_decode_steps(x, state)
    o_ref, S_ref = oracle_chunk(x)
    check("decode o", o, o_ref, TOL[dtype])
    check("decode S", state, S_ref, TOL[dtype])
    oc, Sc = gpu_chunk(x)     # the chunk path over the same tokens agrees too
    check("chunk o", oc, o_ref, TOL[dtype])
    check("chunk S", Sc, S_ref, TOL[dtype])


def test_device_status_clear():
    x = gi.make_inputs(1, 64, 1, 64, 64, dtype=torch.bfloat16, seed=0)
    gpu_chunk(x)
    assert gdn.gdn_read_device_status() == 0


@pytest.mark.parametrize("gate", ["per_dim", "scalar"])
def test_extreme_decay_exact_fallback(gate):
    """Log-decay of ~3.5 per token: the in-chunk decay range (~220) exceeds what
    the factorized exponentials can hold, so the per-dimension prep takes its
    exact CUDA-core path for A and P (and the scalar gate its per-element
    exponentials); the result must still match the oracle."""
    x = gi.make_inputs(2, 160, 2, 128, 128, dtype=torch.bfloat16, gate=gate, gate_scale=5.0,
                       s0_std=1.0, seed=21)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


@pytest.mark.parametrize("gate", ["per_dim", "scalar"])
def test_one_sided_decay_in_chunk(gate):
    """Every chunk decays by ~100 in its first half and not at all in its
    second: the whole-chunk range is moderate, but a half-chunk factor would
    leave the fp32 range, so the prep must take its exact path (a full chunk
    and the ragged tail both meet this)."""
    x = gi.make_inputs(1, 160, 2, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=1.0,
                       seed=23)
    g = x["g"]
    pos = torch.arange(160) % 64
    step = torch.where(pos < 32, torch.tensor(-3.2), torch.tensor(0.0))
    shape = [1, 160] + [1] * (g.dim() - 2)
    x["g"] = torch.broadcast_to(step.view(shape), g.shape).contiguous().to(g.dtype)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["scalar", "per_dim"])
def test_wave_length_follows_workspace_bit_exactly(gate):
    """The same forward with the least workspace (one chunk per wave), a middle
    size and the full-speed size: the waves differ, the results agree to the
    bit (the state between waves is carried in fp32), and the oracle agrees."""
    B, T, H, D = 2, 1000, 3, 128
    x = gi.make_inputs(B, T, H, D, D, dtype=torch.bfloat16, gate=gate, s0_std=0.02, seed=21)
    d = to_dev(x)
    least = gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, D, D, 64, torch.bfloat16, x["gate_kind"])
    full = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, D, D, 64, torch.bfloat16, x["gate_kind"])
    assert 0 < least < full
    outs = []
    for nbytes in (least, (least + full) // 2, full):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o = torch.full((B, T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        S = torch.full((B, H, D, D), float("nan"), device="cuda")
        gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"], o,
                          S, workspace=ws)
        torch.cuda.synchronize()
        outs.append((o.clone(), S.clone()))
    for o, S in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(S, outs[0][1])
    o_ref, S_ref = oracle_chunk(x)
    check("o", outs[0][0], o_ref, TOL[torch.bfloat16])
    check("S", outs[0][1], S_ref, TOL[torch.bfloat16])
    too_small = torch.empty(least - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError):
        gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], x["gate_kind"], d["S0"],
                          outs[0][0], None, workspace=too_small)
    assert gdn.gdn_read_device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("gate", ["scalar", "per_dim"])
def test_more_heads_than_sms(gate):
    """180 (batch, head) pairs: the chain grid has more CTAs than the GPU has
    SMs, so chain CTAs wait for SMs across waves; every output and state still
    matches the oracle."""
    x = gi.make_inputs(3, 200, 60, 128, 128, dtype=torch.bfloat16, gate=gate, s0_std=0.02, seed=23)
    o, S = gpu_chunk(x)
    o_ref, S_ref = oracle_chunk(x)
    check("o", o, o_ref, TOL[torch.bfloat16])
    check("S", S, S_ref, TOL[torch.bfloat16])
    assert gdn.gdn_read_device_status() == 0


@pytest.mark.gpu
def test_one_chunk_waves_with_many_heads():
    """3600 heads of one chunk: the images of one chunk of every head exceed a
    wave buffer's cap, so the forward runs with one-chunk waves; a workspace of
    the least size forces one-chunk waves on a longer sequence too."""
    x = gi.make_inputs(2, 64, 1800, 128, 128, dtype=torch.bfloat16, gate="scalar", seed=24)
    o, S = gpu_chunk(x)
    heads = [0, 911, 1799]
    f = gi.to_f64_numpy(x)
    q, k, v, beta, g = (f[n][:, :, heads] for n in ("q", "k", "v", "beta", "g"))
    o_ref, S_ref = oracle.recurrent(q, k, v, beta, g, x["gate_kind"], None)
    check("o (sampled heads)", o[:, :, heads], o_ref, TOL[torch.bfloat16])
    check("S (sampled heads)", S[:, heads], S_ref, TOL[torch.bfloat16])
    # a longer sequence with the least workspace (one chunk per wave) against the full one
    B, T, H, D = 2, 640, 100, 128
    y = gi.make_inputs(B, T, H, D, D, dtype=torch.bfloat16, gate="scalar", s0_std=0.02, seed=25)
    d = to_dev(y)
    outs = []
    for nbytes in (gdn.gdn_chunk_fwd_workspace_min_bytes(B, T, H, D, D, 64, torch.bfloat16, 1),
                   gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, D, D, 64, torch.bfloat16, 1)):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o2 = torch.full((B, T, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        S2 = torch.full((B, H, D, D), float("nan"), device="cuda")
        gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], y["gate_kind"], d["S0"], o2,
                          S2, workspace=ws)
        torch.cuda.synchronize()
        outs.append((o2, S2))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    o_ref2, S_ref2 = oracle_chunk(y, heads=[0, 57, 99])
    check("o (least workspace, sampled heads)", outs[0][0][:, :, [0, 57, 99]], o_ref2, TOL[torch.bfloat16])
    check("S (least workspace, sampled heads)", outs[0][1][:, [0, 57, 99]], S_ref2, TOL[torch.bfloat16])
    assert gdn.gdn_read_device_status() == 0
