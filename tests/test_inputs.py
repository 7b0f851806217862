"""The seeded input generator: shapes, ranges, determinism (CPU only)."""
import torch

from gated_delta_rule_94_b200 import inputs as gi


def test_shapes_and_ranges():
    x = gi.make_inputs(2, 33, 3, 16, 8, dtype=torch.float32, gate="per_dim", gate_scale=0.05,
                       s0_std=0.02, seed=0)
    assert x["q"].shape == (2, 33, 3, 16) and x["v"].shape == (2, 33, 3, 8)
    assert x["beta"].shape == (2, 33, 3) and x["g"].shape == (2, 33, 3, 16)
    assert x["S0"].shape == (2, 3, 16, 8) and x["S0"].dtype == torch.float32
    assert torch.allclose(x["k"].norm(dim=-1), torch.ones(2, 33, 3), atol=1e-5)
    assert torch.allclose(x["q"].norm(dim=-1), torch.ones(2, 33, 3), atol=1e-5)
    assert (x["beta"] > 0).all() and (x["beta"] < 1).all()
    assert (x["g"] <= 0).all()
    assert abs(float(x["S0"].std()) - 0.02) < 0.005


def test_deterministic_and_dtype():
    a = gi.make_inputs(1, 64, 2, 8, 8, dtype=torch.bfloat16, seed=5)
    b = gi.make_inputs(1, 64, 2, 8, 8, dtype=torch.bfloat16, seed=5)
    for key in ("q", "k", "v", "beta", "g"):
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    assert a["S0"] is None and a["gate_kind"] == gi.GATE_SCALAR


def test_workload_table():
    w = gi.WORKLOADS
    assert (w[1].B, w[1].H, w[1].T, w[1].Dk) == (4, 16, 2048, 128)
    assert w[2].gate == "per_dim" and w[2].s0_std == 0.02
    assert w[3].T == 65536 and w[4].kind == "decode"
    assert all(x.chunk == 64 for x in w.values())
