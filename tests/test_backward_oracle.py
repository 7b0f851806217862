"""Pins of the backward oracle.  The pages print no backward formula; the
gradient of the operator is the derivative of the forward recurrence, so:

  * oracle.backward (reverse-mode autograd of the fp64 token loop) is checked
    against central finite differences of oracle.recurrent -- the C forward,
    independent code -- along random directions in every input;
  * closed forms at beta = 0 (nothing is written: dk = dv = 0 and
    dq_t = (prod a) S0 do_t);
  * oracle.chunk_backward (the hand-derived chunkwise backward the GPU path
    follows) equals oracle.backward for every chunk length, gate kind, with and
    without the initial and final states.
"""
import numpy as np
import pytest

import oracle

GATES = [oracle.GATE_NONE, oracle.GATE_SCALAR, oracle.GATE_PER_DIM]


def case(B, T, H, Dk, Dv, gate, seed, s0=True, ds=True, beta=(0.1, 1.0)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    bt = rng.uniform(*beta, size=(B, T, H))
    g = (None if gate == oracle.GATE_NONE else -rng.uniform(0, 0.5, size=(B, T, H)) if
         gate == oracle.GATE_SCALAR else -rng.uniform(0, 0.5, size=(B, T, H, Dk)))
    S0 = rng.standard_normal((B, H, Dk, Dv)) if s0 else None
    do = rng.standard_normal((B, T, H, Dv))
    dS = rng.standard_normal((B, H, Dk, Dv)) if ds else None
    return dict(q=q, k=k, v=v, beta=bt, g=g, S0=S0), do, dS


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("s0,ds", [(True, True), (False, False), (True, False)])
def test_autograd_matches_finite_differences_of_the_c_forward(gate, s0, ds):
    x, do, dS = case(2, 9, 2, 5, 4, gate, seed=3, s0=s0, ds=ds)
    grads = oracle.backward(x["q"], x["k"], x["v"], x["beta"], x["g"], gate, x["S0"], do, dS)

    def loss(y):
        o, S = oracle.recurrent(y["q"], y["k"], y["v"], y["beta"], y["g"], gate, y["S0"])
        return float((o * do).sum() + (0.0 if dS is None else (S * dS).sum()))
    rng = np.random.default_rng(4)
    names = [n for n in ("q", "k", "v", "beta", "g", "S0") if x[n] is not None]
    for _ in range(3):
        dirs = {n: rng.standard_normal(x[n].shape) for n in names}
        eps = 1e-6
        lp = loss({**x, **{n: x[n] + eps * dirs[n] for n in names}})
        lm = loss({**x, **{n: x[n] - eps * dirs[n] for n in names}})
        fd = (lp - lm) / (2 * eps)
        key = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "g": "dg", "S0": "dS0"}
        an = sum(float((grads[key[n]] * dirs[n]).sum()) for n in names)
        assert an == pytest.approx(fd, rel=1e-7, abs=1e-8)


@pytest.mark.parametrize("gate", [oracle.GATE_NONE, oracle.GATE_SCALAR])
def test_beta_zero_closed_form(gate):
    """beta = 0 writes nothing: the state is the decayed S0, so dk = dv = 0 and
    dq_t = (prod_{s<=t} a_s) S0 do_t."""
    x, do, _ = case(1, 6, 2, 4, 3, gate, seed=5, beta=(0.0, 0.0))
    gr = oracle.backward(x["q"], x["k"], x["v"], x["beta"], x["g"], gate, x["S0"], do)
    np.testing.assert_array_equal(gr["dk"], 0.0)
    np.testing.assert_array_equal(gr["dv"], 0.0)
    G = np.zeros((1, 6, 2)) if gate == oracle.GATE_NONE else np.cumsum(x["g"], axis=1)
    for t in range(6):
        for h in range(2):
            want = np.exp(G[0, t, h]) * x["S0"][0, h] @ do[0, t, h]
            np.testing.assert_allclose(gr["dq"][0, t, h], want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunk_backward_equals_autograd(gate, C):
    x, do, dS = case(1, 70, 2, 6, 5, gate, seed=6)
    a = oracle.backward(x["q"], x["k"], x["v"], x["beta"], x["g"], gate, x["S0"], do, dS)
    c = oracle.chunk_backward(x["q"], x["k"], x["v"], x["beta"], x["g"], gate, x["S0"], do, dS,
                              C=C)
    for n in a:
        if a[n] is None:
            assert c[n] is None
            continue
        np.testing.assert_allclose(c[n], a[n], rtol=1e-10, atol=1e-11, err_msg=n)


def test_chunk_backward_without_states():
    x, do, _ = case(2, 40, 1, 4, 4, oracle.GATE_SCALAR, seed=7, s0=False, ds=False)
    a = oracle.backward(x["q"], x["k"], x["v"], x["beta"], x["g"], 1, None, do)
    c = oracle.chunk_backward(x["q"], x["k"], x["v"], x["beta"], x["g"], 1, None, do, C=16)
    for n in ("dq", "dk", "dv", "dbeta", "dg", "dS0"):
        np.testing.assert_allclose(c[n], a[n], rtol=1e-10, atol=1e-11, err_msg=n)
