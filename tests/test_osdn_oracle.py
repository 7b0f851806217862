"""Pins of the OSDN part of the oracle ("OSDN: Improving Delta Rule with Provable
Online Preconditioning in Linear Attention", sec. 2.1-2.3, sec. 3) against
what the page fixes:

  * sec. 2.2: the surrogate h_t(d) = (f_t(S_t) - f_t(S_{t-1})) / |grad f_t|^2
    has the closed form ((1 - beta <d, k^2>)^2 - 1) / (2 |k|^2) -- checked by
    evaluating f before and after one step of the write-key recurrence;
  * sec. 2.2: Phase 1 is online gradient descent on h_t -- its step equals
    -eta grad h_t, the gradient taken by finite differences of the closed form,
    and the step lowers h_t;
  * sec. 3: the gated Newton condition beta <d, k^2> = 1 gives an exact write;
  * a repeated key drives beta <d, k^2> to 1 geometrically (closed form);
  * sec. 2.3: the retention gate scales d before the step (r = 0: only the
    step remains);
  * eta = 0 with d = 1 is the plain delta rule; the brute-force products and
    the chunk form with a write key equal the write-key recurrence.
"""
import numpy as np
import pytest

import oracle

GATES = [oracle.GATE_NONE, oracle.GATE_SCALAR, oracle.GATE_PER_DIM]


def rand_case(B, T, H, Dk, Dv, gate, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    beta = rng.uniform(0.1, 1.0, size=(B, T, H))
    if gate == oracle.GATE_SCALAR:
        g = -rng.uniform(0.0, 0.5, size=(B, T, H))
    elif gate == oracle.GATE_PER_DIM:
        g = -rng.uniform(0.0, 0.5, size=(B, T, H, Dk))
    else:
        g = None
    S0 = rng.standard_normal((B, H, Dk, Dv)) * 0.5
    kw = k * rng.uniform(0.5, 1.5, size=(B, T, H, Dk))
    return q, k, kw, v, beta, g, S0


def test_surrogate_closed_form_is_the_loss_ratio():
    """(f(S_t) - f(S_{t-1})) / |grad f(S_{t-1})|^2 after one write-key step
    equals the page's closed form, for random states, keys, values, beta, d."""
    rng = np.random.default_rng(3)
    for _ in range(20):
        Dk, Dv = 6, 5
        M = rng.standard_normal((Dk, Dv))          # M = S^T
        k = rng.standard_normal(Dk)
        v = rng.standard_normal(Dv)
        beta = rng.uniform(0.05, 1.5)
        d = rng.uniform(0.2, 2.0, Dk)
        f_before = 0.5 * np.sum((M.T @ k - v) ** 2)
        grad_sq = np.sum((M.T @ k - v) ** 2) * np.dot(k, k)   # |(Sk - v) k^T|_F^2
        _, M1 = oracle.recurrent_wk(k[None, None, None], k[None, None, None],
                                    (d * k)[None, None, None], v[None, None, None],
                                    np.array([[[beta]]]), None, oracle.GATE_NONE,
                                    M[None, None])
        f_after = 0.5 * np.sum((M1[0, 0].T @ k - v) ** 2)
        assert (f_after - f_before) / grad_sq == pytest.approx(
            oracle.osdn_surrogate(d, k, beta), rel=1e-10, abs=1e-12)


@pytest.mark.parametrize("gate", GATES)
def test_residual_contraction_with_write_key(gate):
    """|M_t^T k_t - v_t| = |1 - beta_t <d_t, k_t^2>| |M'^T k_t - v_t| with M' the
    decayed state (the exact-quadratic identity behind sec. 2.2)."""
    q, k, _, v, beta, g, S0 = rand_case(1, 6, 1, 5, 4, gate, seed=5)
    rng = np.random.default_rng(6)
    d = rng.uniform(0.3, 1.7, size=k.shape)
    kw = d * k
    M = S0[0, 0].copy()
    for t in range(6):
        a = (np.ones(5) if gate == oracle.GATE_NONE else
             np.full(5, np.exp(g[0, t, 0])) if gate == oracle.GATE_SCALAR else np.exp(g[0, t, 0]))
        Md = a[:, None] * M
        before = np.linalg.norm(Md.T @ k[0, t, 0] - v[0, t, 0])
        _, Mn = oracle.recurrent_wk(q[:, t:t + 1], k[:, t:t + 1], kw[:, t:t + 1], v[:, t:t + 1],
                                    beta[:, t:t + 1], None if g is None else g[:, t:t + 1], gate,
                                    M[None, None])
        M = Mn[0, 0]
        after = np.linalg.norm(M.T @ k[0, t, 0] - v[0, t, 0])
        ratio = abs(1 - beta[0, t, 0] * np.dot(d[0, t, 0], k[0, t, 0] ** 2))
        assert after == pytest.approx(ratio * before, rel=1e-9, abs=1e-12)


@pytest.mark.parametrize("gate", GATES)
def test_gated_newton_condition_writes_exactly(gate):
    """beta <d, k^2> = 1 (sec. 3) makes the step an exact write: M_t^T k_t = v_t."""
    q, k, _, v, beta, g, S0 = rand_case(1, 5, 2, 6, 3, gate, seed=8)
    rng = np.random.default_rng(9)
    d = rng.uniform(0.5, 1.5, size=k.shape)
    d /= (beta[..., None] * np.sum(d * k * k, -1, keepdims=True))   # beta <d, k^2> = 1
    for t in range(5):
        o, M = oracle.recurrent_wk(q[:, :t + 1], k[:, :t + 1], (d * k)[:, :t + 1],
                                   v[:, :t + 1], beta[:, :t + 1],
                                   None if g is None else g[:, :t + 1], gate, S0)
        for h in range(2):
            np.testing.assert_allclose(M[0, h].T @ k[0, t, h], v[0, t, h], atol=1e-11)


def test_phase1_step_is_gradient_descent_on_the_surrogate():
    """d_{t+1} - r_t d_t = -eta grad h_t(d_t), grad by central differences of
    the closed form; and for a small eta the step lowers h_t."""
    rng = np.random.default_rng(11)
    B, T, H, Dk = 1, 6, 2, 5
    k = rng.standard_normal((B, T, H, Dk))
    beta = rng.uniform(0.2, 1.0, size=(B, T, H))
    r = rng.uniform(0.5, 1.0, size=(B, T, H))
    eta = 0.3
    kw, dT = oracle.osdn_precondition(k, beta, eta, r=r)
    d = np.ones((B, H, Dk))
    for t in range(T):
        d_t = kw[:, t] / k[:, t]
        np.testing.assert_allclose(d_t, d, rtol=1e-12)
        d_next = (oracle.osdn_precondition(k[:, :t + 1], beta[:, :t + 1], eta, r=r[:, :t + 1])[1])
        for h in range(H):
            eps = 1e-6
            grad = np.array([(oracle.osdn_surrogate(d[0, h] + eps * e, k[0, t, h], beta[0, t, h]) -
                              oracle.osdn_surrogate(d[0, h] - eps * e, k[0, t, h], beta[0, t, h]))
                             / (2 * eps) for e in np.eye(Dk)])
            np.testing.assert_allclose(d_next[0, h] - r[0, t, h] * d[0, h], -eta * grad,
                                       rtol=1e-6, atol=1e-9)
            small = oracle.osdn_precondition(k[:, t:t + 1], beta[:, t:t + 1], 1e-3,
                                             d0=d[:, :])[1][0, h]
            assert (oracle.osdn_surrogate(small, k[0, t, h], beta[0, t, h]) <=
                    oracle.osdn_surrogate(d[0, h], k[0, t, h], beta[0, t, h]) + 1e-15)
        d = d_next
    np.testing.assert_allclose(d, dT, rtol=1e-12)


def test_phase1_repeated_key_closed_form():
    """One key repeated with fixed beta and r = 1: s_t = beta <d_t, k^2> obeys
    1 - s_{t+1} = (1 - c)(1 - s_t), c = eta beta^2 |k^2|^2 / |k|^2, so s_t -> 1
    (the gated Newton condition); d_t = 1 + alpha_t k^2 with
    alpha_t = (eta beta / |k|^2) (1 - s_1) (1 - (1 - c)^(t-1)) / c."""
    rng = np.random.default_rng(12)
    Dk, T, beta, eta = 8, 40, 0.7, 0.5
    kv = rng.standard_normal(Dk)
    k = np.tile(kv, (1, T, 1, 1))
    u = kv * kv
    n = np.dot(kv, kv)
    c = eta * beta ** 2 * np.dot(u, u) / n
    s1 = beta * n
    kw, dT = oracle.osdn_precondition(k, np.full((1, T, 1), beta), eta)
    for t in range(1, T + 1):
        d_t = kw[0, t - 1, 0] / kv
        alpha = (eta * beta / n) * (1 - s1) * (1 - (1 - c) ** (t - 1)) / c
        np.testing.assert_allclose(d_t, 1 + alpha * u, rtol=1e-10)
        s_t = beta * np.dot(d_t, u)
        assert 1 - s_t == pytest.approx((1 - c) ** (t - 1) * (1 - s1), rel=1e-9, abs=1e-13)
    assert abs(1 - beta * np.dot(dT[0, 0], u)) < abs(1 - s1) * 1e-3


def test_phase1_planted_ascent_fails_the_closed_form():
    """An ascending step (+eta grad h, the sign the APF line prints) does not
    drive beta <d, k^2> to 1 on a repeated key: the reading is pinned."""
    rng = np.random.default_rng(13)
    kv = rng.standard_normal(8)
    beta, eta = 0.7, 0.5
    d = np.ones(8)
    for _ in range(40):
        u = kv * kv
        s = beta * np.dot(d, u)
        d = d - eta * beta * (1 - beta * s) * u / np.dot(kv, kv)   # ascent
    assert abs(1 - beta * np.dot(d, kv * kv)) > abs(1 - beta * np.dot(kv, kv))


def test_phase1_retention_zero_keeps_only_the_step():
    """r = 0 forgets d entirely: d_{t+1} is the step term alone,
    eta beta_t (1 - beta_t <d_t, k_t^2>) k_t^2 / |k_t|^2."""
    rng = np.random.default_rng(14)
    k = rng.standard_normal((1, 3, 1, 4))
    beta = rng.uniform(0.2, 1.0, size=(1, 3, 1))
    eta = 0.4
    _, d = oracle.osdn_precondition(k, beta, eta, r=np.zeros((1, 3, 1)))
    _, d_prev = oracle.osdn_precondition(k[:, :2], beta[:, :2], eta, r=np.zeros((1, 2, 1)))
    u = k[0, 2, 0] ** 2
    s = beta[0, 2, 0] * np.dot(d_prev[0, 0], u)
    np.testing.assert_allclose(d[0, 0], eta * beta[0, 2, 0] * (1 - s) * u / np.dot(k[0, 2, 0], k[0, 2, 0]),
                               rtol=1e-12)


def test_phase1_zero_key_leaves_d_unchanged():
    k = np.zeros((1, 2, 1, 4))
    kw, d = oracle.osdn_precondition(k, np.full((1, 2, 1), 0.5), 0.3)
    np.testing.assert_array_equal(d, np.ones((1, 1, 4)))
    np.testing.assert_array_equal(kw, 0.0)


@pytest.mark.parametrize("gate", GATES)
def test_eta_zero_is_the_plain_delta_rule(gate):
    q, k, _, v, beta, g, S0 = rand_case(2, 9, 2, 6, 5, gate, seed=15)
    kw, d = oracle.osdn_precondition(k, beta, 0.0)
    np.testing.assert_array_equal(kw, k)
    o1, M1 = oracle.recurrent_wk(q, k, kw, v, beta, g, gate, S0)
    o2, M2 = oracle.recurrent(q, k, v, beta, g, gate, S0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(M1, M2)


@pytest.mark.parametrize("gate", GATES)
def test_write_key_brute_force(gate):
    q, k, kw, v, beta, g, S0 = rand_case(1, 7, 2, 5, 4, gate, seed=16)
    o1, M1 = oracle.recurrent_wk(q, k, kw, v, beta, g, gate, S0)
    o2, M2 = oracle.brute_force(q, k, v, beta, g, gate, S0, kw=kw)
    np.testing.assert_allclose(o1, o2, atol=1e-11)
    np.testing.assert_allclose(M1, M2, atol=1e-11)


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_write_key_chunk_form(gate, C):
    q, k, kw, v, beta, g, S0 = rand_case(1, 70, 2, 8, 6, gate, seed=17)
    o1, M1 = oracle.recurrent_wk(q, k, kw, v, beta, g, gate, S0)
    o2, M2 = oracle.chunk_form(q, k, v, beta, g, gate, S0, C=C, kw=kw)
    np.testing.assert_allclose(o1, o2, atol=1e-9)
    np.testing.assert_allclose(M1, M2, atol=1e-9)


def test_planted_write_with_read_key_fails():
    """Writing along k instead of kw (a plausible slip in Phase 2) fails the
    surrogate identity."""
    rng = np.random.default_rng(18)
    M = rng.standard_normal((4, 3))
    k = rng.standard_normal(4)
    v = rng.standard_normal(3)
    beta, d = 0.8, rng.uniform(0.3, 2.0, 4)
    r = beta * (v - M.T @ k)
    M_wrong = M + np.outer(k, r)                 # write key ignored
    f0 = 0.5 * np.sum((M.T @ k - v) ** 2)
    f1 = 0.5 * np.sum((M_wrong.T @ k - v) ** 2)
    ratio = (f1 - f0) / (np.sum((M.T @ k - v) ** 2) * np.dot(k, k))
    assert abs(ratio - oracle.osdn_surrogate(d, k, beta)) > 1e-3
