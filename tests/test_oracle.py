"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle (and its two NumPy restatements) against something
other than itself: hand-worked values, closed forms, invariants and special
cases that reduce to a simpler operator.  Sources:
  "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
   Attention" sec. 1 (delta rule as online GD), sec. 2.2 (closed-form residual
   contraction), sec. 3 (gated Newton condition -> exact write);
  "Moonshot AI's New Attention Architecture: Key Innovations Explained" sec. 2
   (linear attention -> DeltaNet -> scalar gate -> per-dimension gate), sec. 3
   (chunkwise recurrence, causal Tril), sec. 4 (the evolution line).
"""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GATES = [oracle.GATE_NONE, oracle.GATE_SCALAR, oracle.GATE_PER_DIM]


def rand_case(B, T, H, Dk, Dv, gate, seed, s0=True, beta_range=(0.0, 1.0), unit_k=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk))
    k = rng.standard_normal((B, T, H, Dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, Dv))
    beta = rng.uniform(*beta_range, size=(B, T, H))
    if gate == oracle.GATE_SCALAR:
        g = -rng.uniform(0.0, 0.5, size=(B, T, H))
    elif gate == oracle.GATE_PER_DIM:
        g = -rng.uniform(0.0, 0.5, size=(B, T, H, Dk))
    else:
        g = None
    S0 = rng.standard_normal((B, H, Dk, Dv)) * 0.5 if s0 else None
    return q, k, v, beta, g, S0


def run_all(q, k, v, beta, g, gate, S0, C=4):
    return (oracle.recurrent(q, k, v, beta, g, gate, S0),
            oracle.brute_force(q, k, v, beta, g, gate, S0),
            oracle.chunk_form(q, k, v, beta, g, gate, S0, C=C))


# ---------------------------------------------------------------- hand-worked
def test_golden_hand_worked():
    with open(os.path.join(HERE, "golden", "hand_worked_d2.json")) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        T = len(case["beta"])
        q = np.array(case["q"], float).reshape(1, T, 1, 2)
        k = np.array(case["k"], float).reshape(1, T, 1, 2)
        v = np.array(case["v"], float).reshape(1, T, 1, 2)
        beta = np.array(case["beta"], float).reshape(1, T, 1)
        a = np.array(case["a"], float)
        if case["gate"] == "scalar":
            gate, g = oracle.GATE_SCALAR, np.log(a).reshape(1, T, 1)
        else:
            gate, g = oracle.GATE_PER_DIM, np.log(a).reshape(1, T, 1, 2)
        S0 = np.array(case["M0"], float).reshape(1, 1, 2, 2)
        for (o, M) in run_all(q, k, v, beta, g, gate, S0, C=2):
            np.testing.assert_allclose(o[0, :, 0], np.array(case["o"]), rtol=0, atol=1e-12)
            np.testing.assert_allclose(M[0, 0], np.array(case["M_final"]), rtol=0, atol=1e-12)


# ------------------------------------------------------------ closed forms
@pytest.mark.parametrize("gate", GATES)
def test_beta_zero_is_pure_decay(gate):
    """beta = 0: no write, no erase.  With a = 1 the state is unchanged and
    o_t = M0^T q_t; with a gate the state is the cumulative decay of M0."""
    q, k, v, beta, g, S0 = rand_case(2, 9, 3, 8, 6, gate, seed=11)
    beta[:] = 0.0
    o, M = oracle.recurrent(q, k, v, beta, g, gate, S0)
    B, T, H, Dk = q.shape
    for b in range(B):
        for h in range(H):
            logs = np.zeros(Dk)
            for t in range(T):
                if gate == oracle.GATE_SCALAR:
                    logs += g[b, t, h]
                elif gate == oracle.GATE_PER_DIM:
                    logs += g[b, t, h]
                Mt = np.exp(logs)[:, None] * S0[b, h]
                np.testing.assert_allclose(o[b, t, h], Mt.T @ q[b, t, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(M[b, h], np.exp(logs)[:, None] * S0[b, h], rtol=1e-12,
                                       atol=1e-14)


@pytest.mark.parametrize("gate", GATES)
def test_exact_write(gate):
    """beta = 1 and |k| = 1 erase the old association along k completely, so the
    post-update state recalls v_t for key k_t exactly: S_t k_t = v_t.  Querying
    with q_t = k_t makes that visible in the output: o_t = v_t for every t."""
    q, k, v, beta, g, S0 = rand_case(2, 12, 2, 16, 8, gate, seed=3)
    beta[:] = 1.0
    q = k.copy()
    for (o, _) in run_all(q, k, v, beta, g, gate, S0, C=5):
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("gate", GATES)
def test_residual_contraction(gate):
    """Closed form behind the OSDN hypergradient surrogate (d = 1): the new
    residual is the decayed state's residual times (1 - beta |k|^2):
    M_t^T k_t - v_t = (1 - beta_t |k_t|^2) (M'^T k_t - v_t), M' = Diag(a_t) M_{t-1}."""
    q, k, v, beta, g, S0 = rand_case(1, 10, 2, 12, 7, gate, seed=5, beta_range=(0.0, 2.0),
                                     unit_k=False)
    H = q.shape[2]
    for t in (1, 4, 9):
        _, M_prev = oracle.recurrent(q[:, :t], k[:, :t], v[:, :t], beta[:, :t],
                                     None if g is None else g[:, :t], gate, S0)
        _, M_t = oracle.recurrent(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], beta[:, :t + 1],
                                  None if g is None else g[:, :t + 1], gate, S0)
        for h in range(H):
            if gate == oracle.GATE_SCALAR:
                a = np.exp(g[0, t, h]) * np.ones(q.shape[-1])
            elif gate == oracle.GATE_PER_DIM:
                a = np.exp(g[0, t, h])
            else:
                a = np.ones(q.shape[-1])
            Mp = a[:, None] * M_prev[0, h]
            kt, vt, bt = k[0, t, h], v[0, t, h], beta[0, t, h]
            lhs = M_t[0, h].T @ kt - vt
            rhs = (1.0 - bt * kt @ kt) * (Mp.T @ kt - vt)
            np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("gate", [oracle.GATE_NONE, oracle.GATE_SCALAR])
def test_orthogonal_keys_reduce_to_linear_attention(gate):
    """With mutually orthogonal unit keys the erase term never touches earlier
    writes, so the operator is (decayed) vanilla linear attention:
    o_t = sum_{i<=t} beta_i exp(G_t - G_i) (k_i . q_t) v_i, S0 = 0."""
    rng = np.random.default_rng(7)
    Dk, Dv, T = 16, 5, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((Dk, Dk)))
    k = Qm[:, :T].T.reshape(1, T, 1, Dk)
    q = rng.standard_normal((1, T, 1, Dk))
    v = rng.standard_normal((1, T, 1, Dv))
    beta = rng.uniform(0.1, 1.0, size=(1, T, 1))
    g = -rng.uniform(0.0, 0.4, size=(1, T, 1)) if gate == oracle.GATE_SCALAR else None
    G = np.cumsum(g[0, :, 0]) if g is not None else np.zeros(T)
    expect = np.zeros((T, Dv))
    for t in range(T):
        for i in range(t + 1):
            expect[t] += beta[0, i, 0] * np.exp(G[t] - G[i]) * (k[0, i, 0] @ q[0, t, 0]) * v[0, i, 0]
    for (o, _) in run_all(q, k, v, beta, g, gate, None, C=5):
        np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- brute force
@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("d", [4, 8, 16])
@pytest.mark.parametrize("s0", [False, True])
def test_brute_force(gate, d, s0):
    q, k, v, beta, g, S0 = rand_case(2, 8, 2, d, d + 1, gate, seed=d + 100 * gate, s0=s0,
                                     unit_k=False)
    o, M = oracle.recurrent(q, k, v, beta, g, gate, S0)
    ob, Mb = oracle.brute_force(q, k, v, beta, g, gate, S0)
    assert oracle.rel_err(o, ob) < 1e-12
    assert oracle.rel_err(M, Mb) < 1e-12


# ---------------------------------------------------------------- reductions
def test_per_dim_with_equal_components_is_scalar_gate():
    q, k, v, beta, g, S0 = rand_case(2, 20, 2, 8, 8, oracle.GATE_SCALAR, seed=9)
    g_vec = np.repeat(g[..., None], 8, axis=-1)
    o1, M1 = oracle.recurrent(q, k, v, beta, g, oracle.GATE_SCALAR, S0)
    o2, M2 = oracle.recurrent(q, k, v, beta, g_vec, oracle.GATE_PER_DIM, S0)
    assert oracle.rel_err(o2, o1) < 1e-14 and oracle.rel_err(M2, M1) < 1e-14


def test_unit_gate_is_deltanet():
    q, k, v, beta, _, S0 = rand_case(2, 20, 2, 8, 8, oracle.GATE_NONE, seed=10)
    zeros = np.zeros(beta.shape)
    o1, M1 = oracle.recurrent(q, k, v, beta, None, oracle.GATE_NONE, S0)
    o2, M2 = oracle.recurrent(q, k, v, beta, zeros, oracle.GATE_SCALAR, S0)
    assert oracle.rel_err(o2, o1) == 0.0 and oracle.rel_err(M2, M1) == 0.0


# ------------------------------------------------------------------ structure
@pytest.mark.parametrize("gate", GATES)
def test_split_sequence_carry(gate):
    """Running T1 tokens, then T2 more from the carried state, equals one run
    of T1 + T2 tokens (the state is the whole memory)."""
    q, k, v, beta, g, S0 = rand_case(2, 30, 2, 8, 6, gate, seed=12)
    gsl = (lambda a, b: None) if g is None else (lambda a, b: g[:, a:b])
    o, M = oracle.recurrent(q, k, v, beta, g, gate, S0)
    oa, Ma = oracle.recurrent(q[:, :13], k[:, :13], v[:, :13], beta[:, :13], gsl(0, 13), gate, S0)
    ob, Mb = oracle.recurrent(q[:, 13:], k[:, 13:], v[:, 13:], beta[:, 13:], gsl(13, 30), gate, Ma)
    np.testing.assert_array_equal(np.concatenate([oa, ob], axis=1), o)
    np.testing.assert_array_equal(Mb, M)


@pytest.mark.parametrize("gate", GATES)
def test_a_run_of_tokens_maps_the_state_affinely(gate):
    """A run of tokens maps the entering state affinely, column by column:
    S_out[:, j] = A S_in[:, j] + b[:, j] with one Dk x Dk matrix A for every
    value column (each step is (Diag(a) - beta k k^T Diag(a)) applied to the
    state plus beta k v^T; "Moonshot AI's New Attention Architecture", sec. 3).
    Two runs compose as
    A2 (A1 S + b1) + b2, which is how the segment-parallel pass combines
    segment offsets b and transitions A."""
    B, T, H, Dk, Dv = 1, 24, 2, 6, 5
    q, k, v, beta, g, S0 = rand_case(B, T, H, Dk, Dv, gate, seed=31)
    gsl = (lambda a, b: None) if g is None else (lambda a, b: g[:, a:b])

    def run(a, b, S):
        return oracle.recurrent(q[:, a:b], k[:, a:b], v[:, a:b], beta[:, a:b], gsl(a, b), gate, S)[1]

    def transition(a, b):
        """A (per head, [H][Dk][Dk]) and b ([H][Dk][Dv]) of tokens a..b-1."""
        zero = np.zeros((B, H, Dk, Dv))
        off = run(a, b, zero)
        A = np.empty((H, Dk, Dk))
        for i in range(Dk):
            E = np.zeros((B, H, Dk, Dv))
            E[:, :, i, :] = 1.0                  # e_i in every value column
            cols = run(a, b, E) - off            # A e_i, the same in every column
            np.testing.assert_allclose(cols, cols[..., :1].repeat(Dv, axis=-1), rtol=0, atol=1e-12)
            A[:, :, i] = cols[0, :, :, 0]
        return A, off[0]

    A1, b1 = transition(0, 11)
    A2, b2 = transition(11, T)
    S_in = S0
    # the affine form reproduces each run and the whole sequence
    np.testing.assert_allclose(run(0, 11, S_in)[0], A1 @ S_in[0] + b1, rtol=0, atol=1e-11)
    whole = run(0, T, S_in)[0]
    np.testing.assert_allclose(whole, A2 @ (A1 @ S_in[0] + b1) + b2, rtol=0, atol=1e-11)
    np.testing.assert_allclose(whole, (A2 @ A1) @ S_in[0] + (A2 @ b1 + b2), rtol=0, atol=1e-11)
    # affine combinations of entering states are preserved
    S_alt = np.random.default_rng(5).standard_normal(S_in.shape)
    lam = 0.3
    mix = run(0, T, lam * S_in + (1 - lam) * S_alt)
    np.testing.assert_allclose(mix, lam * run(0, T, S_in) + (1 - lam) * run(0, T, S_alt),
                               rtol=0, atol=1e-11)


@pytest.mark.parametrize("gate", GATES)
def test_causality(gate):
    """Perturbing tokens after t leaves o_{<=t} unchanged."""
    q, k, v, beta, g, S0 = rand_case(1, 24, 2, 8, 8, gate, seed=13)
    o, _ = oracle.recurrent(q, k, v, beta, g, gate, S0)
    t = 10
    k2, v2, q2, b2 = k.copy(), v.copy(), q.copy(), beta.copy()
    k2[:, t + 1:] += 1.0
    v2[:, t + 1:] -= 2.0
    q2[:, t + 1:] *= 3.0
    b2[:, t + 1:] = 0.9
    for (oo, _) in [oracle.recurrent(q2, k2, v2, b2, g, gate, S0),
                    oracle.chunk_form(q2, k2, v2, b2, g, gate, S0, C=8)]:
        np.testing.assert_allclose(oo[:, :t + 1], o[:, :t + 1], rtol=0, atol=1e-13)
        assert np.max(np.abs(oo[:, t + 1:] - o[:, t + 1:])) > 1e-3


def test_contractivity_bound():
    """For beta in [0, 2] and |k| = 1, I - beta k k^T has spectral norm <= 1, so
    |M_t|_F <= max(a) |M_{t-1}|_F + beta |k| |v|."""
    q, k, v, beta, g, S0 = rand_case(1, 16, 1, 8, 8, oracle.GATE_PER_DIM, seed=14,
                                     beta_range=(0.0, 2.0))
    prev = S0[0, 0]
    for t in range(16):
        _, M = oracle.recurrent(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], beta[:, :t + 1],
                                g[:, :t + 1], oracle.GATE_PER_DIM, S0)
        bound = np.exp(g[0, t, 0]).max() * np.linalg.norm(prev) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert np.linalg.norm(M[0, 0]) <= bound * (1 + 1e-12)
        prev = M[0, 0]


# ---------------------------------------------------------------- chunk form
@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("C", [1, 2, 4, 8, 16, 32, 64])
def test_chunk_form_equals_recurrence(gate, C):
    """The chunkwise state recurrence and output equal the token recurrence for
    every chunk length, including a ragged last chunk (T = 100)."""
    q, k, v, beta, g, S0 = rand_case(1, 100, 2, 16, 12, gate, seed=20 + C)
    o, M = oracle.recurrent(q, k, v, beta, g, gate, S0)
    oc, Mc = oracle.chunk_form(q, k, v, beta, g, gate, S0, C=C)
    assert oracle.rel_err(oc, o) < 1e-12
    assert oracle.rel_err(Mc, M) < 1e-12


def test_forward_substitution_inverse():
    rng = np.random.default_rng(0)
    A = np.tril(rng.standard_normal((20, 20)) * 0.3, -1)
    Tm = oracle.forward_substitution_inverse(A)
    np.testing.assert_allclose((np.eye(20) + A) @ Tm, np.eye(20), atol=1e-12)


def test_empty_sequence():
    q, k, v, beta, g, S0 = rand_case(1, 0, 2, 4, 4, oracle.GATE_SCALAR, seed=1)
    o, M = oracle.recurrent(q, k, v, beta, g, oracle.GATE_SCALAR, S0)
    assert o.shape == (1, 0, 2, 4)
    np.testing.assert_array_equal(M, S0)


def test_planted_mistake_is_caught():
    """Sanity of the pins themselves: an oracle that decays after the erase
    (a plausible misreading of the per-dimension form) fails the hand-worked
    per-dimension case and the exact-write pin."""
    def wrong_order(q, k, v, beta, g, S0):
        B, T, H, Dk = q.shape
        o = np.zeros(v.shape)
        M = S0[0, 0].copy()
        for t in range(T):
            kt = k[0, t, 0]
            M = M - beta[0, t, 0] * np.outer(kt, kt @ M)
            M = np.exp(g[0, t, 0])[:, None] * M + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
            o[0, t, 0] = M.T @ q[0, t, 0]
        return o
    with open(os.path.join(HERE, "golden", "hand_worked_d2.json")) as f:
        case = json.load(f)["cases"][1]
    q = np.array(case["q"], float).reshape(1, 2, 1, 2)
    k = np.array(case["k"], float).reshape(1, 2, 1, 2)
    v = np.array(case["v"], float).reshape(1, 2, 1, 2)
    beta = np.array(case["beta"], float).reshape(1, 2, 1)
    g = np.log(np.array(case["a"], float)).reshape(1, 2, 1, 2)
    o = wrong_order(q, k, v, beta, g, np.zeros((1, 1, 2, 2)))
    assert np.max(np.abs(o[0, :, 0] - np.array(case["o"]))) > 1e-3


# ------------------------------------------------------------------ rel_err
# oracle.rel_err is the parity metric every GPU test and every oracle-vs-oracle
# comparison above uses: max|x - ref| / max|ref| over the whole tensor (the
# tolerance metric of the workloads: bf16 <= 1e-2, fp32 <= 1e-4).  The values
# below are worked by hand; each case is chosen so that one plausible slip in
# the metric changes its value.
REL_ERR_CASES = [
    # (x, ref, expected, what a wrong metric would give)
    ([1.0, -3.0], [2.0, -1.0], 1.0),           # |diff| = (1, 2): max 2; max|ref| = 2
    ([10.0, 0.0], [1.0, 0.0], 9.0),            # x larger than ref: den from x -> 0.9
    ([1.0, 1.0, 1.0, 5.0], [1.0, 1.0, 1.0, 1.0], 4.0),   # mean |diff| -> 1.0
    ([1.0, -5.0], [1.0, 1.0], 6.0),            # diff (0, -6): max without abs -> 0
    ([-4.0, 3.0], [-4.0, 1.0], 0.5),           # max ref without abs -> 1 -> 2.0
    ([[0.0, 2.0], [7.0, 1.0]], [[0.0, 2.0], [4.0, -8.0]], 9.0 / 8.0),  # 2-D, whole tensor
    ([0.0, 0.0], [0.0, 0.0], 0.0),             # both zero
]


@pytest.mark.parametrize("x,ref,expected", REL_ERR_CASES)
def test_rel_err_hand_worked(x, ref, expected):
    assert oracle.rel_err(np.array(x), np.array(ref)) == pytest.approx(expected, rel=1e-15)


def test_rel_err_zero_reference_reports_absolute_error():
    """With an all-zero reference there is no scale: the metric is the largest
    absolute deviation, so any nonzero output fails a tolerance of 1e-2."""
    assert oracle.rel_err(np.array([0.0, -0.5]), np.zeros(2)) == 0.5


def test_rel_err_planted_mistakes_fail_the_pins():
    """Each plausible slip in the metric fails at least one hand-worked case."""
    def denominator_from_x(x, ref):
        return np.max(np.abs(x - ref)) / np.max(np.abs(x))

    def mean_for_max(x, ref):
        return np.mean(np.abs(x - ref)) / np.max(np.abs(ref))

    def no_abs_numerator(x, ref):
        return np.max(x - ref) / np.max(np.abs(ref))

    def no_abs_denominator(x, ref):
        return np.max(np.abs(x - ref)) / np.max(ref)

    def per_row(x, ref):   # max over the last axis only, then the mean of rows
        return float(np.mean(np.max(np.abs(x - ref), -1) / np.max(np.abs(ref), -1)))

    for wrong in (denominator_from_x, mean_for_max, no_abs_numerator, no_abs_denominator,
                  per_row):
        failed = False
        for x, ref, expected in REL_ERR_CASES:
            if not np.any(ref):
                continue
            with np.errstate(all="ignore"):
                got = wrong(np.array(x, float), np.array(ref, float))
            if not np.isclose(got, expected, rtol=1e-12):
                failed = True
        assert failed, f"{wrong.__name__} passes every rel_err pin"
