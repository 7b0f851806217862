"""CPU oracle for the gated delta rule (fp64).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm are the only callers.  Nothing here is
imported by the CUDA path, and nothing here imports it.

Three independent restatements of what the operator computes:

* :func:`recurrent` -- the plain token-by-token recurrence in C (fp64,
  OpenMP over (batch, head)), ``gdn_oracle.c``.  This is the oracle proper.
  Sources: the delta rule as online gradient descent ("OSDN: Improving Delta
  Rule with Provable Online Preconditioning in Linear Attention", sec. 1), and
  the scalar / per-dimension gated forms ("Moonshot AI's New Attention
  Architecture: Key Innovations Explained", sec. 2 Core Operator).
* :func:`brute_force` -- NumPy, the state written out as explicit products of
  d_k x d_k transition matrices, in the pages' S = M^T orientation; tiny T only.
* :func:`chunk_form` -- NumPy fp64 restatement of the chunkwise state
  recurrence and output ("Moonshot AI's New Attention Architecture", sec. 3
  Hardware-Friendly Algorithm) with the UT/WY factors T = (I + A)^-1,
  W = T diag(beta) K_bar, U = T diag(beta) V obtained by forward substitution
  ("OSDN ...", sec. 2.1: the chunk Gram matrix and the WY pipeline).

And the preconditioned variant ("OSDN ...", sec. 2.1-2.3), in two phases:

* :func:`osdn_precondition` -- Phase 1, the O(d_k) scan over the key stream:
  the diagonal preconditioner d_t, updated by online gradient descent on the
  closed-form surrogate h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1) / (2 |k_t|^2)
  (sec. 2.2), with the retention gate r_t of adaptive preconditioner forgetting
  (sec. 2.3), and the write keys kw_t = d_t (.) k_t;
* :func:`recurrent_wk` -- Phase 2, the recurrence with the write key kw_t in
  place of k_t in the write (sec. 2.1); :func:`brute_force` and
  :func:`chunk_form` take the same optional ``kw``.

Readings taken where the pages are garbled or silent (each is pinned by a test
in tests/test_oracle.py):
  * orientation: S_t k_t = v_t after an exact write, so in M = S^T form
    M_t = (I - b k k^T) Diag(a) M_{t-1} + b k v^T and o_t = M_t^T q_t;
  * per-dimension decay acts before the erase (Diag(a_t) next to S_{t-1});
  * the output uses the post-update state, so the intra-chunk mask is
    inclusive of the diagonal;
  * the query in the chunk output is scaled by the decay from the chunk start
    to its own position (Gamma_r), the key of the state update by the decay
    from its position to the chunk end (Gamma_C / Gamma_i);
  * g = log a is the gate input, cumulated in the log domain;
  * no 1/sqrt(d) scale on q; q and k are used as given;
  * OSDN: the preconditioner step descends the surrogate (the page's APF line
    prints "+ eta grad h"; the text calls the update online gradient descent
    on h_t, so the step is -eta grad h); d_1 = 1 unless given (the identity
    preconditioner, so the first token is a plain delta-rule step); no
    projection of d; k_t^2 is elementwise; the write key of token t uses d_t,
    the preconditioner before token t's own feedback; a token with k_t = 0
    leaves d unchanged (its surrogate has no direction); with gates the decay
    acts before the erase exactly as in the plain rule.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

GATE_NONE, GATE_SCALAR, GATE_PER_DIM = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c (gcc, -O2, OpenMP, no fast-math) into _build/."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off",
                               "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_recurrent.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, dp, dp, dp,
                                             ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                             ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.gdn_oracle_recurrent.restype = ctypes.c_int
        lib.gdn_oracle_recurrent_wk.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int, dp, dp, dp,
                                                ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                                ctypes.c_long, ctypes.c_long, ctypes.c_int]
        lib.gdn_oracle_recurrent_wk.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return os.cpu_count() or 1


def recurrent(q, k, v, beta, g, gate_kind, S0=None, threads: int | None = None):
    """Token-by-token recurrence in fp64.

    q, k: [B, T, H, Dk]; v: [B, T, H, Dv]; beta: [B, T, H];
    g = log a: [B, T, H] (scalar gate) or [B, T, H, Dk] (per-dimension) or None;
    S0: [B, H, Dk, Dv] (M = S^T) or None.  Returns (o [B,T,H,Dv], S [B,H,Dk,Dv]).
    """
    q, k, v, beta, g, S0 = map(_f64, (q, k, v, beta, g, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if gate_kind == GATE_NONE:
        g = None
    o = np.empty((B, T, H, Dv), np.float64)
    S = np.empty((B, H, Dk, Dv), np.float64)
    rc = _load().gdn_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g),
                                      int(gate_kind), _ptr(S0), _ptr(o), _ptr(S),
                                      B, T, H, Dk, Dv, int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_recurrent failed with code {rc}")
    return o, S


def recurrent_wk(q, k, kw, v, beta, g, gate_kind, S0=None, threads: int | None = None):
    """The recurrence with a separate write key (OSDN Phase 2), fp64:
    per token M <- Diag(a) M; r = beta (v - M^T k); M <- M + kw r^T; o = M^T q.
    kw: [B, T, H, Dk].  Returns (o, S) as :func:`recurrent`."""
    q, k, kw, v, beta, g, S0 = map(_f64, (q, k, kw, v, beta, g, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if gate_kind == GATE_NONE:
        g = None
    o = np.empty((B, T, H, Dv), np.float64)
    S = np.empty((B, H, Dk, Dv), np.float64)
    rc = _load().gdn_oracle_recurrent_wk(_ptr(q), _ptr(k), _ptr(kw), _ptr(v), _ptr(beta),
                                         _ptr(g), int(gate_kind), _ptr(S0), _ptr(o), _ptr(S),
                                         B, T, H, Dk, Dv, int(threads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_recurrent_wk failed with code {rc}")
    return o, S


def osdn_surrogate(d, k, beta):
    """h_t(d) = ((1 - beta <d, k^2>)^2 - 1) / (2 |k|^2), the closed form of
    (f_t(S_t) - f_t(S_{t-1})) / |grad f_t(S_{t-1})|_F^2 for the
    right-preconditioned step ("OSDN ...", sec. 2.2)."""
    d, k = np.asarray(d, np.float64), np.asarray(k, np.float64)
    s = beta * np.dot(d, k * k)
    return ((1.0 - s) ** 2 - 1.0) / (2.0 * np.dot(k, k))


def osdn_precondition(k, beta, eta, r=None, d0=None):
    """Phase 1 of OSDN, fp64, token by token for every (batch, head):

        kw_t    = d_t (.) k_t                        (the write key of token t)
        grad    = -beta_t (1 - beta_t <d_t, k_t^2>) k_t^2 / |k_t|^2
                                                     (= grad_d h_t(d_t))
        d_{t+1} = r_t d_t - eta grad

    ("OSDN ...", sec. 2.1 the preconditioned key, sec. 2.2 the surrogate and
    its online gradient step, sec. 2.3 the retention gate r_t; r = None means
    r_t = 1, no forgetting).  k: [B, T, H, Dk]; beta, r: [B, T, H]; d0:
    [B, H, Dk] or None (ones).  Returns (kw [B, T, H, Dk], d_final [B, H, Dk]).
    """
    k = np.asarray(k, np.float64)
    beta = np.asarray(beta, np.float64)
    B, T, H, Dk = k.shape
    d = np.ones((B, H, Dk)) if d0 is None else np.array(d0, np.float64, copy=True)
    kw = np.empty_like(k)
    for t in range(T):
        kt = k[:, t]                                   # [B, H, Dk]
        u = kt * kt
        n = u.sum(-1)                                  # |k_t|^2
        s = (d * u).sum(-1)                            # <d_t, k_t^2>
        bt = beta[:, t]
        kw[:, t] = d * kt
        with np.errstate(divide="ignore", invalid="ignore"):
            step = np.where(n > 0, eta * bt * (1.0 - bt * s) / np.where(n > 0, n, 1.0), 0.0)
        rt = 1.0 if r is None else np.asarray(r, np.float64)[:, t][..., None]
        d = rt * d + step[..., None] * u
    return kw, d


def _decay_vector(g, gate_kind, b, t, h, Dk):
    if gate_kind == GATE_NONE:
        return np.ones(Dk)
    if gate_kind == GATE_SCALAR:
        return np.full(Dk, np.exp(g[b, t, h]))
    return np.exp(g[b, t, h])


def brute_force(q, k, v, beta, g, gate_kind, S0=None, kw=None):
    """Explicit-product expansion of the recurrence, in the S (d_v x d_k) form.

    With E_t = Diag(a_t) (I - beta_t k_t kw_t^T) (a d_k x d_k matrix; scalar gate:
    Diag(a_t) = a_t I; kw = k unless a write key is given), the recurrence
    S_t = S_{t-1} E_t + beta_t v_t kw_t^T gives
        S_t = S_0 E_1 ... E_t + sum_{i<=t} beta_i v_i kw_i^T E_{i+1} ... E_t,
    evaluated here literally for every t; o_t = S_t q_t.  Meant for T <= 8.
    Returns (o [B,T,H,Dv], M_final = S_T^T [B,H,Dk,Dv]).
    """
    q, k, v, beta, g, S0, kw = map(_f64, (q, k, v, beta, g, S0, kw))
    if kw is None:
        kw = k
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((B, T, H, Dv))
    M_final = np.zeros((B, H, Dk, Dv))
    I = np.eye(Dk)
    for b in range(B):
        for h in range(H):
            E = []
            for t in range(T):
                kt = k[b, t, h][:, None]
                kwt = kw[b, t, h][:, None]
                a = _decay_vector(g, gate_kind, b, t, h, Dk)
                E.append(np.diag(a) @ (I - beta[b, t, h] * (kt @ kwt.T)))
            for t in range(T):
                prod = I.copy()
                for s in range(t + 1):
                    prod = prod @ E[s]
                S_t = (np.zeros((Dv, Dk)) if S0 is None else S0[b, h].T) @ prod
                for i in range(t + 1):
                    tail = I.copy()
                    for s in range(i + 1, t + 1):
                        tail = tail @ E[s]
                    S_t = S_t + beta[b, i, h] * (v[b, i, h][:, None] @ kw[b, i, h][None, :]) @ tail
                o[b, t, h] = S_t @ q[b, t, h]
                if t == T - 1:
                    M_final[b, h] = S_t.T
            if T == 0:
                M_final[b, h] = 0 if S0 is None else S0[b, h]
    return o, M_final


def forward_substitution_inverse(A):
    """T = (I + A)^{-1} for strictly lower-triangular A, row by row:
    row r of (I + A) T = I gives T_r = e_r - sum_{i<r} A_ri T_i."""
    n = A.shape[0]
    Tm = np.zeros_like(A)
    for r in range(n):
        row = np.zeros(n)
        row[r] = 1.0
        for i in range(r):
            row -= A[r, i] * Tm[i]
        Tm[r] = row
    return Tm


def chunk_form(q, k, v, beta, g, gate_kind, S0=None, C: int = 64, kw=None):
    """Chunkwise evaluation (fp64) of the same operator, chunk length C.

    Per chunk, with h the entering M (= S^T, d_k x d_v), G_r = sum_{i<=r} log a_i
    (within the chunk, per key dimension), Gamma_r = exp(G_r):
      A   = StrictTril(diag(beta) (K_bar K_breve^T)), where
            (K_bar K_breve^T)_ri = sum_d k_rd k_id exp(G_rd - G_id)
      T   = (I + A)^{-1}                      (forward substitution)
      W   = T diag(beta) K_bar,  U = T diag(beta) V,   K_bar = Gamma * K
      D   = U - W h                            (the chunk's pseudo-values)
      O   = Q_bar h + Tril_incl(Q_bar K_breve^T) D,   Q_bar = Gamma * Q
      h'  = Diag(gamma_C) h + K_tilde^T D,  K_tilde_i = k_i * Gamma_C / Gamma_i
    The last chunk may be shorter than C.  With a write key kw (OSDN), kw
    replaces k in K_breve (the Gram matrix and the intra-chunk scores) and in
    K_tilde (the state update); the read key k stays in K_bar (sec. 2.1 of the
    OSDN page).  Returns (o, M_final).
    """
    q, k, v, beta, g, S0, kw = map(_f64, (q, k, v, beta, g, S0, kw))
    if kw is None:
        kw = k
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((B, T, H, Dv))
    M_final = np.zeros((B, H, Dk, Dv))
    for b in range(B):
        for h_ in range(H):
            h = np.zeros((Dk, Dv)) if S0 is None else S0[b, h_].copy()
            for c0 in range(0, T, C):
                c1 = min(T, c0 + C)
                n = c1 - c0
                Q = q[b, c0:c1, h_]
                K = k[b, c0:c1, h_]
                KW = kw[b, c0:c1, h_]
                V = v[b, c0:c1, h_]
                bt = beta[b, c0:c1, h_]
                if gate_kind == GATE_NONE:
                    logs = np.zeros((n, Dk))
                elif gate_kind == GATE_SCALAR:
                    logs = np.repeat(g[b, c0:c1, h_][:, None], Dk, axis=1)
                else:
                    logs = g[b, c0:c1, h_]
                G = np.cumsum(logs, axis=0)               # [n, Dk], log domain
                Gam = np.exp(G)
                gamma_C = Gam[n - 1]
                # pairwise decay exp(G_r - G_i), only where i <= r (no overflow)
                diff = G[:, None, :] - G[None, :, :]       # [r, i, d]
                lower = np.tril(np.ones((n, n), bool))
                diff = np.where(lower[:, :, None], diff, -np.inf)
                dec = np.exp(diff)
                KK = np.einsum("rd,id,rid->ri", K, KW, dec)
                QK = np.einsum("rd,id,rid->ri", Q, KW, dec)
                A = np.tril(bt[:, None] * KK, -1)
                Tm = forward_substitution_inverse(A)
                K_bar = Gam * K
                W = Tm @ (bt[:, None] * K_bar)
                U = Tm @ (bt[:, None] * V)
                D = U - W @ h
                Q_bar = Gam * Q
                o[b, c0:c1, h_] = Q_bar @ h + np.tril(QK) @ D
                K_tilde = KW * np.exp(G[n - 1][None, :] - G)
                h = gamma_C[:, None] * h + K_tilde.T @ D
            M_final[b, h_] = h
    return o, M_final


def backward(q, k, v, beta, g, gate_kind, S0, do, dS=None):
    """Gradients of the operator by reverse-mode automatic differentiation of
    the plain token loop (torch autograd, fp64, CPU): the scalar
        L = sum(o * do) + sum(S_T * dS)
    differentiated with respect to q, k, v, beta, g and S0.  The loop is the
    recurrence of :func:`recurrent` (decay, recall, residual, write, output),
    written with torch ops so that autograd can run through it; the pages print
    no backward formula, so the definition of the gradient is the derivative of
    the forward itself.  Returns a dict dq, dk, dv, dbeta, dg (None without a
    gate), dS0 (of the same shapes as the inputs; dS0 also when S0 is None).
    """
    import torch
    t = {n: None if a is None else torch.tensor(np.asarray(a, np.float64), requires_grad=True)
         for n, a in (("q", q), ("k", k), ("v", v), ("beta", beta), ("g", g))}
    B, T, H, Dk = t["q"].shape
    Dv = t["v"].shape[-1]
    S0t = torch.zeros(B, H, Dk, Dv, dtype=torch.float64) if S0 is None else \
        torch.tensor(np.asarray(S0, np.float64))
    S0t.requires_grad_(True)
    M = S0t
    outs = []
    for step in range(T):
        if gate_kind == GATE_SCALAR:
            M = torch.exp(t["g"][:, step])[:, :, None, None] * M
        elif gate_kind == GATE_PER_DIM:
            M = torch.exp(t["g"][:, step])[:, :, :, None] * M
        kt, vt, qt = t["k"][:, step], t["v"][:, step], t["q"][:, step]
        x = torch.einsum("bhij,bhi->bhj", M, kt)
        r = t["beta"][:, step][..., None] * (vt - x)
        M = M + kt[..., :, None] * r[..., None, :]
        outs.append(torch.einsum("bhij,bhi->bhj", M, qt))
    o = torch.stack(outs, 1) if T else torch.zeros(B, 0, H, Dv, dtype=torch.float64)
    loss = (o * torch.tensor(np.asarray(do, np.float64))).sum()
    if dS is not None:
        loss = loss + (M * torch.tensor(np.asarray(dS, np.float64))).sum()
    wrt = [t["q"], t["k"], t["v"], t["beta"], S0t] + ([t["g"]] if gate_kind != GATE_NONE else [])
    grads = torch.autograd.grad(loss, wrt, allow_unused=True)
    z = lambda gr, ref: (np.zeros(ref.shape) if gr is None else gr.detach().numpy())
    out = {"dq": z(grads[0], t["q"]), "dk": z(grads[1], t["k"]), "dv": z(grads[2], t["v"]),
           "dbeta": z(grads[3], t["beta"]), "dS0": z(grads[4], S0t),
           "dg": z(grads[5], t["g"]) if gate_kind != GATE_NONE else None}
    return out


def chunk_backward(q, k, v, beta, g, gate_kind, S0, do, dS=None, C: int = 64):
    """The same gradients as :func:`backward`, chunk by chunk (fp64 NumPy), by
    differentiating the chunk form of :func:`chunk_form` by hand.  Per chunk,
    with h the entering state, h' = Diag(gamma) h + K_tilde^T D the leaving one,
    O = Q_bar h + P D, D = U - W h, and the upstream dO, dh':

      dD  = P^T dO + K_tilde dh'
      dh  = Q_bar^T dO - W^T dD + Diag(gamma) dh'       (the adjoint state: the
            transpose of the chunk's affine map, run from the last chunk back)
      dU = dD,  dW = -dD h^T,  dT = dU (beta V)^T + dW (beta K_bar)^T,
      dA = StrictTril(-T^T dT T^T)                       (T = (I + A)^-1)
      then through P = Tril(Q_bar K_breve^T), A = StrictTril(beta K_bar
      K_breve^T), K_bar = Gamma K, Q_bar = Gamma Q, K_tilde = K Gamma_C / Gamma
      to dq, dk, dv, dbeta and the in-chunk log-decays G, and dg as the
      reverse cumulative sum of dG within the chunk (a scalar gate sums dG over
      the key dimensions).
    Returns the dict of :func:`backward`.
    """
    q, k, v, beta, g, S0, do, dS = map(_f64, (q, k, v, beta, g, S0, do, dS))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dbeta": np.zeros_like(beta), "dS0": np.zeros((B, H, Dk, Dv)),
           "dg": None if gate_kind == GATE_NONE else np.zeros_like(g)}
    for b in range(B):
        for h_ in range(H):
            # forward over the chunks, keeping each entering state
            chunks = [(c0, min(T, c0 + C)) for c0 in range(0, T, C)]
            hs = []
            h = np.zeros((Dk, Dv)) if S0 is None else S0[b, h_].copy()
            saved = []
            for c0, c1 in chunks:
                n = c1 - c0
                Q, K, V = q[b, c0:c1, h_], k[b, c0:c1, h_], v[b, c0:c1, h_]
                bt = beta[b, c0:c1, h_]
                if gate_kind == GATE_NONE:
                    logs = np.zeros((n, Dk))
                elif gate_kind == GATE_SCALAR:
                    logs = np.repeat(g[b, c0:c1, h_][:, None], Dk, axis=1)
                else:
                    logs = g[b, c0:c1, h_]
                G = np.cumsum(logs, axis=0)
                Gam = np.exp(G)
                diff = G[:, None, :] - G[None, :, :]
                lower = np.tril(np.ones((n, n), bool))
                E = np.exp(np.where(lower[:, :, None], diff, -np.inf))      # [r, i, d]
                KK = np.einsum("rd,id,rid->ri", K, K, E)
                QK = np.einsum("rd,id,rid->ri", Q, K, E)
                A = np.tril(bt[:, None] * KK, -1)
                Tm = forward_substitution_inverse(A)
                Kbar, Qbar = Gam * K, Gam * Q
                W, U = Tm @ (bt[:, None] * Kbar), Tm @ (bt[:, None] * V)
                D = U - W @ h
                P = np.tril(QK)
                Kt = K * np.exp(G[n - 1][None, :] - G)
                gam = Gam[n - 1]
                hs.append(h)
                saved.append((c0, c1, n, Q, K, V, bt, G, E, KK, Tm, Kbar, Qbar, W, D, P, Kt, gam))
                h = gam[:, None] * h + Kt.T @ D
            # backward over the chunks
            dhn = np.zeros((Dk, Dv)) if dS is None else dS[b, h_].copy()
            for (c0, c1, n, Q, K, V, bt, G, E, KK, Tm, Kbar, Qbar, W, D, P, Kt, gam), h in \
                    zip(reversed(saved), reversed(hs)):
                dO = do[b, c0:c1, h_]
                dD = P.T @ dO + Kt @ dhn
                dh = Qbar.T @ dO - W.T @ dD + gam[:, None] * dhn
                dq = np.zeros((n, Dk)); dk = np.zeros((n, Dk)); dG = np.zeros((n, Dk))
                dQbar = dO @ h.T
                dq += np.exp(G) * dQbar
                dG += dQbar * Qbar
                dP = np.tril(dO @ D.T)
                dq += np.einsum("ri,id,rid->rd", dP, K, E)
                dk += np.einsum("ri,rd,rid->id", dP, Q, E)
                tP = np.einsum("ri,rd,id,rid->rid", dP, Q, K, E)
                dG += tP.sum(1)
                dG -= tP.sum(0)
                dKt = D @ dhn.T
                dk += dKt * np.exp(G[n - 1][None, :] - G)
                tK = dKt * Kt
                dG -= tK
                dG[n - 1] += tK.sum(0)
                dG[n - 1] += gam * np.sum(h * dhn, axis=1)
                dU, dW = dD, -dD @ h.T
                dT = dU @ (bt[:, None] * V).T + dW @ (bt[:, None] * Kbar).T
                TdU, TdW = Tm.T @ dU, Tm.T @ dW
                out["dv"][b, c0:c1, h_] = bt[:, None] * TdU
                dbeta = np.sum(TdU * V, axis=1) + np.sum(TdW * Kbar, axis=1)
                dKbar = bt[:, None] * TdW
                dk += np.exp(G) * dKbar
                dG += dKbar * Kbar
                dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
                dbeta += np.sum(dA * KK, axis=1)
                dKK = bt[:, None] * dA
                dk += np.einsum("ri,id,rid->rd", dKK, K, E)
                dk += np.einsum("ri,rd,rid->id", dKK, K, E)
                tA = np.einsum("ri,rd,id,rid->rid", dKK, K, K, E)
                dG += tA.sum(1)
                dG -= tA.sum(0)
                out["dq"][b, c0:c1, h_] = dq
                out["dk"][b, c0:c1, h_] = dk
                out["dbeta"][b, c0:c1, h_] = dbeta
                dgc = np.cumsum(dG[::-1], axis=0)[::-1]      # dg_t = sum_{r >= t} dG_r
                if gate_kind == GATE_SCALAR:
                    out["dg"][b, c0:c1, h_] = dgc.sum(1)
                elif gate_kind == GATE_PER_DIM:
                    out["dg"][b, c0:c1, h_] = dgc
                dhn = dh
            out["dS0"][b, h_] = dhn
    return out


def rel_err(x, ref) -> float:
    """max|x - ref| / max|ref| over the whole tensor (0 when both are zero)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    num = np.max(np.abs(x - ref)) if ref.size else 0.0
    if den == 0.0:
        return float(num)
    return float(num / den)
