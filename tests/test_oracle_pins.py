"""Pins for the fp64 CPU oracle (CPU only).

Each test checks the oracle against something other than itself: a worked
example computed by hand, closed forms derived by hand from the update rules,
invariants the method fixes (Kaczmarz interpolation, decay-only, NLMS scale
invariance, linearity), gradient steps checked by finite differences of the
two objectives, Kaczmarz convergence, and agreement between the recurrent,
masked-parallel and chunk-parallel forms ("Fast Weight Attention for Continual
Learning", authors' abstract: the three forms compute the same rule).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from delta_rule_linear_falcon_b200 import inputs as I

HERE = os.path.dirname(os.path.abspath(__file__))
R1, R1A, R3, R3A = oracle.RULE_1, oracle.RULE_1A, oracle.RULE_3, oracle.RULE_3A
ALL_RULES = [(R1, 1), (R1A, 1), (R3, 3), (R3A, 3)]


def rng_problem(seed, B=1, H=2, T=37, dk=8, dv=6, normal_keys=False, alpha_lo=0.6):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, T, dk))
    k = r.standard_normal((B, H, T, dk))
    if normal_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, H, T, dv))
    alpha = r.uniform(alpha_lo, 1.0, (B, H, T))
    eta = r.uniform(0.1, 1.0, (B, H, T))
    return q, k, v, alpha, eta


def relerr(a, b):
    return float(np.max(np.abs(a - b)) / max(1e-300, np.max(np.abs(b))))


# ---------------------------------------------------------------- worked example

@pytest.mark.parametrize("name", ["falcon1", "falcon1a", "falcon3", "falcon3a"])
@pytest.mark.parametrize("form", ["recurrent", "chunk1", "chunk2", "masked"])
def test_hand_worked_example(name, form):
    g = json.load(open(os.path.join(HERE, "golden", "hand_worked_T3_d2.json")))
    inp, exp = g["inputs"], g["expected"][name]
    arr = lambda key: np.asarray(inp[key], dtype=np.float64)[None, None]
    q, k, v = arr("q"), arr("k"), arr("v")
    a = np.asarray(inp["alpha"], dtype=np.float64)[None, None]
    e = np.asarray(inp["eta"], dtype=np.float64)[None, None]
    if form == "recurrent":
        o, S, kl = oracle.recurrent(exp["rule"], q, k, v, a, e, inp["eps"], exp["window"])
    elif form == "masked":
        o, S, kl = oracle.masked(exp["rule"], q, k, v, a, e, inp["eps"], exp["window"])
    else:
        o, S, kl = oracle.chunk(exp["rule"], q, k, v, a, e, inp["eps"], exp["window"],
                                chunk=int(form[-1]))
    np.testing.assert_allclose(o[0, 0], exp["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], exp["S"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(kl[0, 0], exp["k_last"], rtol=0, atol=0)


# ---------------------------------------------------------------- hand-expanded algebra

def test_falcon1_hand_expanded_first_three_steps():
    """Falcon-1, S_0 = 0, no cache. Expanded by hand (1-based steps):
    o_1 = 0;  o_2 = beta_2 (k_1.q_2) v_2;
    o_3 = alpha_3 beta_2 (k_1.q_3 - beta_3 (k_1.k_2)(k_2.q_3)) v_2 + beta_3 (k_2.q_3) v_3,
    with beta_t = eta_t / (||k_{t-1}||^2 + eps)."""
    q, k, v, alpha, eta = rng_problem(3, B=1, H=1, T=3, dk=5, dv=4)
    eps = 1e-3
    o, _, _ = oracle.recurrent(R1, q, k, v, alpha, eta, eps)
    q, k, v, a, e = q[0, 0], k[0, 0], v[0, 0], alpha[0, 0], eta[0, 0]
    b2 = e[1] / (k[0] @ k[0] + eps)
    b3 = e[2] / (k[1] @ k[1] + eps)
    o1 = np.zeros(4)
    o2 = b2 * (k[0] @ q[1]) * v[1]
    o3 = a[2] * b2 * (k[0] @ q[2] - b3 * (k[0] @ k[1]) * (k[1] @ q[2])) * v[1] + b3 * (k[1] @ q[2]) * v[2]
    np.testing.assert_allclose(o[0, 0], np.stack([o1, o2, o3]), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("name", ["falcon3", "falcon3a"])
@pytest.mark.parametrize("form", ["recurrent", "masked", "chunk2", "chunk4", "chunk6"])
def test_falcon3_window_slides_worked_by_hand(name, form):
    """Falcon-3 / 3A with w = 2 over four tokens, every step worked by hand in exact rationals
    (derivation in the fixture): the window fills, then slides and drops a pair. Each prefix of
    the sequence gives the state after that step, so every step's output and state are pinned.
    The chunk forms hold floor(chunk / w) tokens per block (1, 2 and 3)."""
    from fractions import Fraction as Fr
    g = json.load(open(os.path.join(HERE, "golden", "hand_worked_falcon3_w2_T4.json")))
    inp, exp = g["inputs"], g["expected"][name]
    val = lambda a: np.vectorize(lambda x: float(Fr(x)))(np.asarray(a, dtype=object)).astype(np.float64)
    o_exp, S_exp = val(exp["o"]), val(exp["S_after"])
    arr = lambda key: np.asarray(inp[key], dtype=np.float64)[None, None]
    for T in range(1, 5):
        q, k, v = arr("q")[:, :, :T], arr("k")[:, :, :T], arr("v")[:, :, :T]
        a, e = arr("alpha")[:, :, :T], arr("eta")[:, :, :T]
        if form == "recurrent":
            o, S, kl = oracle.recurrent(exp["rule"], q, k, v, a, e, inp["eps"], inp["window"])
        elif form == "masked":
            o, S, kl = oracle.masked(exp["rule"], q, k, v, a, e, inp["eps"], inp["window"])
        else:
            o, S, kl = oracle.chunk(exp["rule"], q, k, v, a, e, inp["eps"], inp["window"],
                                    chunk=int(form[5:]))
        np.testing.assert_allclose(o[0, 0], o_exp[:T], rtol=0, atol=1e-14)
        np.testing.assert_allclose(S[0, 0], S_exp[T - 1], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(kl[0, 0], g["expected"]["k_last"])


def _unrolled_falcon1(k, v, q, alpha, eta, eps, S0, k_prev):
    """Falcon-1 written out without its recurrence, in exact rationals: with
    M_s = alpha_s (I - beta_s x_s x_s^T) (the state transition of step s, acting on the right),
        S_t = S_0 M_1 ... M_t + sum_{j<=t} beta_j y_j x_j^T M_{j+1} ... M_t,   o_t = S_t q_t,
    x_1 = k_prev (or 0), x_j = k_{j-1}, y_j = v_j, beta_j = eta_j / (||x_j||^2 + eps) (0 when that
    denominator is 0). Returns the list of o_t and the final S as Fraction matrices."""
    from fractions import Fraction as Fr
    T, dk, dv = len(k), len(k[0]), len(v[0])
    eye = [[Fr(int(i == j)) for j in range(dk)] for i in range(dk)]
    mul = lambda A, B: [[sum(A[i][m] * B[m][j] for m in range(len(B))) for j in range(len(B[0]))]
                        for i in range(len(A))]
    x = [k_prev if k_prev is not None else [Fr(0)] * dk] + [k[j - 1] for j in range(1, T)]
    beta = []
    for j in range(T):
        den = sum(c * c for c in x[j]) + eps
        beta.append(eta[j] / den if den != 0 else Fr(0))
    M = [[[alpha[s] * (eye[i][c] - beta[s] * x[s][i] * x[s][c]) for c in range(dk)] for i in range(dk)]
         for s in range(T)]
    outs, S = [], None
    for t in range(T):
        prod = eye
        for s in range(t, -1, -1):          # prod = M_s ... M_t, built from the right
            prod = mul(M[s], prod)
        S = mul(S0, prod)                    # S_0 M_1 ... M_t
        for j in range(t + 1):
            tail = eye
            for s in range(t, j, -1):
                tail = mul(M[s], tail)       # M_{j+1} ... M_t
            write = [[beta[j] * v[j][i] * x[j][c] for c in range(dk)] for i in range(dv)]
            W = mul(write, tail)
            S = [[S[i][c] + W[i][c] for c in range(dk)] for i in range(dv)]
        outs.append([sum(S[i][c] * q[t][c] for c in range(dk)) for i in range(dv)])
    return outs, S


@pytest.mark.parametrize("with_cache", [False, True])
def test_falcon1_unrolled_closed_form_T8(with_cache):
    """Falcon-1 over eight tokens against the recurrence unrolled by hand into a sum of products
    of step transitions, evaluated in exact rational arithmetic (d_k = 3, d_v = 2, small integer
    keys, rational gates, an initial state and optionally a cached key). Every o_1..o_8 and the
    final state are pinned."""
    from fractions import Fraction as Fr
    k = [[1, 0, 2], [0, 1, -1], [2, 1, 0], [1, -1, 1], [0, 2, 1], [1, 1, 1], [-1, 0, 2], [3, 1, -2]]
    v = [[1, 2], [0, -1], [2, 1], [-1, 3], [1, 0], [2, -2], [0, 1], [1, 1]]
    q = [[1, 1, 0], [0, 1, 2], [1, 0, -1], [2, 1, 1], [0, 0, 1], [1, -1, 0], [1, 2, 1], [0, 1, 1]]
    alpha = [Fr(9, 10), Fr(4, 5), Fr(1), Fr(1, 2), Fr(7, 8), Fr(3, 4), Fr(1), Fr(5, 8)]
    eta = [Fr(1), Fr(1, 2), Fr(3, 4), Fr(1), Fr(1, 4), Fr(2, 3), Fr(1), Fr(1, 2)]
    eps = Fr(1, 10)
    S0 = [[Fr(1, 2), Fr(0), Fr(-1, 4)], [Fr(0), Fr(1, 3), Fr(1)]]
    k_prev = [Fr(1), Fr(-2), Fr(0)] if with_cache else None
    F = lambda rows: [[Fr(c) for c in r] for r in rows]
    outs, S = _unrolled_falcon1(F(k), F(v), F(q), alpha, eta, eps, S0, k_prev)
    f64 = lambda a: np.asarray([[float(c) for c in r] for r in a], dtype=np.float64)[None, None]
    o, So, kl = oracle.recurrent(R1, f64(q), f64(k), f64(v), np.asarray([[list(map(float, alpha))]]),
                                 np.asarray([[list(map(float, eta))]]), float(eps), 1, S0=f64(S0),
                                 k_prev=(np.asarray([[[float(c) for c in k_prev]]]) if with_cache else None))
    np.testing.assert_allclose(o[0, 0], f64(outs)[0, 0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(So[0, 0], f64(S)[0, 0], rtol=1e-13, atol=1e-14)
    for form, kw in (("chunk", {"chunk": 3}), ("masked", {})):
        fn = oracle.chunk if form == "chunk" else oracle.masked
        o2, S2, _ = fn(R1, f64(q), f64(k), f64(v), np.asarray([[list(map(float, alpha))]]),
                       np.asarray([[list(map(float, eta))]]), float(eps), 1, S0=f64(S0),
                       k_prev=(np.asarray([[[float(c) for c in k_prev]]]) if with_cache else None), **kw)
        np.testing.assert_allclose(o2[0, 0], f64(outs)[0, 0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(S2[0, 0], f64(S)[0, 0], rtol=1e-12, atol=1e-13)


def test_falcon1a_is_gated_linear_attention():
    """Falcon-1A closed form (S_0 = 0): S_T = sum_t (prod_{s>t} alpha_s) beta_t y_t x_t^T and
    o_t = sum_{j<=t} (prod_{j<s<=t} alpha_s) beta_j (x_j.q_t) y_j."""
    q, k, v, alpha, eta = rng_problem(4, B=1, H=1, T=20, dk=6, dv=5)
    eps = 1e-6
    o, S, _ = oracle.recurrent(R1A, q, k, v, alpha, eta, eps)
    q, k, v, a, e = q[0, 0], k[0, 0], v[0, 0], alpha[0, 0], eta[0, 0]
    T = 20
    x = np.vstack([np.zeros(6), k[:-1]])
    beta = e / (np.sum(x * x, axis=1) + eps)
    o_ref = np.zeros((T, 5))
    for t in range(T):
        for j in range(t + 1):
            o_ref[t] += np.prod(a[j + 1:t + 1]) * beta[j] * (x[j] @ q[t]) * v[j]
    S_ref = sum(np.prod(a[t + 1:]) * beta[t] * np.outer(v[t], x[t]) for t in range(T))
    np.testing.assert_allclose(o[0, 0], o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kaczmarz_interpolation_any_decay(seed):
    """Falcon-1 with eta = 1, eps = 0 is an exact Kaczmarz projection: S_t x_t = y_t for every
    step with x_t != 0, whatever alpha is. Reading back with q_t = x_t gives o_t = v_t."""
    q, k, v, alpha, eta = rng_problem(seed, alpha_lo=0.05)
    q[:, :, 1:] = k[:, :, :-1]
    eta[:] = 1.0
    for form in ("recurrent", "chunk"):
        if form == "recurrent":
            o, _, _ = oracle.recurrent(R1, q, k, v, alpha, eta, 0.0)
        else:
            o, _, _ = oracle.chunk(R1, q, k, v, alpha, eta, 0.0, chunk=8)
        np.testing.assert_allclose(o[:, :, 1:], v[:, :, 1:], rtol=0, atol=1e-11)


@pytest.mark.parametrize("rule,w", ALL_RULES)
def test_decay_only_when_eta_zero(rule, w):
    """eta = 0: no write, S_t = (prod_{s<=t} alpha_s) S_0 and o_t = S_t q_t; S_0 = 0 gives o = 0."""
    q, k, v, alpha, eta = rng_problem(5)
    eta[:] = 0.0
    r = np.random.default_rng(9)
    S0 = r.standard_normal((1, 2, 6, 8))
    o, S, _ = oracle.recurrent(rule, q, k, v, alpha, eta, 1e-6, w, S0=S0)
    cum = np.cumprod(alpha, axis=-1)
    o_ref = cum[..., None] * np.einsum("bhic,bhtc->bhti", S0, q)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(S, cum[..., -1, None, None] * S0, rtol=1e-12)
    o0, S0o, _ = oracle.chunk(rule, q, k, v, alpha, eta, 1e-6, w, chunk=7)
    assert np.all(o0 == 0) and np.all(S0o == 0)


def test_nlms_scale_invariance():
    """Falcon-1 with eps = 0, S_0 = 0: scaling every key and query by c leaves o unchanged
    (the normalised step absorbs the key scale; the NLMS property)."""
    q, k, v, alpha, eta = rng_problem(6)
    o1, _, _ = oracle.recurrent(R1, q, k, v, alpha, eta, 0.0)
    for c in (1e-3, -2.5, 40.0):
        o2, _, _ = oracle.recurrent(R1, c * q, c * k, v, alpha, eta, 0.0)
        assert relerr(o2, o1) < 1e-11


@pytest.mark.parametrize("rule,w", ALL_RULES)
def test_linearity_in_values(rule, w):
    """With S_0 = 0 every rule is linear in v."""
    q, k, v, alpha, eta = rng_problem(7)
    v2 = np.random.default_rng(8).standard_normal(v.shape)
    o1, S1, _ = oracle.recurrent(rule, q, k, v, alpha, eta, 1e-6, w)
    o2, S2, _ = oracle.recurrent(rule, q, k, v2, alpha, eta, 1e-6, w)
    o3, S3, _ = oracle.recurrent(rule, q, k, v - 3.0 * v2, alpha, eta, 1e-6, w)
    assert relerr(o3, o1 - 3.0 * o2) < 1e-11
    assert relerr(S3, S1 - 3.0 * S2) < 1e-11


def test_orthonormal_keys_recall():
    """alpha = 1, eta = 1, eps = 0, orthonormal keys: every written pair is recalled exactly
    (projections onto orthogonal directions do not disturb one another)."""
    d = 8
    Q, _ = np.linalg.qr(np.random.default_rng(10).standard_normal((d, d)))
    T = d + 1
    k = np.zeros((1, 1, T, d)); k[0, 0, :d] = Q.T
    v = np.random.default_rng(11).standard_normal((1, 1, T, 5))
    q = np.zeros_like(k)
    a = np.ones((1, 1, T)); e = np.ones((1, 1, T))
    _, S, _ = oracle.recurrent(R1, q, k, v, a, e, 0.0)
    # pair t is (k_{t-1}, v_t) for t >= 1
    np.testing.assert_allclose(S[0, 0] @ Q, v[0, 0, 1:].T, atol=1e-12)


def test_kaczmarz_converges_on_consistent_system():
    """Cycling a consistent system y = W x with keys spanning R^d (alpha = eta = 1, eps = 0)
    drives S to W (Kaczmarz convergence)."""
    d, dv, m, sweeps = 6, 4, 9, 60
    r = np.random.default_rng(12)
    W = r.standard_normal((dv, d))
    K = r.standard_normal((m, d))
    T = m * sweeps + 1
    k = np.zeros((1, 1, T, d)); v = np.zeros((1, 1, T, dv))
    for t in range(T - 1):
        k[0, 0, t] = K[t % m]
        v[0, 0, t + 1] = W @ K[t % m]     # pair t+1 = (k_t, v_{t+1})
    q = np.zeros_like(k)
    one = np.ones((1, 1, T))
    _, S, _ = oracle.recurrent(R1, q, k, v, one, one, 0.0)
    assert np.max(np.abs(S[0, 0] - W)) < 1e-8


def test_falcon3_orthonormal_window_closed_form():
    """Falcon-3 step with mutually orthonormal window keys: S_t x_j = (1-beta) Sbar x_j + beta y_j
    for every j in the window, beta = eta / (w + eps)."""
    d, w = 8, 3
    Q, _ = np.linalg.qr(np.random.default_rng(13).standard_normal((d, d)))
    T = w + 1
    k = np.zeros((1, 1, T, d)); k[0, 0, :w] = Q[:, :w].T
    r = np.random.default_rng(14)
    v = r.standard_normal((1, 1, T, 5)); q = r.standard_normal((1, 1, T, d))
    a = r.uniform(0.5, 1.0, (1, 1, T)); e = r.uniform(0.2, 1.0, (1, 1, T))
    S0 = r.standard_normal((1, 1, 5, d))
    _, Sa, _ = oracle.recurrent(R3, q[:, :, :T - 1], k[:, :, :T - 1], v[:, :, :T - 1], a[:, :, :T - 1],
                                e[:, :, :T - 1], 0.0, w, S0=S0)
    _, Sb, _ = oracle.recurrent(R3, q, k, v, a, e, 0.0, w, S0=S0)
    t = T - 1
    Sbar = a[0, 0, t] * Sa[0, 0]
    beta = e[0, 0, t] / w
    for m in range(w):
        j = t - m
        x = k[0, 0, j - 1]
        np.testing.assert_allclose(Sb[0, 0] @ x, (1 - beta) * Sbar @ x + beta * v[0, 0, j], atol=1e-12)


# ---------------------------------------------------------------- gradient steps (finite differences)

def _fd_grad(loss, S, h=1e-4):
    G = np.zeros_like(S)
    for idx in np.ndindex(*S.shape):
        E = np.zeros_like(S); E[idx] = h
        G[idx] = (loss(S + E) - loss(S - E)) / (2 * h)
    return G


@pytest.mark.parametrize("rule,w", ALL_RULES)
def test_step_is_normalised_gradient_step(rule, w):
    """One step equals Sbar - beta * grad L(Sbar), with the gradient taken by central finite
    differences of the step's objective: squared-error regression 1/2 sum_j ||S x_j - y_j||^2
    for Falcon-1/3, negative inner product -sum_j y_j^T S x_j for Falcon-1A/3A (abstract), and
    beta = eta / (sum_j ||x_j||^2 + eps). The read after the write is o_t = S_t q_t."""
    r = np.random.default_rng(20 + rule)
    T, dk, dv, eps = 6, 5, 4, 1e-3
    q = r.standard_normal((1, 1, T, dk)); k = r.standard_normal((1, 1, T, dk))
    v = r.standard_normal((1, 1, T, dv)); a = r.uniform(0.5, 1, (1, 1, T)); e = r.uniform(0.2, 1, (1, 1, T))
    S0 = r.standard_normal((1, 1, dv, dk))
    _, Sa, _ = oracle.recurrent(rule, q[:, :, :-1], k[:, :, :-1], v[:, :, :-1], a[:, :, :-1],
                                e[:, :, :-1], eps, w, S0=S0)
    ob, Sb, _ = oracle.recurrent(rule, q, k, v, a, e, eps, w, S0=S0)
    t = T - 1
    win = [t - m for m in range(w) if t - m >= 0]
    xs = [k[0, 0, j - 1] for j in win]
    ys = [v[0, 0, j] for j in win]
    if rule in (R1, R3):
        loss = lambda S: 0.5 * sum(np.sum((S @ x - y) ** 2) for x, y in zip(xs, ys))
    else:
        loss = lambda S: -sum(y @ S @ x for x, y in zip(xs, ys))
    Sbar = a[0, 0, t] * Sa[0, 0]
    beta = e[0, 0, t] / (sum(x @ x for x in xs) + eps)
    S_ref = Sbar - beta * _fd_grad(loss, Sbar)
    np.testing.assert_allclose(Sb[0, 0], S_ref, atol=1e-8)
    np.testing.assert_allclose(ob[0, 0, t], Sb[0, 0] @ q[0, 0, t], atol=1e-12)


# ---------------------------------------------------------------- forms agree

@pytest.mark.parametrize("rule,w", ALL_RULES + [(R3, 1), (R3, 4), (R3A, 4)])
@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 16, 64])
def test_three_forms_agree(rule, w, C):
    """Recurrent, masked-parallel and chunk-parallel forms agree to fp64 round-off,
    with an initial state, a cached key and a ragged last chunk (T = 37)."""
    q, k, v, alpha, eta = rng_problem(30 + C, normal_keys=True, alpha_lo=0.3)
    r = np.random.default_rng(31)
    S0 = r.standard_normal((1, 2, 6, 8)); kp = r.standard_normal((1, 2, 8))
    o_r, S_r, kl_r = oracle.recurrent(rule, q, k, v, alpha, eta, 1e-6, w, S0=S0, k_prev=kp)
    o_c, S_c, kl_c = oracle.chunk(rule, q, k, v, alpha, eta, 1e-6, w, chunk=C, S0=S0, k_prev=kp)
    assert relerr(o_c, o_r) < 1e-12 and relerr(S_c, S_r) < 1e-12
    assert np.array_equal(kl_c, kl_r)
    if C == 64:
        o_m, S_m, _ = oracle.masked(rule, q, k, v, alpha, eta, 1e-6, w, S0=S0, k_prev=kp)
        assert relerr(o_m, o_r) < 1e-12 and relerr(S_m, S_r) < 1e-12


def test_falcon3_window_one_is_falcon1():
    q, k, v, alpha, eta = rng_problem(40)
    a = oracle.recurrent(R1, q, k, v, alpha, eta, 1e-6)
    b = oracle.recurrent(R3, q, k, v, alpha, eta, 1e-6, 1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    c = oracle.chunk(R3, q, k, v, alpha, eta, 1e-6, 1, chunk=5)
    assert relerr(c[0], a[0]) < 1e-12


def test_falcon3_window_differs_from_falcon1():
    """A wider window must change the result (guards against the window being ignored)."""
    q, k, v, alpha, eta = rng_problem(41)
    a = oracle.recurrent(R1, q, k, v, alpha, eta, 1e-6)[0]
    b = oracle.recurrent(R3, q, k, v, alpha, eta, 1e-6, 2)[0]
    assert relerr(a, b) > 1e-3


# ---------------------------------------------------------------- state continuation

@pytest.mark.parametrize("rule", [R1, R1A])
def test_segment_split_and_decode(rule):
    """fwd(T) == fwd(T1) then fwd(T - T1) from (S_out, k_last) == T single-token decode steps."""
    q, k, v, alpha, eta = rng_problem(50, T=23)
    o, S, kl = oracle.recurrent(rule, q, k, v, alpha, eta, 1e-6)
    T1 = 9
    oa, Sa, kla = oracle.chunk(rule, q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], alpha[:, :, :T1],
                               eta[:, :, :T1], 1e-6, chunk=4)
    ob, Sb, klb = oracle.chunk(rule, q[:, :, T1:], k[:, :, T1:], v[:, :, T1:], alpha[:, :, T1:],
                               eta[:, :, T1:], 1e-6, chunk=4, S0=Sa, k_prev=kla)
    assert relerr(np.concatenate([oa, ob], axis=2), o) < 1e-12 and relerr(Sb, S) < 1e-12
    assert np.array_equal(klb, kl)
    Sd = np.zeros_like(S)
    kd = np.zeros(k.shape[:2] + k.shape[-1:])
    for t in range(23):
        od, Sd, kd = oracle.decode_step(rule, Sd, kd, q[:, :, t], k[:, :, t], v[:, :, t],
                                        alpha[:, :, t], eta[:, :, t], 1e-6)
        assert relerr(od, o[:, :, t]) < 1e-12 or np.max(np.abs(o[:, :, t])) == 0
    assert relerr(Sd, S) < 1e-12


# ---------------------------------------------------------------- renormalisation

def test_tiny_alpha_no_underflow_nan():
    """alpha down to 1e-30 (log alpha = -69) and long products stay finite in every form."""
    q, k, v, alpha, eta = rng_problem(60, T=50)
    alpha[..., ::7] = 1e-30
    alpha[..., 3::11] = 1e-12
    o_r, S_r, _ = oracle.recurrent(R1, q, k, v, alpha, eta, 1e-6)
    o_c, S_c, _ = oracle.chunk(R1, q, k, v, alpha, eta, 1e-6, chunk=16)
    assert np.all(np.isfinite(o_c)) and np.all(np.isfinite(S_c))
    assert relerr(o_c, o_r) < 1e-12


def test_long_sequence_strong_decay_products_underflow_safely():
    """Cumulative log decay far below the fp64 range (sum log alpha ~ -2000): the chunk form
    never forms a global product and still matches the recurrence."""
    q, k, v, alpha, eta = rng_problem(61, H=1, T=400, dk=4, dv=3, alpha_lo=0.0)
    alpha = np.full_like(alpha, math.exp(-5.0))
    o_r, S_r, _ = oracle.recurrent(R1, q, k, v, alpha, eta, 1e-6)
    o_c, S_c, _ = oracle.chunk(R1, q, k, v, alpha, eta, 1e-6, chunk=64)
    assert np.all(np.isfinite(o_c))
    assert relerr(o_c, o_r) < 1e-12


# ---------------------------------------------------------------- input generator sanity

def test_input_generator_is_deterministic_and_distributed():
    a = I.normal(7, 1, 200001)
    b = I.normal(7, 1, 200001)
    assert np.array_equal(a, b)
    assert abs(float(a.mean())) < 0.01 and abs(float(a.std()) - 1.0) < 0.01
    c = I.normal(7, 2, 1000)
    assert not np.array_equal(a[:1000], c)
    x = I.round_bf16(np.array([1.0, 1.00390625, 1.005859375, -3.14159], dtype=np.float32))
    assert x[0] == 1.0 and x[1] == 1.0 and x[2] == 1.0078125
    s = I.make_seq(I.RULE_1, 1, 2, 16, 32, 32, seed=0, normalise_qk=True)
    np.testing.assert_allclose(np.linalg.norm(s.k, axis=-1), 1.0, atol=1e-2)
