"""Pins for the Falcon-2 / Falcon-2A oracle (CPU only), under the reading the design notes record
for "its per-column extension" of the scalar NLMS update ("Fast Weight Attention for Continual
Learning": authors' abstract; ai.info overview, Key Contributions 3 and Methodology in Plain
English, "a version that keeps a separate normalization per column"): each column of S keeps the
running energy of its key coordinate, and the step is the NLMS step in that diagonal metric.

Pins: a worked example in exact rationals; the step against a finite-difference gradient of the
squared error with the per-column step sizes; the limit of equal column energies, where it is
Falcon-1 (and Falcon-2A is Falcon-1A); exact interpolation; NLMS scale invariance; decay only; and
the recurrent, blocked and masked forms agreeing, with a state, a cached key, initial column
energies and the same-step flag.
"""
import json
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
R2, R2A = oracle.RULE_2, oracle.RULE_2A
SS = 0x100


def rand(seed, B=1, H=2, T=23, dk=6, dv=5):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, T, dk)), r.standard_normal((B, H, T, dk)), r.standard_normal((B, H, T, dv)),
            r.uniform(0.5, 1.0, (B, H, T)), r.uniform(0.1, 1.0, (B, H, T)))


@pytest.mark.parametrize("name", ["falcon2", "falcon2a"])
@pytest.mark.parametrize("chunk", [0, 1, 2, 3])
def test_falcon2_worked_by_hand(name, chunk):
    g = json.load(open(os.path.join(HERE, "golden", "hand_worked_falcon2_T3.json")))
    inp, exp = g["inputs"], g["expected"][name]
    arr = lambda key: np.asarray(inp[key], dtype=np.float64)[None, None]
    val = lambda a: np.vectorize(lambda x: float(Fr(x)))(np.asarray(a, dtype=object)).astype(np.float64)
    o, S, kl, n = oracle.falcon2(exp["rule"], arr("q"), arr("k"), arr("v"), arr("alpha"), arr("eta"), inp["eps"],
                                 chunk=chunk)
    np.testing.assert_allclose(o[0, 0], val(exp["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], val(exp["S"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(n[0, 0], g["expected"]["n_out"], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(kl[0, 0], g["expected"]["k_last"])


@pytest.mark.parametrize("rule", [R2, R2A])
def test_step_is_the_per_column_normalised_gradient(rule):
    """One step from a random state and random column energies: S_1 - Sbar equals
    -(eta / (x^T D x + eps)) * grad * D, with grad the finite-difference gradient of
    1/2 ||Sbar x - y||^2 (Falcon-2) or of -y^T Sbar x (Falcon-2A), D = diag(1 / (n + eps)),
    n = alpha n0 + x^2."""
    r = np.random.default_rng(3)
    dk, dv, eps = 5, 4, 0.02
    S0 = r.standard_normal((1, 1, dv, dk))
    n0 = r.uniform(0.1, 2.0, (1, 1, dk))
    x = r.standard_normal(dk)
    y = r.standard_normal(dv)
    a, e = 0.8, 0.7
    q = r.standard_normal((1, 1, 1, dk))
    k = r.standard_normal((1, 1, 1, dk))   # only k_last; the pair of step 0 is (k_prev, v_0)
    _, S1, _, n1 = oracle.falcon2(rule, q, k, y[None, None, None], np.full((1, 1, 1), a), np.full((1, 1, 1), e),
                                  eps, S0=S0, k_prev=x[None, None], n0=n0)
    Sbar = a * S0[0, 0]
    loss = (lambda M: 0.5 * np.sum((M @ x - y) ** 2)) if rule == R2 else (lambda M: -(y @ M @ x))
    h = 1e-6
    grad = np.zeros_like(Sbar)
    for i in range(dv):
        for c in range(dk):
            P = Sbar.copy(); P[i, c] += h
            M = Sbar.copy(); M[i, c] -= h
            grad[i, c] = (loss(P) - loss(M)) / (2 * h)
    n = a * n0[0, 0] + x * x
    np.testing.assert_allclose(n1[0, 0], n, rtol=1e-14)
    d = 1.0 / (n + eps)
    step = -(e / (x @ (d * x) + eps)) * grad * d[None, :]
    np.testing.assert_allclose(S1[0, 0] - Sbar, step, rtol=1e-7, atol=1e-9)


@pytest.mark.parametrize("rules", [(R2, oracle.RULE_1), (R2A, oracle.RULE_1A)])
def test_equal_column_energies_give_falcon1(rules):
    """Keys whose coordinates all have the same magnitude keep every column's energy equal, so D is
    a multiple of I; with eps = 0 the step is then the scalar NLMS step of Falcon-1 (Falcon-1A)."""
    r2, r1 = rules
    r = np.random.default_rng(11)
    B, H, T, dk, dv = 1, 2, 31, 8, 5
    mag = r.uniform(0.5, 2.0, (B, H, T, 1))
    k = mag * r.choice([-1.0, 1.0], (B, H, T, dk))
    q, _, v, alpha, eta = rand(12, B, H, T, dk, dv)
    kp = 1.3 * r.choice([-1.0, 1.0], (B, H, dk))
    S0 = r.standard_normal((B, H, dv, dk))
    o2, S2, _, _ = oracle.falcon2(r2, q, k, v, alpha, eta, 0.0, S0=S0, k_prev=kp)
    o1, S1, _ = oracle.recurrent(r1, q, k, v, alpha, eta, 0.0, S0=S0, k_prev=kp)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=1e-11, atol=1e-12)


def test_exact_interpolation():
    """eta = 1, eps = 0, keys without zero coordinates: S_t x_t = y_t after every write, whatever
    alpha and the column energies are; reading back with q_t = x_t gives o_t = v_t."""
    q, k, v, alpha, eta = rand(13)
    q[:, :, 1:] = k[:, :, :-1]
    eta[:] = 1.0
    for chunk in (0, 5):
        o, _, _, _ = oracle.falcon2(R2, q, k, v, alpha, eta, 0.0, chunk=chunk)
        np.testing.assert_allclose(o[:, :, 1:], v[:, :, 1:], rtol=0, atol=1e-10)


@pytest.mark.parametrize("rule", [R2, R2A])
def test_scale_invariance(rule):
    """eps = 0, S_0 = 0, no initial energies: scaling every key and query by c leaves o unchanged."""
    q, k, v, alpha, eta = rand(14)
    o1, _, _, _ = oracle.falcon2(rule, q, k, v, alpha, eta, 0.0)
    o2, _, _, _ = oracle.falcon2(rule, 3.0 * q, 3.0 * k, v, alpha, eta, 0.0)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-12)


def test_decay_only():
    q, k, v, alpha, eta = rand(15)
    eta[:] = 0.0
    S0 = np.random.default_rng(1).standard_normal((1, 2, 5, 6))
    o, S, _, _ = oracle.falcon2(R2, q, k, v, alpha, eta, 1e-6, S0=S0)
    cum = np.cumprod(alpha, axis=-1)
    np.testing.assert_allclose(S, cum[..., -1, None, None] * S0, rtol=1e-12)
    np.testing.assert_allclose(o, cum[..., None] * np.einsum("bhic,bhtc->bhti", S0, q), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("rule", [R2, R2A, R2 | SS, R2A | SS])
def test_three_forms_agree_with_state_cache_and_energies(rule):
    q, k, v, alpha, eta = rand(16 + (rule & 0xff), T=41)
    r = np.random.default_rng(2)
    S0 = r.standard_normal((1, 2, 5, 6))
    kp = r.standard_normal((1, 2, 6))
    n0 = r.uniform(0.0, 3.0, (1, 2, 6))
    ref = oracle.falcon2(rule, q, k, v, alpha, eta, 1e-3, S0=S0, k_prev=kp, n0=n0)
    for chunk in (1, 4, 16, 41):
        got = oracle.falcon2(rule, q, k, v, alpha, eta, 1e-3, chunk=chunk, S0=S0, k_prev=kp, n0=n0)
        for g_, r_ in zip(got, ref):
            np.testing.assert_allclose(g_, r_, rtol=1e-11, atol=1e-12)


def test_segment_split_carries_the_column_energies():
    """fwd(T) == fwd(T1) then fwd(T - T1) from (S_out, k_last, n_out)."""
    q, k, v, alpha, eta = rand(17, T=30)
    full = oracle.falcon2(R2, q, k, v, alpha, eta, 1e-4)
    a = oracle.falcon2(R2, q[:, :, :11], k[:, :, :11], v[:, :, :11], alpha[:, :, :11], eta[:, :, :11], 1e-4)
    b = oracle.falcon2(R2, q[:, :, 11:], k[:, :, 11:], v[:, :, 11:], alpha[:, :, 11:], eta[:, :, 11:], 1e-4,
                       S0=a[1], k_prev=a[2], n0=a[3])
    np.testing.assert_allclose(np.concatenate([a[0], b[0]], axis=2), full[0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(b[1], full[1], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(b[3], full[3], rtol=1e-12)
