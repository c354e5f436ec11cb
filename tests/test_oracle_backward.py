"""Pins for the fp64 backward oracle (CPU only): its gradients of the recurrent form against
central finite differences of the forward oracle, for every input, every rule, the same-step
flag, an initial state and a cached key. The loss is L = <dO, o> + <dS_T, S_T> with random
upstream gradients, so every output and the final state enter it.
"""
import numpy as np
import pytest

import oracle

R1, R1A, R3, R3A = oracle.RULE_1, oracle.RULE_1A, oracle.RULE_3, oracle.RULE_3A
SS = 0x100


def problem(seed, T=9, dk=5, dv=4):
    r = np.random.default_rng(seed)
    q = r.standard_normal((1, 2, T, dk))
    k = r.standard_normal((1, 2, T, dk))
    v = r.standard_normal((1, 2, T, dv))
    alpha = r.uniform(0.5, 1.0, (1, 2, T))
    eta = r.uniform(0.2, 1.0, (1, 2, T))
    S0 = r.standard_normal((1, 2, dv, dk)) * 0.5
    kp = r.standard_normal((1, 2, dk))
    dO = r.standard_normal((1, 2, T, dv))
    dST = r.standard_normal((1, 2, dv, dk))
    return q, k, v, alpha, eta, S0, kp, dO, dST


def loss(rule, w, eps, q, k, v, alpha, eta, S0, kp, dO, dST):
    o, S, _ = oracle.recurrent(rule, q, k, v, alpha, eta, eps, w, S0=S0, k_prev=kp)
    return float(np.sum(dO * o) + np.sum(dST * S))


@pytest.mark.parametrize("rule,w", [(R1, 1), (R1A, 1), (R3, 3), (R3A, 2), (R1 | SS, 1), (R3 | SS, 2)])
def test_backward_matches_finite_differences(rule, w):
    q, k, v, alpha, eta, S0, kp, dO, dST = problem(40 + (rule & 0xff) + w)
    eps = 0.05
    g = oracle.backward(rule, q, k, v, alpha, eta, eps, dO, dST, window=w, S0=S0, k_prev=kp)
    inputs = {"q": q, "k": k, "v": v, "alpha": alpha, "eta": eta, "S0": S0, "k_prev": kp}
    names = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "eta": "deta", "S0": "dS0", "k_prev": "dk_prev"}
    r = np.random.default_rng(7)
    h = 1e-6
    for name, arr in inputs.items():
        for _ in range(6):
            idx = tuple(r.integers(0, n) for n in arr.shape)
            args = {kk: vv.copy() for kk, vv in inputs.items()}
            args[name][idx] += h
            lp = loss(rule, w, eps, args["q"], args["k"], args["v"], args["alpha"], args["eta"], args["S0"],
                      args["k_prev"], dO, dST)
            args[name][idx] -= 2 * h
            lm = loss(rule, w, eps, args["q"], args["k"], args["v"], args["alpha"], args["eta"], args["S0"],
                      args["k_prev"], dO, dST)
            fd = (lp - lm) / (2 * h)
            an = g[names[name]][idx]
            if rule & SS and name == "k_prev":
                assert an == 0.0 and abs(fd) < 1e-8   # the cached key is not read with the flag
                continue
            assert abs(an - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, an, fd)


def test_backward_without_state_gradient_and_zero_keys():
    """dS_T = 0 (outputs only); zero keys with eps = 0 write nothing and carry no gradient through
    the step size (beta = 0 there)."""
    q, k, v, alpha, eta, S0, kp, dO, _ = problem(5)
    k[:, :, 3] = 0.0
    g = oracle.backward(R1, q, k, v, alpha, eta, 0.0, dO, None, S0=S0, k_prev=kp)
    h = 1e-6
    for t in range(9):
        e = eta.copy(); e[0, 1, t] += h
        lp = loss(R1, 1, 0.0, q, k, v, alpha, e, S0, kp, dO, np.zeros_like(S0))
        e[0, 1, t] -= 2 * h
        lm = loss(R1, 1, 0.0, q, k, v, alpha, e, S0, kp, dO, np.zeros_like(S0))
        assert abs(g["deta"][0, 1, t] - (lp - lm) / (2 * h)) <= 1e-6
    assert g["deta"][0, 0, 4] == 0.0   # step 4 writes x_4 = k_3 = 0


def test_backward_decay_only():
    """eta = 0: o_t = (prod alpha) S_0 q_t, so dq_t = (prod_{s<=t} alpha_s) S_0^T dO_t and the keys and
    values get no gradient."""
    q, k, v, alpha, eta, S0, kp, dO, dST = problem(6)
    eta[:] = 0.0
    g = oracle.backward(R1, q, k, v, alpha, eta, 0.1, dO, dST, S0=S0, k_prev=kp)
    cum = np.cumprod(alpha, axis=-1)
    dq = cum[..., None] * np.einsum("bhic,bhti->bhtc", S0, dO)
    np.testing.assert_allclose(g["dq"], dq, rtol=1e-12, atol=1e-14)
    assert np.all(g["dk"] == 0) and np.all(g["dv"] == 0)
