"""The block algebra the tensor-core chunk kernel evaluates, restated in numpy (fp64) and
checked against the oracle's literal recurrence.

The chunk-parallel form with positive-decay renormalisation ("Fast Weight Attention for
Continual Learning", authors' abstract; ai.info overview, Methodology in Plain English)
computes per block U = T diag(beta) R', R' = Y - diag(2^g) X S^T, O = diag(2^g) Q S^T + P~ U,
S <- 2^g_last S + U^T diag(2^(g_last - g)) X. The kernel regroups it so that the state
crosses two tensor-core steps per block:
    A = T_f^T X,  B' = P~ T',  T' = T diag(beta),  T_f = diag(2^(g_last - g)) T'
    O^T = (S Q^T) diag(2^g) + R'^T B'^T,   S <- 2^g_last S + R'^T A.
This test pins that regrouping (and its Falcon-1A case, T = I) to the oracle.
"""
import numpy as np
import pytest

from oracle import oracle as O


def regrouped(rule, q, k, v, alpha, eta, eps, S0, kp, C=64):
    T = q.shape[0]
    X = np.concatenate([kp[None], k[:-1]])
    S = S0.copy()
    out = np.zeros((T, v.shape[1]))
    for t0 in range(0, T, C):
        n = min(C, T - t0)
        x, qq, y = X[t0:t0 + n], q[t0:t0 + n], v[t0:t0 + n]
        beta = eta[t0:t0 + n] / ((x * x).sum(1) + eps)
        g = np.cumsum(np.log2(alpha[t0:t0 + n]))
        gam = np.tril(np.exp2(np.minimum(g[:, None] - g[None, :], 0.0)))    # 2^(g_i - g_j), j <= i
        if rule == O.RULE_1:
            L = beta[:, None] * np.tril(gam * (x @ x.T), -1)
            Tm = np.linalg.inv(np.eye(n) + L)
        else:
            Tm = np.eye(n)
        Tp = Tm * beta[None, :]
        Tf = np.exp2(g[-1] - g)[:, None] * Tp
        A = Tf.T @ x
        Bp = (gam * (qq @ x.T)) @ Tp
        Rt = y.T - (S @ x.T) * np.exp2(g)[None, :] if rule == O.RULE_1 else y.T
        out[t0:t0 + n] = ((S @ qq.T) * np.exp2(g)[None, :] + Rt @ Bp.T).T
        S = np.exp2(g[-1]) * S + Rt @ A
    return out, S


@pytest.mark.parametrize("rule", [O.RULE_1, O.RULE_1A])
@pytest.mark.parametrize("T", [64, 200])
def test_regrouped_block_algebra_matches_recurrence(rule, T):
    rng = np.random.default_rng(11 + T + rule)
    dk, dv, eps = 16, 12, 1e-6
    q = rng.standard_normal((T, dk)); k = rng.standard_normal((T, dk)); v = rng.standard_normal((T, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.standard_normal(T) - 2.0))
    eta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    S0 = 0.1 * rng.standard_normal((dv, dk)); kp = rng.standard_normal(dk)
    o_ref, S_ref, _ = O.recurrent(rule, q[None, None], k[None, None], v[None, None], alpha[None, None],
                                  eta[None, None], eps, S0=S0[None, None], k_prev=kp[None, None])
    o, S = regrouped(rule, q, k, v, alpha, eta, eps, S0, kp)
    assert np.abs(o - o_ref[0, 0]).max() <= 1e-12 * np.abs(o_ref).max()
    assert np.abs(S - S_ref[0, 0]).max() <= 1e-12 * np.abs(S_ref).max()
