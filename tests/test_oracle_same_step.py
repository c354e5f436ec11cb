"""Pins of the oracle's same-step association (flag SAME_STEP in the rule): the pair written at
step t is (k_t, v_t), the association of Kaczmarz Linear Attention (thelatestinai.com page,
KLA abstract), against the prefix-aligned (k_{t-1}, v_t) of the authors' abstract.

Pinned to things other than the oracle's own formula: a shift identity to the prefix-aligned
path (itself pinned by test_oracle_pins.py), agreement of the three forms, the exact Kaczmarz
projection (with q = k, eta = 1, eps = 0, Falcon-1 returns o_t = v_t), and the closed form of
the additive rule.
"""
import numpy as np
import pytest

from oracle import oracle as O

SS = O.SAME_STEP


def _inputs(rng, T, dk, dv, B=1, H=2):
    q = rng.standard_normal((B, H, T, dk)); k = rng.standard_normal((B, H, T, dk))
    v = rng.standard_normal((B, H, T, dv))
    alpha = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T)) - 2.0))
    eta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T))))
    S0 = 0.1 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, alpha, eta, S0


@pytest.mark.parametrize("rule,w", [(O.RULE_1, 1), (O.RULE_1A, 1), (O.RULE_3, 3), (O.RULE_3A, 2)])
def test_same_step_is_prefix_aligned_with_shifted_keys(rule, w):
    rng = np.random.default_rng(5 + rule)
    T, dk, dv = 37, 6, 5
    q, k, v, alpha, eta, S0 = _inputs(rng, T, dk, dv)
    o_s, S_s, kl_s = O.recurrent(rule | SS, q, k, v, alpha, eta, 1e-6, window=w, S0=S0)
    # prefix-aligned pair j uses k_prev for j = 0 and k'_{j-1} after: k_prev = k_0, k' = k shifted left
    k_shift = np.concatenate([k[:, :, 1:], rng.standard_normal((1, 2, 1, dk))], axis=2)
    o_p, S_p, _ = O.recurrent(rule, q, k_shift, v, alpha, eta, 1e-6, window=w, S0=S0, k_prev=k[:, :, 0])
    assert np.abs(o_s - o_p).max() <= 1e-13 * max(1.0, np.abs(o_p).max())
    assert np.abs(S_s - S_p).max() <= 1e-13 * max(1.0, np.abs(S_p).max())
    assert np.array_equal(kl_s, k[:, :, -1])          # the last key is still the cache for decode


@pytest.mark.parametrize("rule,w", [(O.RULE_1, 1), (O.RULE_1A, 1), (O.RULE_3, 4)])
@pytest.mark.parametrize("C", [1, 7, 16, 64])
def test_same_step_three_forms_agree(rule, w, C):
    rng = np.random.default_rng(11 * C + rule)
    T, dk, dv = 70, 5, 4
    q, k, v, alpha, eta, S0 = _inputs(rng, T, dk, dv)
    ref = O.recurrent(rule | SS, q, k, v, alpha, eta, 1e-6, window=w, S0=S0)
    for got in (O.chunk(rule | SS, q, k, v, alpha, eta, 1e-6, window=w, chunk=C, S0=S0),
                O.masked(rule | SS, q, k, v, alpha, eta, 1e-6, window=w, S0=S0)):
        for a, b in zip(got[:2], ref[:2]):
            assert np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(b).max())


def test_same_step_kaczmarz_projection_returns_the_value():
    """eta = 1, eps = 0: S_t k_t = v_t after each write, so reading with q_t = k_t returns v_t."""
    rng = np.random.default_rng(3)
    T, d = 40, 8
    _, k, v, alpha, _, S0 = _inputs(rng, T, d, d)
    o, _, _ = O.recurrent(O.RULE_1 | SS, k, k, v, alpha, np.ones_like(alpha), 0.0, S0=S0)
    assert np.abs(o - v).max() <= 1e-12 * np.abs(v).max()


def test_same_step_additive_rule_closed_form():
    """alpha = 1, S_0 = 0: S_T = sum_t beta_t v_t k_t^T with beta_t = eta_t / (||k_t||^2 + eps)."""
    rng = np.random.default_rng(4)
    T, dk, dv, eps = 23, 6, 4, 1e-3
    q, k, v, _, eta, _ = _inputs(rng, T, dk, dv)
    _, S, _ = O.recurrent(O.RULE_1A | SS, q, k, v, np.ones((1, 2, T)), eta, eps)
    beta = eta / ((k * k).sum(-1) + eps)
    want = np.einsum("bht,bhti,bhtj->bhij", beta, v, k)
    assert np.abs(S - want).max() <= 1e-12 * np.abs(want).max()


def test_rule_flag_validation():
    rng = np.random.default_rng(0)
    q, k, v, alpha, eta, S0 = _inputs(rng, 4, 3, 3)
    with pytest.raises(ValueError):
        O.recurrent(O.RULE_1 | 0x200, q, k, v, alpha, eta, 1e-6)
