"""GPU parity of the recurrent kernel under extreme decay gates.

The recurrent kernel keeps each head's rows as S = sigma S' with one running scale per
head: a step's decay multiplies sigma, and sigma is folded back into the rows whenever
it leaves [2^-60, 2^60]. These cases drive that fold: decays that are exactly zero (the
state is wiped at that step, so sigma would be 0), and runs of tiny decays whose product
falls far below 2^-60 within a few steps, between stretches of decay 1. Each case is
compared with the fp64 oracle at the fp32 tolerance, outputs and final state.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_falcon_b200 import inputs as I

from test_gpu_parity import TOL_F32, dev, host, relerr, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F(cuda_ok):
    from delta_rule_linear_falcon_b200 import build, falcon
    build.build()
    falcon.lib()
    return falcon


def extreme_decays(shape, seed):
    """Decay gates of value 1 with exact zeros, isolated tiny values and runs of tiny values."""
    rng = np.random.default_rng(seed)
    a = np.ones(shape, dtype=np.float32)
    T = shape[-1]
    for idx in np.ndindex(*shape[:-1]):
        row = a[idx]
        row[rng.choice(T, size=3, replace=False)] = 0.0          # state wiped at these steps
        row[rng.choice(T, size=4, replace=False)] = 1e-30        # one step under the fold bound
        for start in rng.choice(T - 6, size=2, replace=False):   # products down to 1e-40
            row[start:start + 5] = 1e-8
    return a


@pytest.mark.parametrize("rule,w", [(1, 1), (2, 1), (3, 4), (4, 3)])
@pytest.mark.parametrize("dk,dv", [(32, 32), (128, 128)])
def test_recurrent_extreme_decays(F, rule, w, dk, dv):
    s = I.make_seq(rule, 1, 2, 96, dk, dv, seed=700 + rule + dk, io_dtype="f32", window=w,
                   with_state=True, with_kprev=True)
    s = dataclasses.replace(s, alpha=extreme_decays(s.alpha.shape, seed=rule + dk))
    o, S, kl = run_gpu(F, s, "recurrent")
    o_r, S_r, kl_r = run_oracle(s)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    assert relerr(o, o_r) <= TOL_F32
    assert relerr(S, S_r) <= TOL_F32


@pytest.mark.parametrize("rule", [5, 6])
def test_falcon2_extreme_decays(F, rule):
    s = I.make_seq(rule, 1, 2, 96, 64, 64, seed=720 + rule, io_dtype="f32", with_state=True, with_kprev=True)
    s = dataclasses.replace(s, alpha=extreme_decays(s.alpha.shape, seed=rule))
    q, k, v = dev(s.q, torch.float32), dev(s.k, torch.float32), dev(s.v, torch.float32)
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0, kp = dev(s.S0, torch.float32), dev(s.k_prev, torch.float32)
    n_out = torch.empty((1, 2, 64), dtype=torch.float32, device="cuda")
    o, S, _ = F.falcon_fwd_recurrent(q, k, v, a, e, rule=rule, eps=s.eps, S0=S0, k_prev=kp, n_out=n_out)
    torch.cuda.synchronize()
    assert F.falcon_check_device_errors() == F.FALCON_OK
    o_r, S_r, _, n_r = oracle.falcon2(rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps, S0=s.S0, k_prev=s.k_prev)
    o, S = host(o), host(S)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    assert relerr(o, o_r) <= TOL_F32
    assert relerr(S, S_r) <= TOL_F32
    assert relerr(host(n_out), n_r) <= 1e-5
