"""GPU parity of the backward pass of the recurrent form (falcon_bwd_recurrent, through the C ABI)
against the fp64 oracle's reverse-mode gradients (which are pinned by finite differences on the CPU):
every gradient array (dq, dk, dv, dalpha, deta, dS0, dk_prev) within TOL_BWD of its largest entry,
for Falcon-1/1A/3/3A, the same-step flag, an initial state, a cached key, an upstream gradient of the
final state, fp32 and bf16 inputs, square and non-square heads, and checkpointed segments with a
ragged last one."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, dev, host, relerr  # noqa: F401

pytestmark = pytest.mark.gpu
SS = 0x100
# The backward pass runs in fp32 from the same (bf16-representable) inputs as the oracle, so its
# error is fp32 rounding accumulated over the T steps of the reverse sweep and the recomputed
# forward states; the forward recurrent form is held to 1e-4 of max|o| for the same reason.
TOL_BWD = 1e-4
NAMES = ("dq", "dk", "dv", "dalpha", "deta", "dS0", "dk_prev")


def _upstream(seed, B, H, T, dk, dv, with_dST):
    dO = I.normal(seed, 8, B * H * T * dv).reshape(B, H, T, dv).astype(np.float32)
    dST = I.normal(seed, 9, B * H * dv * dk).reshape(B, H, dv, dk).astype(np.float32) if with_dST else None
    return dO, dST


def _gpu(F, s, dO, dST):
    dt = torch.bfloat16 if s.io_dtype == "bf16" else torch.float32
    q, k, v = dev(s.q, dt), dev(s.k, dt), dev(s.v, dt)
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0 = dev(s.S0, torch.float32) if s.S0 is not None else None
    kp = dev(s.k_prev, dt) if s.k_prev is not None else None
    g = F.falcon_bwd_recurrent(q, k, v, a, e, dev(dO, torch.float32), rule=s.rule, eps=s.eps, window=s.window,
                               S0=S0, k_prev=kp, dS_T=dev(dST, torch.float32) if dST is not None else None)
    torch.cuda.synchronize()
    assert F.falcon_check_device_errors() == F.FALCON_OK
    return {n: (host(t) if t is not None else None) for n, t in g.items()}


def _check(F, s, dO, dST):
    got = _gpu(F, s, dO, dST)
    ref = oracle.backward(s.rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps, dO, dS_T=dST, window=s.window,
                          S0=s.S0, k_prev=s.k_prev)
    for n in NAMES:
        if ref[n] is None:
            assert got[n] is None, n
            continue
        assert np.all(np.isfinite(got[n])), n
        err = relerr(got[n], ref[n])
        assert err <= TOL_BWD, (n, err)


CASES = [(1, 1), (2, 1), (3, 2), (3, 4), (4, 2), (4, 4), (1 | SS, 1), (2 | SS, 1), (3 | SS, 2), (4 | SS, 4)]


@pytest.mark.parametrize("rule,w", CASES)
def test_backward_matches_oracle_small_heads(F, rule, w):
    """The parity workload's shape (B1 H2 T256 d32, fp32) with every optional input."""
    s = I.make_seq(rule, 1, 2, 256, 32, 32, seed=600 + rule + 10 * w, io_dtype="f32", normalise_qk=False,
                   alpha_mu=3.0, window=w, with_state=True, with_kprev=True)
    dO, dST = _upstream(601 + rule, 1, 2, 256, 32, 32, True)
    _check(F, s, dO, dST)


@pytest.mark.parametrize("rule,w", [(1, 1), (2, 1), (3, 4), (4, 4), (1 | SS, 1)])
def test_backward_matches_oracle_bf16_full_width(F, rule, w):
    """bf16 inputs, d_k = d_v = 128, 12 checkpointed segments of 9 steps with a ragged last one."""
    s = I.make_seq(rule, 1, 2, 100, 128, 128, seed=620 + rule + w, io_dtype="bf16", window=w,
                   with_state=True, with_kprev=True)
    dO, dST = _upstream(621 + rule, 1, 2, 100, 128, 128, True)
    _check(F, s, dO, dST)


@pytest.mark.parametrize("rule,w,T,dk,dv", [(1, 1, 1, 32, 32), (3, 2, 2, 48, 24), (2, 1, 50, 24, 48),
                                            (4, 4, 3, 16, 16), (1, 1, 37, 128, 64)])
def test_backward_edges(F, rule, w, T, dk, dv):
    """One to three steps (windows larger than the sequence), non-square heads, no initial state, no
    cached key (no dk_prev) and no upstream gradient of the final state."""
    s = I.make_seq(rule, 2, 1, T, dk, dv, seed=640 + T + dk, io_dtype="f32", window=w)
    dO, _ = _upstream(641 + T, 2, 1, T, dk, dv, False)
    _check(F, s, dO, None)


def test_backward_state_gradient_only(F):
    """dO = 0 and dS_T given: the gradients are those of <dS_T, S_T> alone."""
    s = I.make_seq(1, 1, 1, 64, 32, 32, seed=660, io_dtype="f32", with_state=True, with_kprev=True)
    dO = np.zeros((1, 1, 64, 32), dtype=np.float32)
    _, dST = _upstream(661, 1, 1, 64, 32, 32, True)
    _check(F, s, dO, dST)


def test_backward_refuses_falcon2(F):
    s = I.make_seq(5, 1, 1, 8, 16, 16, seed=670, io_dtype="f32")
    dO, _ = _upstream(671, 1, 1, 8, 16, 16, False)
    with pytest.raises(F.FalconError) as ei:
        _gpu(F, s, dO, None)
    assert ei.value.status == F.FALCON_ERR_UNSUPPORTED


def test_backward_bench_workload_heads(F):
    """The benchmark's backward shape (bf16, T1024 d128, initial state, cached key, dS_T), two of its
    heads: 32 checkpointed segments of 32 steps."""
    s = I.make_seq(1, 1, 2, 1024, 128, 128, seed=7, io_dtype="bf16", with_state=True, with_kprev=True)
    dO, dST = _upstream(680, 1, 2, 1024, 128, 128, True)
    _check(F, s, dO, dST)
