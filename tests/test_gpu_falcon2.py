"""GPU parity of Falcon-2 / Falcon-2A (the per-column extension, under the reading the design notes
record) on the recurrent kernel, through the C ABI, against the fp64 oracle: fp32 inputs at 1e-4,
bf16 inputs at 2e-2 (the fp32 state and the running column energies at 1e-4), with an initial
state, a cached key, initial column energies and the same-step flag; the continuation cache
(S_out, k_last, n_out) resumes a split sequence. The chunk and decode entry points refuse these
rules."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, TOL_F32, dev, host, relerr  # noqa: F401

pytestmark = pytest.mark.gpu
SS = 0x100


def _run(F, s, n0):
    dt = torch.bfloat16 if s.io_dtype == "bf16" else torch.float32
    q, k, v = dev(s.q, dt), dev(s.k, dt), dev(s.v, dt)
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0 = dev(s.S0, torch.float32) if s.S0 is not None else None
    kp = dev(s.k_prev, dt) if s.k_prev is not None else None
    n0d = dev(n0, torch.float32) if n0 is not None else None
    B, H, T, dk = q.shape
    n_out = torch.empty((B, H, dk), dtype=torch.float32, device="cuda")
    o, S, kl = F.falcon_fwd_recurrent(q, k, v, a, e, rule=s.rule, eps=s.eps, S0=S0, k_prev=kp, n0=n0d,
                                      n_out=n_out)
    torch.cuda.synchronize()
    assert F.falcon_check_device_errors() == F.FALCON_OK
    return host(o), host(S), host(kl), host(n_out)


@pytest.mark.parametrize("rule", [5, 6, 5 | SS, 6 | SS])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48), (128, 128), (17, 5)])
def test_falcon2_recurrent_matches_oracle(F, rule, io, dk, dv):
    s = I.make_seq(rule, 2, 2, 77, dk, dv, seed=500 + dk + (rule & 0xff), io_dtype=io, with_state=True,
                   with_kprev=True)
    n0 = np.random.default_rng(dk).uniform(0.0, 2.0, (2, 2, dk)).astype(np.float32)
    o, S, kl, n = _run(F, s, n0)
    o_r, S_r, kl_r, n_r = oracle.falcon2(rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps, S0=s.S0, k_prev=s.k_prev,
                                         n0=n0)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    assert relerr(o, o_r) <= tol
    assert relerr(S, S_r) <= TOL_F32
    assert relerr(n, n_r) <= 1e-5
    assert np.array_equal(kl, kl_r.astype(np.float32).astype(np.float64))


def test_falcon2_continuation(F):
    """fwd(T) == fwd(T1) then fwd(T - T1) from (S_out, k_last, n_out), on the GPU."""
    s = I.make_seq(5, 1, 3, 90, 64, 64, seed=520, io_dtype="f32")
    full = _run(F, s, None)
    T1 = 37
    cut = lambda x, a, b: np.ascontiguousarray(x[:, :, a:b])
    a = I.SeqInputs(5, "f32", cut(s.q, 0, T1), cut(s.k, 0, T1), cut(s.v, 0, T1), cut(s.alpha, 0, T1),
                    cut(s.eta, 0, T1), s.eps)
    ga = _run(F, a, None)
    b = I.SeqInputs(5, "f32", cut(s.q, T1, 90), cut(s.k, T1, 90), cut(s.v, T1, 90), cut(s.alpha, T1, 90),
                    cut(s.eta, T1, 90), s.eps, S0=ga[1].astype(np.float32), k_prev=ga[2].astype(np.float32))
    gb = _run(F, b, ga[3].astype(np.float32))
    assert relerr(np.concatenate([ga[0], gb[0]], axis=2), full[0]) <= 1e-5
    assert relerr(gb[1], full[1]) <= 1e-5 and relerr(gb[3], full[3]) <= 1e-6


def test_falcon2_refused_by_chunk_and_decode(F):
    s = I.make_seq(5, 1, 2, 64, 128, 128, seed=530, io_dtype="bf16")
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    with pytest.raises(F.FalconError) as ei:
        F.falcon_fwd_chunk(q, k, v, a, e, rule=5)
    assert ei.value.status == F.FALCON_ERR_UNSUPPORTED
    S = torch.zeros((1, 2, 128, 128), dtype=torch.float32, device="cuda")
    kp = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(F.FalconError) as ei:
        F.falcon_decode_step(S, kp, q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous(),
                             a[:, :, 0].contiguous(), e[:, :, 0].contiguous(), rule=6)
    assert ei.value.status == F.FALCON_ERR_UNSUPPORTED


@pytest.mark.parametrize("rule", [5, 6])
def test_falcon2_bench_shape(F, rule):
    """The benchmark's Falcon-2 / 2A shape (bf16, T4096 d128), two heads: outputs at the bf16
    tolerance, the fp32 state and column energies at 1e-4."""
    s = I.make_seq(rule, 1, 2, 4096, 128, 128, seed=11, io_dtype="bf16")
    o, S, kl, n = _run(F, s, None)
    o_r, S_r, kl_r, n_r = oracle.falcon2(rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps)
    assert relerr(o, o_r) <= TOL_BF16
    assert relerr(S, S_r) <= TOL_F32
    assert relerr(n, n_r) <= TOL_F32
