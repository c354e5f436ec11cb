"""GPU parity of the same-step association (FALCON_SAME_STEP: the pair written at step t is
(k_t, v_t), the Kaczmarz Linear Attention association) against the fp64 oracle, through the
C ABI: the warp-specialised tensor-core chunk kernel (d = 128, bf16, Falcon-1/1A), the
mma.sync chunk kernel (other shapes and the windowed rules), the recurrent kernel and the
decode step. Tolerances as in test_gpu_parity.py."""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, TOL_F32, check, dev, host, relerr, run_gpu, run_oracle  # noqa: F401

pytestmark = pytest.mark.gpu
SS = 0x100


@pytest.mark.parametrize("rule,w,d,chunk,io", [
    (1, 1, 128, 64, "bf16"),   # tensor-core kernel
    (2, 1, 128, 64, "bf16"),   # tensor-core kernel, inner-product rule
    (1, 1, 64, 32, "bf16"),    # mma.sync kernel
    (3, 4, 64, 64, "bf16"),    # windowed
    (4, 2, 32, 16, "bf16"),
])
def test_same_step_chunk(F, rule, w, d, chunk, io):
    """Several blocks and a ragged tail, an initial state and a cached key (which must be ignored)."""
    s = I.make_seq(rule | SS, 2, 3, 201, d, d, seed=300 + d + chunk, io_dtype=io, window=w, chunk=chunk,
                   with_state=True, with_kprev=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


def test_same_step_chunk_full_length_heads(F):
    """The tensor-core kernel at the benchmark's sequence length (T = 4096), two heads checked."""
    s = I.make_seq(1 | SS, 1, 2, 4096, 128, 128, seed=310, io_dtype="bf16", with_state=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


@pytest.mark.parametrize("rule,w", [(1, 1), (2, 1), (3, 3)])
def test_same_step_recurrent(F, rule, w):
    s = I.make_seq(rule | SS, 1, 2, 97, 32, 24, seed=320 + rule, io_dtype="f32", window=w,
                   with_state=True, with_kprev=True)
    check(s, run_gpu(F, s, "recurrent"), run_oracle(s), TOL_F32)


@pytest.mark.parametrize("rule", [1, 2])
def test_same_step_decode(F, rule):
    """T decode steps with the flag == the oracle's same-step recurrence over those T tokens;
    the cached key is still replaced by k."""
    s = I.make_seq(rule | SS, 3, 2, 12, 128, 64, seed=330, io_dtype="bf16", with_state=True, with_kprev=True)
    S = dev(s.S0, torch.float32)
    kp = dev(s.k_prev, torch.bfloat16)
    outs = []
    for t in range(12):
        o = F.falcon_decode_step(S, kp, dev(s.q[:, :, t], torch.bfloat16), dev(s.k[:, :, t], torch.bfloat16),
                                 dev(s.v[:, :, t], torch.bfloat16), dev(s.alpha[:, :, t], torch.float32),
                                 dev(s.eta[:, :, t], torch.float32), rule=rule | SS, eps=s.eps)
        outs.append(host(o))
    torch.cuda.synchronize()
    o_r, S_r, _ = run_oracle(s)
    assert relerr(np.stack(outs, axis=2), o_r) <= TOL_BF16
    assert relerr(host(S), S_r) <= TOL_F32
    assert np.array_equal(host(kp), s.k[:, :, -1].astype(np.float64))
    assert F.falcon_check_device_errors() == F.FALCON_OK
