"""The regression rules' two-pass path on the GPU (falcon_fwd_chunk with a workspace that holds
every block's solved tiles) against the single-kernel path (a smaller workspace) and the fp64
oracle: both paths within the bf16 tolerance of the oracle and within a small fraction of it of
each other, over several blocks with a ragged tail, lengths around one block, an initial state
and a cached key, the same-step flag, Falcon-3 at windows 1, 2 and 4 (the windowed layout:
rows in m-major order, the solve in token-major order), strong and tiny decays, and the
Falcon-1 and Falcon-3 benchmark workloads at full size."""
import ctypes

import numpy as np
import pytest
import torch

from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, dev, host, relerr, run_oracle, _full, _spread_heads, _gather  # noqa: F401

pytestmark = pytest.mark.gpu
SS = 0x100
# the two paths run the same arithmetic; they may differ only in the accumulation order of the
# key Gram products, far below the tolerance either is held to
TOL_PATHS = 2e-3


def _both(F, s):
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0 = dev(s.S0, torch.float32) if s.S0 is not None else None
    kp = dev(s.k_prev, torch.bfloat16) if s.k_prev is not None else None
    args = F.make_args(q, k, v, a, e, rule=s.rule, eps=s.eps, window=s.window, chunk=64, S0=S0, k_prev=kp,
                       o=torch.empty_like(v))
    need = F.falcon_workspace_size(args)
    out = {}
    for name, ws in (("two_pass", torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")),
                     ("single", torch.empty(16, dtype=torch.uint8, device="cuda"))):
        o, S, kl = F.falcon_fwd_chunk(q, k, v, a, e, rule=s.rule, eps=s.eps, window=s.window, chunk=64, S0=S0,
                                      k_prev=kp, workspace=ws)
        torch.cuda.synchronize()
        assert F.falcon_check_device_errors() == F.FALCON_OK
        out[name] = (host(o), host(S), host(kl))
    return need, out


def _check(s, out, heads=None):
    ref = run_oracle(s) if heads is None else None
    for name, (o, S, kl) in out.items():
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(S)), name
        if ref is not None:
            assert relerr(o, ref[0]) <= TOL_BF16, (name, relerr(o, ref[0]))
            assert relerr(S, ref[1]) <= TOL_BF16, (name, relerr(S, ref[1]))
    (o1, S1, k1), (o2, S2, k2) = out["two_pass"], out["single"]
    assert relerr(o1, o2) <= TOL_PATHS and relerr(S1, S2) <= TOL_PATHS
    assert np.array_equal(k1, k2)


@pytest.mark.parametrize("rule,w", [(1, 1), (3, 1), (1 | SS, 1), (3, 2), (3, 4), (3 | SS, 4)])
@pytest.mark.parametrize("T", [1, 2, 5, 15, 16, 17, 63, 64, 65, 201, 640])
def test_two_pass_matches_single_kernel_and_oracle(F, rule, w, T):
    s = I.make_seq(rule, 2, 3, T, 128, 128, seed=1100 + T + rule + 7 * w, io_dtype="bf16", window=w,
                   with_state=True, with_kprev=True)
    need, out = _both(F, s)
    tb = 64 // w
    assert need == 2 * 3 * ((T + tb - 1) // tb) * 16384
    _check(s, out)


def test_two_pass_strong_and_tiny_decay(F):
    """alpha down to 1e-30 and runs of alpha = 1: every factor the first pass forms stays in (0, 1]."""
    s = I.make_seq(1, 1, 4, 257, 128, 128, seed=1114, io_dtype="bf16", with_state=True)
    s.alpha[..., ::9] = 1e-30
    s.alpha[..., 100:140] = 1.0
    _check(s, _both(F, s)[1])


def test_two_pass_zero_keys_and_decay_only(F):
    s = I.make_seq(1, 1, 4, 130, 128, 128, seed=1113, io_dtype="bf16", with_state=True, eps=0.0)
    s.k[:, :, ::5] = 0.0
    _check(s, _both(F, s)[1])
    s.eta[:] = 0.0
    _check(s, _both(F, s)[1])


def test_two_pass_workspace_sizes(F):
    """Only window-1 regression rules on the d = 128 bf16 kernel with 64-token blocks use tiles."""
    z = lambda *sh: torch.zeros(*sh, dtype=torch.bfloat16, device="cuda")
    one = lambda *sh: torch.ones(*sh, dtype=torch.float32, device="cuda")
    def size(rule, B, H, T, d, chunk=64, window=1):
        q, k, v = z(B, H, T, d), z(B, H, T, d), z(B, H, T, d)
        args = F.make_args(q, k, v, one(B, H, T), one(B, H, T), rule=rule, chunk=chunk, window=window,
                           o=z(B, H, T, d))
        return F.falcon_workspace_size(args)
    assert size(1, 2, 3, 130, 128) == 2 * 3 * 3 * 16384
    assert size(3, 1, 2, 64, 128, window=1) == 2 * 16384
    assert size(1 | SS, 1, 1, 65, 128) == 2 * 16384
    assert size(3, 1, 2, 256, 128, window=4) == 2 * 16 * 16384   # 16 tokens per block
    assert size(3, 1, 2, 100, 128, window=2) == 2 * 4 * 16384     # 32 tokens per block
    assert size(3, 1, 2, 256, 128, window=3) == 0     # w = 3: the mma.sync kernel
    assert size(1, 1, 2, 256, 64) == 0                # d = 64: the mma.sync kernel
    assert size(1, 1, 2, 256, 128, chunk=32) == 0
    assert size(4, 1, 2, 256, 128, window=1) == 0     # inner-product rules have no solve


def test_two_pass_full_benchmark_workload(F):
    """B8 H16 T4096 d128: both paths over all heads against each other, 16 sampled heads of each
    against the oracle."""
    s = _full("f1")
    need, out = _both(F, s)
    assert need == 8 * 16 * 64 * 16384
    (o1, S1, k1), (o2, S2, k2) = out["two_pass"], out["single"]
    assert relerr(o1, o2) <= TOL_PATHS and relerr(S1, S2) <= TOL_PATHS and np.array_equal(k1, k2)
    pairs = _spread_heads(8, 16)
    b = np.array([p[0] for p in pairs])
    h = np.array([p[1] for p in pairs])
    g = _gather(s, pairs)
    ref = run_oracle(g)
    for o, S in ((o1, S1), (o2, S2)):
        assert relerr(o[b, h][None], ref[0]) <= TOL_BF16
        assert relerr(S[b, h][None], ref[1]) <= TOL_BF16


def test_two_pass_full_falcon3_workload(F):
    """Falcon-3 (w = 4) at B4 H16 T8192 d128: both paths over all heads against each other, 16 sampled
    heads of the two-pass result against the oracle."""
    s = _full("f3")
    need, out = _both(F, s)
    assert need == 4 * 16 * 512 * 16384
    (o1, S1, k1), (o2, S2, k2) = out["two_pass"], out["single"]
    assert relerr(o1, o2) <= TOL_PATHS and relerr(S1, S2) <= TOL_PATHS and np.array_equal(k1, k2)
    pairs = _spread_heads(4, 16)
    b = np.array([p[0] for p in pairs])
    h = np.array([p[1] for p in pairs])
    g = _gather(s, pairs)
    ref = run_oracle(g)
    assert relerr(o1[b, h][None], ref[0]) <= TOL_BF16
    assert relerr(S1[b, h][None], ref[1]) <= TOL_BF16
