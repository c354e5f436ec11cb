"""falcon_fwd_chunk_noalloc: the chunk-parallel pass with its scratch in the library's
fixed device array, for callers that cannot allocate device memory where they run it (a
plugin handed raw device pointers by a runtime with no allocator, a serving loop in
which a cudaMalloc could synchronise the device).

Called through the C ABI and compared with falcon_fwd_chunk on a workspace of the
caller's own, on two calls in a row with different inputs (the second call finds the
first one's leftovers in the shared array), on a smaller problem without state outputs
after a larger one, on a problem that needs no scratch, on the regression rules' two-pass
path with its tiles in the array and with tiles that would not fit (the single kernel runs),
and on a sequence split whose scratch would not fit, which must be refused before anything
runs. This
file is collected last so that a run stopping at its first failure has run every other
test; it passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, dev, host, relerr  # noqa: F401

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20   # FALCON_NOALLOC_SCRATCH_BYTES


def _noalloc(F):
    fn = F.lib().falcon_fwd_chunk_noalloc
    fn.argtypes = [ctypes.POINTER(F.FalconArgs), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _tensors(F, s: I.SeqInputs, want_state=True):
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0 = dev(s.S0, torch.float32) if s.S0 is not None else None
    kp = dev(s.k_prev, torch.bfloat16) if s.k_prev is not None else None
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    o = torch.empty_like(v)
    S = torch.empty((B, H, dv, dk), dtype=torch.float32, device="cuda") if want_state else None
    kl = torch.empty((B, H, dk), dtype=torch.bfloat16, device="cuda") if want_state else None
    args = F.make_args(q, k, v, a, e, rule=s.rule, eps=s.eps, chunk=64, S0=S0, k_prev=kp, o=o, S_out=S,
                       k_last=kl)
    outs = (o, S, kl) if want_state else (o,)
    return args, outs, (q, k, v, a, e, S0, kp)


def _run(F, s, noalloc, want_state=True):
    args, outs, keep = _tensors(F, s, want_state)
    L = F.lib()
    need = L.falcon_workspace_size(ctypes.byref(args))
    if noalloc:
        st = _noalloc(F)(ctypes.byref(args), None)
    else:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
        st = L.falcon_fwd_chunk(ctypes.byref(args), ctypes.c_void_p(ws.data_ptr()), need, None)
    assert st == F.FALCON_OK, F.falcon_status_string(st)
    torch.cuda.synchronize()
    assert F.falcon_check_device_errors() == F.FALCON_OK
    del keep
    return need, tuple(host(t) for t in outs)


def _same(got, ref):
    (o, S, kl), (o_r, S_r, kl_r) = got, ref
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    assert relerr(o, o_r) <= TOL_BF16
    assert relerr(S, S_r) <= TOL_BF16
    assert np.array_equal(kl, kl_r)


def test_noalloc_matches_the_workspace_entry_point_on_two_calls(F):
    """Falcon-1A with two heads of 4096 tokens takes the sequence split, whose state pass and
    scan keep their intermediates in the scratch."""
    cases = [I.make_seq(2, 1, 2, 4096, 128, 128, seed=seed, io_dtype="bf16", normalise_qk=False,
                        alpha_mu=6.0, with_state=True, with_kprev=True) for seed in (760, 761)]
    refs = [_run(F, s, noalloc=False) for s in cases]
    for s, (need, ref) in zip(cases, refs):
        assert 0 < need <= SCRATCH_BYTES
        need2, got = _run(F, s, noalloc=True)
        assert need2 == need
        _same(got, ref)


def test_noalloc_smaller_problem_without_state_after_a_larger_one(F):
    """A larger split problem fills more of the shared array; a smaller one with a different
    head count and length, and no final state or key requested (the split then skips the last
    segment's pieces and takes that segment's start state from the scan alone), follows it and
    must not read the leftovers."""
    big = I.make_seq(2, 1, 2, 8192, 128, 128, seed=780, io_dtype="bf16", normalise_qk=False,
                     alpha_mu=6.0, with_state=True, with_kprev=True)
    small = I.make_seq(2, 1, 3, 2048, 128, 128, seed=781, io_dtype="bf16", normalise_qk=False,
                       alpha_mu=6.0, with_state=True, with_kprev=True)
    need_b, ref_b = _run(F, big, noalloc=False)
    need_s, ref_s = _run(F, small, noalloc=False, want_state=False)
    assert 0 < need_s < need_b <= SCRATCH_BYTES
    _same(_run(F, big, noalloc=True)[1], ref_b)
    for _ in range(2):
        need2, (o,) = _run(F, small, noalloc=True, want_state=False)
        assert need2 == need_s
        assert np.all(np.isfinite(o))
        assert relerr(o, ref_s[0]) <= TOL_BF16


def test_noalloc_without_scratch_runs_the_plain_pass(F):
    """Falcon-1A with 15 blocks per head is too short to split: no scratch at all."""
    s = I.make_seq(2, 1, 2, 960, 128, 128, seed=770, io_dtype="bf16", normalise_qk=False, with_state=True)
    need, ref = _run(F, s, noalloc=False)
    assert need == 0
    _same(_run(F, s, noalloc=True)[1], ref)


def test_noalloc_two_pass_tiles_in_the_scratch(F):
    """Falcon-1: every block's solved tiles (16 KB per block) fit in the array, so the two-pass
    path runs on it, and a second call with other inputs overwrites the first one's tiles."""
    cases = [I.make_seq(1, 1, 2, 1024, 128, 128, seed=seed, io_dtype="bf16", with_state=True,
                        with_kprev=True) for seed in (771, 772)]
    for s in cases:
        need, ref = _run(F, s, noalloc=False)
        assert need == 2 * 16 * 16384
        _same(_run(F, s, noalloc=True)[1], ref)


def test_noalloc_two_pass_beyond_the_scratch_runs_one_kernel(F):
    """Falcon-1 with 16 heads of 8704 tokens would need 34.8 MB of tiles: the call is not refused
    (that workspace is optional) and runs the single-kernel path."""
    s = I.make_seq(1, 1, 16, 8704, 128, 128, seed=773, io_dtype="bf16", with_state=True)
    need, ref = _run(F, s, noalloc=False)
    assert need == 16 * 136 * 16384 > SCRATCH_BYTES
    _same(_run(F, s, noalloc=True)[1], ref)


def test_noalloc_refuses_a_problem_beyond_the_scratch(F):
    """Sixteen heads of 65536 tokens need more than the fixed array: refused with
    FALCON_ERR_WORKSPACE, and the output buffer is left as it was."""
    B, H, T, d = 1, 16, 65536, 128
    z = lambda *sh: torch.zeros(*sh, dtype=torch.bfloat16, device="cuda")
    q, k, v = z(B, H, T, d), z(B, H, T, d), z(B, H, T, d)
    a = torch.full((B, H, T), 0.99, dtype=torch.float32, device="cuda")
    e = torch.full((B, H, T), 0.5, dtype=torch.float32, device="cuda")
    o = torch.full((B, H, T, d), 7.0, dtype=torch.bfloat16, device="cuda")
    args = F.make_args(q, k, v, a, e, rule=2, chunk=64, o=o)
    assert F.lib().falcon_workspace_size(ctypes.byref(args)) > SCRATCH_BYTES
    assert _noalloc(F)(ctypes.byref(args), None) == F.FALCON_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool(torch.all(o == 7.0))
