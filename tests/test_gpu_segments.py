"""GPU parity of the sequence split of the inner-product rule (Falcon-1A): with fewer
heads than SMs, falcon_fwd_chunk cuts each head into segments, forms every segment's
starting state from a parallel pass over pieces and a scan, and runs the segments as
heads of their own on the tensor-core chunk kernel. Compared with the fp64 oracle through
the C ABI; tolerances as in test_gpu_parity.py."""
import ctypes

import numpy as np
import pytest
import torch

from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, check, dev, host, run_gpu, run_oracle  # noqa: F401

pytestmark = pytest.mark.gpu
SS = 0x100


def _ws_bytes(F, rule, B, H, T, d=128, chunk=64, io=torch.bfloat16, window=1):
    z = lambda *s: torch.zeros(*s, dtype=io, device="cuda")
    zf = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")
    q, k, v = z(B, H, T, d), z(B, H, T, d), z(B, H, T, d)
    args = F.make_args(q, k, v, zf(B, H, T), zf(B, H, T), rule=rule, chunk=chunk, o=z(B, H, T, d),
                       window=window)
    return F.falcon_workspace_size(args)


def test_split_is_chosen_only_where_it_applies(F):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert _ws_bytes(F, 2, 1, 2, 4096) > 0                  # inner-product rule, few heads
    assert _ws_bytes(F, 2 | SS, 1, 2, 4096) > 0
    # regression rule: no split; its workspace is the two-pass path's tiles, 16 KB per block
    assert _ws_bytes(F, 1, 1, 2, 4096) == 2 * 64 * 16384
    assert _ws_bytes(F, 2, 1, 2, 4096 + 9) == 0             # ragged length
    assert _ws_bytes(F, 2, 1, 2, 448) == 0                  # too short for two segments of 8 blocks
    assert _ws_bytes(F, 2, 1, 2, 4096, chunk=32) == 0       # not the 64-token tensor-core kernel
    assert _ws_bytes(F, 2, 1, sms, 4096) == 0               # one head per SM already
    assert _ws_bytes(F, 4, 1, 2, 4096, window=4) == 0       # windowed inner-product rule: no split
    assert _ws_bytes(F, 4, 1, 2, 4096, window=2) == 0


@pytest.mark.parametrize("w", [2, 4])
def test_windowed_inner_product_with_few_heads(F, w):
    """Falcon-3A with few heads and a long sequence runs unsplit on the tensor-core kernel (the
    state pass writes one pair per token, so the split does not apply to a window)."""
    s = I.make_seq(4, 1, 2, 2048, 128, 128, seed=640 + w, io_dtype="bf16", window=w, with_state=True,
                   with_kprev=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


@pytest.mark.parametrize("T", [1024, 4096])
@pytest.mark.parametrize("same_step", [False, True])
def test_split_parity(F, T, same_step):
    """Segments of 512 tokens, an initial state and a cached key (ignored with the flag)."""
    s = I.make_seq(2 | (SS if same_step else 0), 1, 2, T, 128, 128, seed=700 + T // 64 + same_step,
                   io_dtype="bf16", normalise_qk=False, alpha_mu=6.0, with_state=True, with_kprev=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


def test_split_parity_no_state_in_or_out(F):
    """Without S0, k_prev, S_out or k_last: the last segment's pieces are skipped."""
    s = I.make_seq(2, 2, 3, 2048, 128, 128, seed=720, io_dtype="bf16", normalise_qk=False, alpha_mu=5.0)
    o, S, kl = run_gpu(F, s, "chunk", want_state=False)
    assert S is None and kl is None
    o_r, _, _ = run_oracle(s)
    assert np.all(np.isfinite(o))
    assert float(np.max(np.abs(o - o_r))) <= TOL_BF16 * float(np.max(np.abs(o_r)))


def test_split_parity_two_pieces_per_segment(F):
    """Forty heads of 8192 tokens: two segments of 4096 tokens, each of two 2048-token pieces;
    three heads compared with the oracle."""
    s = I.make_seq(2, 2, 20, 8192, 128, 128, seed=730, io_dtype="bf16", normalise_qk=False,
                   alpha_mu=6.0, with_state=True, with_kprev=True)
    assert _ws_bytes(F, 2, 2, 20, 8192) > 0
    got = run_gpu(F, s, "chunk")
    hs = (slice(0, 2), slice(3, 20, 8))
    check(s, got, run_oracle(s, hs), TOL_BF16, heads=hs)


def test_split_rejects_small_workspace(F):
    s = I.make_seq(2, 1, 2, 1024, 128, 128, seed=740, io_dtype="bf16")
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(F.FalconError) as ei:
        F.falcon_fwd_chunk(q, k, v, a, e, rule=2, eps=s.eps, workspace=ws)
    assert ei.value.status == F.FALCON_ERR_WORKSPACE
    o = torch.empty_like(v)
    args = F.make_args(q, k, v, a, e, rule=2, eps=s.eps, o=o)
    assert F.lib().falcon_fwd_chunk(ctypes.byref(args), None, 0, None) == F.FALCON_ERR_WORKSPACE


def test_split_on_a_side_stream_with_binding_workspace(F):
    """The caller's current stream is the default one and the work goes to a side stream: the
    binding allocates the workspace on the current stream and records the side stream on it,
    so blocks of the same size allocated and filled on the current stream right after the call
    cannot take the workspace while the split still runs."""
    s = I.make_seq(2, 1, 2, 1024, 128, 128, seed=750, io_dtype="bf16", normalise_qk=False,
                   alpha_mu=6.0, with_state=True, with_kprev=True)
    need = _ws_bytes(F, 2, 1, 2, 1024)
    assert need > 0
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0, kp = dev(s.S0, torch.float32), dev(s.k_prev, torch.bfloat16)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    o, S, kl = F.falcon_fwd_chunk(q, k, v, a, e, rule=2, eps=s.eps, S0=S0, k_prev=kp, stream=side)
    junk = [torch.empty(need, dtype=torch.uint8, device="cuda").fill_(0xFF) for _ in range(8)]
    side.synchronize()
    torch.cuda.synchronize()
    del junk
    assert F.falcon_check_device_errors() == F.FALCON_OK
    check(s, (host(o), host(S), host(kl)), run_oracle(s), TOL_BF16)
