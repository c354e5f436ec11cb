"""Failure detection on the GPU, driven without a fault: the test hook
falcon_debug_stall_next_call makes the TMA producer of each tensor-core kernel of the next
chunk call stop loading at a given block and shortens every bounded wait of that call. A
consumer's wait then runs out; the kernel records FALCON_ERR_TIMEOUT in the device error word,
waits for its own loads in flight, frees its tensor memory and returns. Nothing here traps,
faults or spins without a bound: each wait gives up after about a millisecond.

Each case checks that the stalled call returns and the stream synchronises, that
falcon_check_device_errors reports the timeout, and that the very next normal call on the same
GPU still matches the fp64 oracle.
"""
import pytest
import torch

from delta_rule_linear_falcon_b200 import inputs as I
from test_gpu_parity import F, TOL_BF16, check, dev, run_gpu, run_oracle  # noqa: F401

pytestmark = pytest.mark.gpu

BUDGET = 2_000_000   # SM clocks a wait may take in the stalled call (about 1 ms)

CASES = {
    # Falcon-1 on the two-pass path: the solve pass completes, the chain kernel's 5th of 10 blocks
    # of 64 tokens is never loaded
    "falcon1_chunk": dict(rule=1, H=2, T=640, window=1, alpha_mu=4.0, block=4),
    # the same on the single-kernel path (a workspace too small for the two-pass tiles)
    "falcon1_single_kernel": dict(rule=1, H=2, T=640, window=1, alpha_mu=4.0, block=4, single=True),
    # the same kernel for the windowed rule: 20 blocks of 16 tokens (w = 4)
    "falcon3_chunk": dict(rule=3, H=2, T=320, window=4, alpha_mu=4.0, block=7),
    # Falcon-1A with few heads takes the sequence split: the state pass (seg_piece_kernel) and the
    # chunk kernel on the segments both stall at their third block
    "falcon1a_split": dict(rule=2, H=2, T=4096, window=1, alpha_mu=6.0, block=2),
}


def _problem(c):
    return I.make_seq(c["rule"], 1, c["H"], c["T"], 128, 128, seed=900 + c["block"], io_dtype="bf16",
                      window=c["window"], alpha_mu=c["alpha_mu"], normalise_qk=c["rule"] != 2,
                      with_state=True, with_kprev=True)


def _call(F, s, single=False):
    q, k, v = (dev(x, torch.bfloat16) for x in (s.q, s.k, s.v))
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0, kp = dev(s.S0, torch.float32), dev(s.k_prev, torch.bfloat16)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda") if single else None
    F.falcon_fwd_chunk(q, k, v, a, e, rule=s.rule, eps=s.eps, window=s.window, chunk=64, S0=S0, k_prev=kp,
                       workspace=ws)


@pytest.mark.parametrize("name", list(CASES))
def test_stalled_load_times_out_and_the_gpu_stays_usable(F, name):
    s = _problem(CASES[name])
    assert F.falcon_check_device_errors() == F.FALCON_OK
    assert F.falcon_debug_stall_next_call(CASES[name]["block"], BUDGET) == F.FALCON_OK
    _call(F, s, CASES[name].get("single", False))   # launches normally; its waits run out on the device
    torch.cuda.synchronize()         # the kernels returned
    assert F.falcon_check_device_errors() == F.FALCON_ERR_TIMEOUT
    assert F.falcon_check_device_errors() == F.FALCON_OK      # the error word was cleared
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)  # the next call is correct


def test_short_budget_without_a_stall_changes_nothing(F):
    """A stall past the last block leaves the loads alone: with the same short budget every wait
    of a normal run completes in time and the result matches the oracle."""
    c = CASES["falcon1_chunk"]
    s = _problem(c)
    assert F.falcon_debug_stall_next_call(10_000, BUDGET) == F.FALCON_OK
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)
