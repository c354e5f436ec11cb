"""GPU parity: the CUDA library (through its C ABI) against the fp64 CPU oracle,
element by element on the same seeded inputs.

Tolerance (max |gpu - oracle| / max |oracle|): 1e-4 for fp32 inputs (the recurrent
and decode paths, fp32 arithmetic), 2e-2 for bf16 inputs with an fp32 state. The
chunk-parallel path takes bf16 inputs only (its tensor-core operands are the bf16
inputs themselves) and refuses fp32 ones, so no fp32 input is ever held to 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_falcon_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
RULE_NAMES = {1: "falcon1", 2: "falcon1a", 3: "falcon3", 4: "falcon3a"}


@pytest.fixture(scope="module")
def F(cuda_ok):
    from delta_rule_linear_falcon_b200 import build, falcon
    build.build()
    falcon.lib()
    return falcon


def dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(dtype)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def relerr(a, b):
    den = float(np.max(np.abs(b)))
    return float(np.max(np.abs(a - b))) / (den if den > 0 else 1.0)


def run_gpu(F, s: I.SeqInputs, form="chunk", chunk=None, want_state=True):
    dt = torch.bfloat16 if s.io_dtype == "bf16" else torch.float32
    q, k, v = dev(s.q, dt), dev(s.k, dt), dev(s.v, dt)
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    S0 = dev(s.S0, torch.float32) if s.S0 is not None else None
    kp = dev(s.k_prev, dt) if s.k_prev is not None else None
    if form == "chunk":
        o, S, kl = F.falcon_fwd_chunk(q, k, v, a, e, rule=s.rule, eps=s.eps, window=s.window,
                                      chunk=chunk or s.chunk, S0=S0, k_prev=kp, want_state=want_state)
    else:
        o, S, kl = F.falcon_fwd_recurrent(q, k, v, a, e, rule=s.rule, eps=s.eps, window=s.window,
                                          S0=S0, k_prev=kp, want_state=want_state)
    torch.cuda.synchronize()
    assert F.falcon_check_device_errors() == F.FALCON_OK
    return host(o), (host(S) if S is not None else None), (host(kl) if kl is not None else None)


def run_oracle(s: I.SeqInputs, heads=None):
    sl = (slice(None), slice(None)) if heads is None else heads
    take = lambda x: None if x is None else x[sl]
    return oracle.recurrent(s.rule, take(s.q), take(s.k), take(s.v), take(s.alpha), take(s.eta),
                            s.eps, s.window, S0=take(s.S0), k_prev=take(s.k_prev))


def check(s, got, ref, tol, heads=None):
    o, S, kl = got
    o_r, S_r, kl_r = ref
    if heads is not None:
        o, S, kl = o[heads], S[heads], kl[heads]
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    eo, eS = relerr(o, o_r), relerr(S, S_r)
    assert eo <= tol, f"o rel err {eo:.3e} > {tol}"
    assert eS <= tol, f"S rel err {eS:.3e} > {tol}"
    assert np.array_equal(kl, kl_r.astype(np.float32).astype(np.float64)), "k_last"
    return eo, eS


# ------------------------------------------------------------------ recurrent path

def test_recurrent_small_fp32_workload(F):
    """Falcon-1 recurrent, fp32, B1 H2 T256 d32, seed 0: the fp32 tolerance."""
    s = I.workload_recurrent_small()
    check(s, run_gpu(F, s, "recurrent"), run_oracle(s), TOL_F32)


@pytest.mark.parametrize("rule,w", [(1, 1), (2, 1), (3, 4), (4, 3), (3, 1)])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 48), (128, 128), (17, 5)])
def test_recurrent_rules(F, rule, w, io, dk, dv):
    s = I.make_seq(rule, 2, 2, 77, dk, dv, seed=11 + rule, io_dtype=io, window=w,
                   with_state=True, with_kprev=True)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    got = run_gpu(F, s, "recurrent")
    ref = run_oracle(s)
    if io == "bf16":  # o is rounded to bf16 on output; the state stays fp32
        assert relerr(got[1], ref[1]) <= TOL_F32
    check(s, got, ref, tol)


# ------------------------------------------------------------------ chunk path, small shapes

@pytest.mark.parametrize("rule,w", [(1, 1), (2, 1), (3, 4), (4, 4), (3, 2), (3, 3)])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_chunk_parity_small(F, rule, w, d, chunk):
    """Several blocks and a ragged tail (T = 3 * 64 + 9), an initial state and a cached key."""
    s = I.make_seq(rule, 2, 3, 201, d, d, seed=100 + d + chunk, io_dtype="bf16", window=w,
                   chunk=chunk, with_state=True, with_kprev=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


@pytest.mark.parametrize("dk,dv", [(128, 32), (64, 128), (32, 64), (128, 64)])
def test_chunk_mixed_widths(F, dk, dv):
    s = I.make_seq(1, 1, 5, 150, dk, dv, seed=7, io_dtype="bf16", with_state=True)
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


@pytest.mark.parametrize("rule,d", [(1, 128), (2, 128), (3, 64)])
def test_chunk_refuses_fp32_io(F, rule, d):
    """fp32 I/O is refused by the chunk path (its bf16 tensor-core operands could not meet the
    fp32 error bound) before anything is launched; the recurrent path serves fp32 at 1e-4."""
    s = I.make_seq(rule, 2, 4, 300, d, d, seed=8, io_dtype="f32", window=2 if rule == 3 else 1,
                   with_state=True, with_kprev=True)
    with pytest.raises(F.FalconError) as ei:
        run_gpu(F, s, "chunk")
    assert ei.value.status == F.FALCON_ERR_UNSUPPORTED
    check(s, run_gpu(F, s, "recurrent"), run_oracle(s), TOL_F32)


@pytest.mark.parametrize("T", [0, 1, 2, 63, 64, 65])
def test_chunk_edge_lengths(F, T):
    s = I.make_seq(1, 2, 2, T, 64, 64, seed=9, io_dtype="bf16", with_state=True, with_kprev=True)
    if T == 0:
        o, S, kl = run_gpu(F, s, "chunk")
        assert o.size == 0
        np.testing.assert_array_equal(S, s.S0)
        np.testing.assert_array_equal(kl, s.k_prev)
        return
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


def test_chunk_decay_only_and_zero_keys(F):
    """eta = 0: the state only decays. Zero keys with eps = 0 write nothing (beta = 0)."""
    s = I.make_seq(1, 1, 4, 130, 128, 128, seed=12, io_dtype="bf16", with_state=True)
    s.eta[:] = 0.0
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)
    s2 = I.make_seq(1, 1, 4, 130, 128, 128, seed=13, io_dtype="bf16", with_state=True, eps=0.0)
    s2.k[:, :, ::5] = 0.0
    got = run_gpu(F, s2, "chunk")
    assert np.all(np.isfinite(got[0]))
    check(s2, got, run_oracle(s2), TOL_BF16)


def test_chunk_strong_and_tiny_decay(F):
    """alpha down to 1e-30 and alpha = 1 runs: every decay factor stays in (0, 1]."""
    s = I.make_seq(1, 1, 4, 257, 128, 128, seed=14, io_dtype="bf16", with_state=True)
    s.alpha[..., ::9] = 1e-30
    s.alpha[..., 100:140] = 1.0
    check(s, run_gpu(F, s, "chunk"), run_oracle(s), TOL_BF16)


def test_chunk_segment_split(F):
    """fwd(T) == fwd(T1) then fwd(T - T1) from (S_out, k_last), on the GPU."""
    s = I.make_seq(1, 2, 3, 300, 128, 128, seed=15, io_dtype="bf16")
    full = run_gpu(F, s, "chunk")
    T1 = 100
    a = I.SeqInputs(1, "bf16", s.q[:, :, :T1], s.k[:, :, :T1], s.v[:, :, :T1], s.alpha[:, :, :T1],
                    s.eta[:, :, :T1], s.eps)
    ga = run_gpu(F, a, "chunk")
    b = I.SeqInputs(1, "bf16", s.q[:, :, T1:], s.k[:, :, T1:], s.v[:, :, T1:], s.alpha[:, :, T1:],
                    s.eta[:, :, T1:], s.eps, S0=ga[1].astype(np.float32), k_prev=ga[2].astype(np.float32))
    gb = run_gpu(F, b, "chunk")
    o_split = np.concatenate([ga[0], gb[0]], axis=2)
    assert relerr(o_split, full[0]) < TOL_BF16 and relerr(gb[1], full[1]) < TOL_BF16
    assert np.array_equal(gb[2], full[2])


def test_chunk_guard_bands_untouched(F):
    """Outputs written exactly in place: NaN sentinels around o and S_out stay intact."""
    s = I.make_seq(1, 2, 3, 150, 128, 64, seed=16, io_dtype="bf16")
    q, k, v = dev(s.q, torch.bfloat16), dev(s.k, torch.bfloat16), dev(s.v, torch.bfloat16)
    a, e = dev(s.alpha, torch.float32), dev(s.eta, torch.float32)
    G = 4096
    n_o = q.shape[0] * q.shape[1] * q.shape[2] * 64
    ob = torch.full((n_o + 2 * G,), float("nan"), dtype=torch.bfloat16, device="cuda")
    n_s = 2 * 3 * 64 * 128
    sb = torch.full((n_s + 2 * G,), float("nan"), dtype=torch.float32, device="cuda")
    o = ob[G:G + n_o].view(2, 3, 150, 64)
    S = sb[G:G + n_s].view(2, 3, 64, 128)
    F.falcon_fwd_chunk(q, k, v, a, e, rule=1, eps=s.eps, o=o, S_out=S)
    torch.cuda.synchronize()
    assert torch.isnan(ob[:G].float()).all() and torch.isnan(ob[G + n_o:].float()).all()
    assert torch.isnan(sb[:G]).all() and torch.isnan(sb[G + n_s:]).all()
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()


# ------------------------------------------------------------------ full-size workloads

def _spread_heads(B, H, n=16):
    """n distinct (b, h) pairs spread over the batch and the heads (so over CTAs and SMs)."""
    pairs, i = [], 0
    while len(pairs) < min(n, B * H):
        bh = (i * 37 + 5) % (B * H)
        if (bh // H, bh % H) not in pairs:
            pairs.append((bh // H, bh % H))
        i += 1
    return pairs


def _gather(s: I.SeqInputs, pairs):
    """The sampled heads of a workload as one (1, n, ...) problem, so that the oracle runs them
    in one call (OpenMP over heads)."""
    b = np.array([p[0] for p in pairs])
    h = np.array([p[1] for p in pairs])
    take = lambda x: None if x is None else np.ascontiguousarray(x[b, h][None])
    return I.SeqInputs(s.rule, s.io_dtype, take(s.q), take(s.k), take(s.v), take(s.alpha), take(s.eta),
                       s.eps, window=s.window, chunk=s.chunk, S0=take(s.S0), k_prev=take(s.k_prev))


def _check_full(name):
    s = _full(name)
    o, S, kl = _full_gpu(name)
    B, H = s.q.shape[:2]
    pairs = _spread_heads(B, H)
    b = np.array([p[0] for p in pairs])
    h = np.array([p[1] for p in pairs])
    g = _gather(s, pairs)
    return check(g, (o[b, h][None], S[b, h][None], kl[b, h][None]), run_oracle(g), TOL_BF16)


def test_full_falcon1_chunk_workload(F):
    """Falcon-1 chunk-parallel at full size (B8 H16 T4096 d128, chunk 64), 16 heads spread over
    the batch and the heads."""
    _check_full("f1")


def test_full_falcon1a_long_workload(F):
    """Falcon-1A at full size (B1 H16 T32768 d128): long-range decay renormalisation, all 16 heads."""
    _check_full("f1a")


def test_full_falcon3_workload(F):
    """Falcon-3 (w = 4) at full size (B4 H16 T8192 d128), 16 sampled heads."""
    _check_full("f3")


def test_full_falcon3a_workload(F):
    """Falcon-3A (w = 4) at full size (B4 H16 T8192 d128, the Falcon-3 inputs), 16 sampled heads."""
    _check_full("f3a")


_FULL = {}


def _full(name):
    if name not in _FULL:
        if name == "f3a":
            s = I.workload_chunk_f3()
            s.rule = I.RULE_3A
            _FULL[name] = s
        else:
            _FULL[name] = {"f1": I.workload_chunk_f1, "f1a": I.workload_chunk_f1a_long,
                           "f3": I.workload_chunk_f3}[name]()
    return _FULL[name]


_FULL_OUT = {}


def _full_gpu(name):
    import delta_rule_linear_falcon_b200.falcon as F
    if name not in _FULL_OUT:
        _FULL_OUT.clear()   # one full-size result on the device at a time
        _FULL_OUT[name] = run_gpu(F, _full(name), "chunk")
    return _FULL_OUT[name]


# ------------------------------------------------------------------ decode

def _decode_dev(d: I.DecodeInputs, p):
    return (dev(d.q[p], torch.bfloat16), dev(d.k[p], torch.bfloat16), dev(d.v[p], torch.bfloat16),
            dev(d.alpha[p], torch.float32), dev(d.eta[p], torch.float32))


@pytest.mark.parametrize("rule", [1, 2])
def test_decode_full_workload_steps(F, rule):
    """Decode workload (256 sequences x 32 heads, 128x128 fp32 state): three steps in place,
    every head compared with the oracle's single-token recurrence."""
    d = I.workload_decode(rule=rule)
    S = dev(d.S, torch.float32)
    kp = dev(d.k_prev, torch.bfloat16)
    S_ref = d.S.astype(np.float64)
    kp_ref = d.k_prev.astype(np.float64)
    for step in range(3):
        p = step % d.q.shape[0]
        q, k, v, a, e = _decode_dev(d, p)
        o = F.falcon_decode_step(S, kp, q, k, v, a, e, rule=rule, eps=d.eps)
        torch.cuda.synchronize()
        o_ref, S_ref, kp_ref = oracle.decode_step(rule, S_ref, kp_ref, d.q[p], d.k[p], d.v[p],
                                                  d.alpha[p], d.eta[p], d.eps)
        assert relerr(host(o), o_ref) <= TOL_BF16
        assert relerr(host(S), S_ref) <= TOL_F32      # fp32 state, fp32 arithmetic
        assert np.array_equal(host(kp), kp_ref)
    assert F.falcon_check_device_errors() == F.FALCON_OK


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 100), (128, 256), (128, 8)])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_shapes_match_recurrence(F, dk, dv, io):
    """T decode steps == the oracle recurrence over the same T tokens (x_1 = k_prev)."""
    s = I.make_seq(1, 3, 2, 12, dk, dv, seed=21, io_dtype=io, with_state=True, with_kprev=True)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    S = dev(s.S0, torch.float32)
    kp = dev(s.k_prev, dt)
    outs = []
    for t in range(12):
        o = F.falcon_decode_step(S, kp, dev(s.q[:, :, t], dt), dev(s.k[:, :, t], dt),
                                 dev(s.v[:, :, t], dt), dev(s.alpha[:, :, t], torch.float32),
                                 dev(s.eta[:, :, t], torch.float32), rule=1, eps=s.eps)
        outs.append(host(o))
    torch.cuda.synchronize()
    o_r, S_r, kl_r = run_oracle(s)
    tol = TOL_F32 if io == "f32" else TOL_BF16
    assert relerr(np.stack(outs, axis=2), o_r) <= tol
    assert relerr(host(S), S_r) <= TOL_F32
    assert np.array_equal(host(kp), kl_r)


def test_decode_equals_gpu_recurrent(F):
    """Repeated GPU decode steps reproduce the GPU recurrent form (fp32)."""
    s = I.make_seq(2, 2, 2, 20, 128, 128, seed=22, io_dtype="f32", with_state=True, with_kprev=True)
    rec = run_gpu(F, s, "recurrent")
    S = dev(s.S0, torch.float32)
    kp = dev(s.k_prev, torch.float32)
    outs = []
    for t in range(20):
        outs.append(host(F.falcon_decode_step(S, kp, dev(s.q[:, :, t], torch.float32),
                                              dev(s.k[:, :, t], torch.float32),
                                              dev(s.v[:, :, t], torch.float32),
                                              dev(s.alpha[:, :, t], torch.float32),
                                              dev(s.eta[:, :, t], torch.float32), rule=2, eps=s.eps)))
    torch.cuda.synchronize()
    assert relerr(np.stack(outs, axis=2), rec[0]) < 1e-5
    assert relerr(host(S), rec[1]) < 1e-5
