"""Seeded synthetic inputs for the Falcon fast-weight forward pass.

This module is the one piece shared by the CUDA path's tests/bench and the
CPU oracle's tests. It holds no arithmetic of the method itself: it only draws
random numbers, normalises keys/queries where a workload asks for it, and
rounds values to bf16 so that both sides start from identical numbers.

Generator (counter based, so any element can be drawn independently):
  * splitmix64 finaliser applied to ``base + i``, where ``base`` mixes the
    workload seed with a per-tensor stream id;
  * two 53-bit uniforms in (0, 1] per pair of normals, Box-Muller transform;
  * sigmoid(N(mu, 1)) for the gates alpha and eta.

Workloads (the five shapes the forward pass is exercised on; the pages give
none, see "Fast Weight Attention for Continual Learning", abstract: the
method is evaluated on language modelling, so these are language-model-like
head shapes with synthetic values):
  recurrent_small : Falcon-1, fp32, B1 H2 T256 d32, seed 0
  chunk_f1        : Falcon-1, bf16, B8 H16 T4096 d128, chunk 64, seed 1
  chunk_f1a_long  : Falcon-1A, bf16, B1 H16 T32768 d128, chunk 64, seed 2
  chunk_f3        : Falcon-3 (w=4), bf16, B4 H16 T8192 d128, chunk 64, seed 3
  decode          : Falcon-1 decode, 256 seq x 32 heads, S 128x128, seed 4
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
import math
import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, stream: int) -> np.uint64:
    s = np.array([(seed * 1_000_003 + stream) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(s * _GOLDEN + _GOLDEN)[0]


def uniform01(seed: int, stream: int, n: int) -> np.ndarray:
    """n uniforms in (0, 1], float64, element i = f(seed, stream, i)."""
    base = _stream_base(seed, stream)
    i = np.arange(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(base + i * _GOLDEN)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)


def _normal_block(base, p0, p1, n, out):
    i = np.arange(2 * p0, 2 * p1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix(base + i * _GOLDEN)
    u = ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * math.pi * u2
    pair = np.empty(2 * (p1 - p0), dtype=np.float64)
    pair[0::2] = r * np.cos(th)
    pair[1::2] = r * np.sin(th)
    lo = 2 * p0
    hi = min(n, 2 * p1)
    out[lo:hi] = pair[: hi - lo]


def normal(seed: int, stream: int, n: int, chunk: int = 1 << 21) -> np.ndarray:
    """n standard normals (float32) by Box-Muller on pairs of uniforms. Element i
    depends only on (seed, stream, i); blocks are drawn on host threads."""
    out = np.empty(n, dtype=np.float32)
    npair = (n + 1) // 2
    base = _stream_base(seed, stream)
    blocks = [(p0, min(npair, p0 + chunk)) for p0 in range(0, npair, chunk)]
    if len(blocks) <= 1:
        for p0, p1 in blocks:
            _normal_block(base, p0, p1, n, out)
        return out
    with ThreadPoolExecutor(max_workers=min(len(blocks), os.cpu_count() or 1)) as ex:
        list(ex.map(lambda b: _normal_block(base, b[0], b[1], n, out), blocks))
    return out


def sigmoid_normal(seed: int, stream: int, n: int, mu: float) -> np.ndarray:
    z = normal(seed, stream, n).astype(np.float64) + mu
    return (1.0 / (1.0 + np.exp(-z))).astype(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    # finite values cannot carry out of 32 bits (largest finite pattern 0xFF7FFFFF)
    out = ((b + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).view(np.float32)
    return np.where(np.isnan(x), x, out).reshape(x.shape)


def l2_normalise_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    n = np.where(n > 0, n, 1.0)
    return (x / n).astype(np.float32)


RULE_1, RULE_1A, RULE_3, RULE_3A, RULE_2, RULE_2A = 1, 2, 3, 4, 5, 6
RULE_NAMES = {RULE_1: "falcon1", RULE_1A: "falcon1a", RULE_3: "falcon3", RULE_3A: "falcon3a",
              RULE_2: "falcon2", RULE_2A: "falcon2a"}


@dataclass
class SeqInputs:
    """One forward-pass problem. Arrays are float32 (bf16-representable when
    ``io_dtype == 'bf16'``); layout (B,H,T,d) and (B,H,T) for the gates."""
    rule: int
    io_dtype: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    alpha: np.ndarray
    eta: np.ndarray
    eps: float
    window: int = 1
    chunk: int = 64
    S0: np.ndarray | None = None
    k_prev: np.ndarray | None = None
    name: str = ""
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, H, T, dk = self.k.shape
        return B, H, T, dk, self.v.shape[-1]


def make_seq(rule: int, B: int, H: int, T: int, dk: int, dv: int, *, seed: int,
             io_dtype: str = "bf16", normalise_qk: bool = True, alpha_mu: float = 4.0,
             eta_mu: float = 0.0, eps: float = 1e-6, window: int = 1, chunk: int = 64,
             with_state: bool = False, with_kprev: bool = False, name: str = "") -> SeqInputs:
    """Draw one problem. Stream ids: q=1, k=2, v=3, alpha=4, eta=5, S0=6, k_prev=7."""
    q = normal(seed, 1, B * H * T * dk).reshape(B, H, T, dk)
    k = normal(seed, 2, B * H * T * dk).reshape(B, H, T, dk)
    v = normal(seed, 3, B * H * T * dv).reshape(B, H, T, dv)
    if normalise_qk:
        q = l2_normalise_rows(q)
        k = l2_normalise_rows(k)
    alpha = sigmoid_normal(seed, 4, B * H * T, alpha_mu).reshape(B, H, T)
    eta = sigmoid_normal(seed, 5, B * H * T, eta_mu).reshape(B, H, T)
    S0 = None
    kp = None
    if with_state:
        S0 = (normal(seed, 6, B * H * dv * dk) / math.sqrt(dk)).astype(np.float32).reshape(B, H, dv, dk)
    if with_kprev:
        kp = normal(seed, 7, B * H * dk).reshape(B, H, dk)
        if normalise_qk:
            kp = l2_normalise_rows(kp)
    if io_dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
        if kp is not None:
            kp = round_bf16(kp)
    return SeqInputs(rule=rule, io_dtype=io_dtype, q=q, k=k, v=v, alpha=alpha, eta=eta,
                     eps=eps, window=window, chunk=chunk, S0=S0, k_prev=kp, name=name)


# ---- the five workloads ---------------------------------------------------

def workload_recurrent_small(T: int = 256) -> SeqInputs:
    """Falcon-1 recurrent, fp32: B1 H2 T256 d32; q,k,v ~ N(0,1); alpha = sigmoid(N(3,1));
    eta = sigmoid(N(0,1)); eps 1e-6; x_1 = 0; seed 0."""
    return make_seq(RULE_1, 1, 2, T, 32, 32, seed=0, io_dtype="f32", normalise_qk=False,
                    alpha_mu=3.0, name="falcon1_recurrent_f32_B1H2T256d32")


def workload_chunk_f1(B=8, H=16, T=4096, d=128) -> SeqInputs:
    """Falcon-1 chunk-parallel, bf16 q/k/v, fp32 state: B8 H16 T4096 d128, chunk 64; q,k
    L2-normalised; alpha = sigmoid(N(4,1)); eta = sigmoid(N(0,1)); eps 1e-6; seed 1."""
    return make_seq(RULE_1, B, H, T, d, d, seed=1, io_dtype="bf16", normalise_qk=True,
                    alpha_mu=4.0, chunk=64, name=f"falcon1_chunk_bf16_B{B}H{H}T{T}d{d}")


def workload_chunk_f1a_long(B=1, H=16, T=32768, d=128) -> SeqInputs:
    """Falcon-1A chunk-parallel, bf16: B1 H16 T32768 d128, chunk 64; q,k,v ~ N(0,1)
    (the first workload's distributions), alpha = sigmoid(N(6,1)); seed 2."""
    return make_seq(RULE_1A, B, H, T, d, d, seed=2, io_dtype="bf16", normalise_qk=False,
                    alpha_mu=6.0, chunk=64, name=f"falcon1a_chunk_bf16_B{B}H{H}T{T}d{d}")


def workload_chunk_f3(B=4, H=16, T=8192, d=128, window=4) -> SeqInputs:
    """Falcon-3 (w=4) chunk-parallel, bf16: B4 H16 T8192 d128, chunk 64; q,k L2-normalised;
    alpha = sigmoid(N(4,1)); eta = sigmoid(N(0,1)); seed 3."""
    return make_seq(RULE_3, B, H, T, d, d, seed=3, io_dtype="bf16", normalise_qk=True,
                    alpha_mu=4.0, window=window, chunk=64,
                    name=f"falcon3_w{window}_chunk_bf16_B{B}H{H}T{T}d{d}")


@dataclass
class DecodeInputs:
    rule: int
    S: np.ndarray        # (N,H,dv,dk) float32
    k_prev: np.ndarray   # (N,H,dk) bf16-representable float32
    q: np.ndarray        # (P,N,H,dk) P distinct token inputs, cycled over steps
    k: np.ndarray
    v: np.ndarray        # (P,N,H,dv)
    alpha: np.ndarray    # (P,N,H)
    eta: np.ndarray
    eps: float = 1e-6


def workload_decode(N=256, H=32, d=128, P=4, seed=4, rule=RULE_1) -> DecodeInputs:
    """Falcon-1 decode: N sequences x H heads, fp32 S (d x d) ~ N(0,1)/sqrt(d); k_prev and
    per-step k L2-normalised; q, v ~ N(0,1); alpha = sigmoid(N(4,1)); eta = sigmoid(N(0,1));
    bf16 token inputs; P distinct token inputs that the steps cycle through."""
    S = (normal(seed, 6, N * H * d * d) / math.sqrt(d)).astype(np.float32).reshape(N, H, d, d)
    kp = round_bf16(l2_normalise_rows(normal(seed, 7, N * H * d).reshape(N, H, d)))
    q = round_bf16(normal(seed, 1, P * N * H * d).reshape(P, N, H, d))
    k = round_bf16(l2_normalise_rows(normal(seed, 2, P * N * H * d).reshape(P, N, H, d)))
    v = round_bf16(normal(seed, 3, P * N * H * d).reshape(P, N, H, d))
    a = sigmoid_normal(seed, 4, P * N * H, 4.0).reshape(P, N, H)
    e = sigmoid_normal(seed, 5, P * N * H, 0.0).reshape(P, N, H)
    return DecodeInputs(rule=rule, S=S, k_prev=kp, q=q, k=k, v=v, alpha=a, eta=e)
