"""ctypes front end of the fp64 C oracle (falcon_oracle.c) -- TEST INFRASTRUCTURE ONLY.

Compiles ``falcon_oracle.c`` with gcc (OpenMP over heads) into
``oracle/_build/libfalcon_oracle.so`` on first use and exposes numpy-level
functions. Inputs may be float32 (for example bf16-rounded values); they are
widened to float64 exactly before the call.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

RULE_1, RULE_1A, RULE_3, RULE_3A, RULE_2, RULE_2A = 1, 2, 3, 4, 5, 6
SAME_STEP = 0x100  # flag OR-ed into a rule: pair (k_t, v_t) at step t (same-step association)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "falcon_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libfalcon_oracle.so")
_lock = threading.Lock()
_lib = None


def oracle_lib_path() -> str:
    return _LIB


def build_oracle(force: bool = False) -> str:
    """Compile the oracle shared library (gcc -O2 -fopenmp)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build_oracle()
            lib = ctypes.CDLL(_LIB)
            D = ctypes.POINTER(ctypes.c_double)
            I = ctypes.c_int
            common = [I, I, I, I, I, I, D, D, D, D, D, ctypes.c_double, I]
            lib.falcon_oracle_recurrent.argtypes = common + [D, D, D, D, D, I]
            lib.falcon_oracle_recurrent.restype = I
            lib.falcon_oracle_chunk.argtypes = common + [I, D, D, D, D, D, I]
            lib.falcon_oracle_chunk.restype = I
            lib.falcon_oracle_masked.argtypes = common + [D, D, D, D, D, I]
            lib.falcon_oracle_masked.restype = I
            lib.falcon_oracle_backward.argtypes = common[:12] + [I, D, D, D, D, D, D, D, D, D, D, D, I]
            lib.falcon_oracle_backward.restype = I
            lib.falcon_oracle_f2.argtypes = [I, I, I, I, I, I, D, D, D, D, D, ctypes.c_double, I,
                                             D, D, D, D, D, D, D, I]
            lib.falcon_oracle_f2.restype = I
            lib.falcon_oracle_max_threads.argtypes = []
            lib.falcon_oracle_max_threads.restype = I
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().falcon_oracle_max_threads())


def _d(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(q, k, v, alpha, eta, S0, k_prev):
    q, k, v, alpha, eta = (_d(x) for x in (q, k, v, alpha, eta))
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    assert q.shape == (B, H, T, dk) and v.shape == (B, H, T, dv)
    assert alpha.shape == (B, H, T) and eta.shape == (B, H, T)
    S0 = _d(S0)
    k_prev = _d(k_prev)
    if S0 is not None:
        assert S0.shape == (B, H, dv, dk)
    if k_prev is not None:
        assert k_prev.shape == (B, H, dk)
    return q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv)


def _outs(B, H, T, dk, dv):
    return (np.zeros((B, H, T, dv)), np.zeros((B, H, dv, dk)), np.zeros((B, H, dk)))


def recurrent(rule, q, k, v, alpha, eta, eps, window=1, S0=None, k_prev=None, threads=None):
    """Literal per-token recurrence. Returns (o, S_out, k_last) as float64."""
    lib = _load()
    q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv) = _prep(q, k, v, alpha, eta, S0, k_prev)
    o, S, kl = _outs(B, H, T, dk, dv)
    rc = lib.falcon_oracle_recurrent(int(rule), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(alpha), _ptr(eta), float(eps), int(window), _ptr(S0),
                                     _ptr(k_prev), _ptr(o), _ptr(S), _ptr(kl),
                                     int(threads or max_threads()))
    if rc != 0:
        raise ValueError(f"oracle recurrent failed: {rc}")
    return o, S, kl


def chunk(rule, q, k, v, alpha, eta, eps, window=1, chunk=64, S0=None, k_prev=None, threads=None):
    """Chunk-parallel form with block-local cumulative log decay."""
    lib = _load()
    q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv) = _prep(q, k, v, alpha, eta, S0, k_prev)
    o, S, kl = _outs(B, H, T, dk, dv)
    rc = lib.falcon_oracle_chunk(int(rule), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(alpha), _ptr(eta), float(eps), int(window), int(chunk),
                                 _ptr(S0), _ptr(k_prev), _ptr(o), _ptr(S), _ptr(kl),
                                 int(threads or max_threads()))
    if rc != 0:
        raise ValueError(f"oracle chunk failed: {rc}")
    return o, S, kl


def masked(rule, q, k, v, alpha, eta, eps, window=1, S0=None, k_prev=None, threads=None):
    """Masked-parallel form: one block spanning the whole sequence."""
    lib = _load()
    q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv) = _prep(q, k, v, alpha, eta, S0, k_prev)
    o, S, kl = _outs(B, H, T, dk, dv)
    rc = lib.falcon_oracle_masked(int(rule), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(alpha), _ptr(eta), float(eps), int(window), _ptr(S0),
                                  _ptr(k_prev), _ptr(o), _ptr(S), _ptr(kl),
                                  int(threads or max_threads()))
    if rc != 0:
        raise ValueError(f"oracle masked failed: {rc}")
    return o, S, kl


def decode_step(rule, S, k_prev, q, k, v, alpha, eta, eps, threads=None):
    """One token of the recurrence per (sequence, head): x = k_prev, y = v, then the
    cache key becomes k. Shapes: S (N,H,dv,dk), k_prev/q/k (N,H,dk), v (N,H,dv),
    alpha/eta (N,H). Returns (o (N,H,dv), S_new, k_prev_new)."""
    S = _d(S)
    N, H, dv, dk = S.shape
    o, S_new, kl = recurrent(rule, _d(q)[:, :, None, :], _d(k)[:, :, None, :],
                             _d(v)[:, :, None, :], _d(alpha)[:, :, None], _d(eta)[:, :, None],
                             eps, 1, S0=S, k_prev=k_prev, threads=threads)
    return o[:, :, 0, :], S_new, kl


def backward(rule, q, k, v, alpha, eta, eps, dO, dS_T=None, window=1, S0=None, k_prev=None, threads=None):
    """Gradients of the recurrent form (reverse mode through the literal recurrence) for upstream
    gradients dO (B,H,T,dv) of the outputs and dS_T (B,H,dv,dk) of the final state. Returns a dict
    with dq, dk, dv, dalpha, deta, dS0 and dk_prev (None when k_prev is None)."""
    lib = _load()
    q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv) = _prep(q, k, v, alpha, eta, S0, k_prev)
    dO = _d(dO)
    dS_T = _d(dS_T)
    assert dO.shape == (B, H, T, dv)
    out = {"dq": np.zeros((B, H, T, dk)), "dk": np.zeros((B, H, T, dk)), "dv": np.zeros((B, H, T, dv)),
           "dalpha": np.zeros((B, H, T)), "deta": np.zeros((B, H, T)), "dS0": np.zeros((B, H, dv, dk)),
           "dk_prev": np.zeros((B, H, dk)) if k_prev is not None else None}
    rc = lib.falcon_oracle_backward(int(rule), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                    _ptr(eta), float(eps), int(window), _ptr(S0), _ptr(k_prev), _ptr(dO),
                                    _ptr(dS_T), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                    _ptr(out["dalpha"]), _ptr(out["deta"]), _ptr(out["dS0"]),
                                    _ptr(out["dk_prev"]), int(threads or max_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle backward failed ({rc})")
    return out


def falcon2(rule, q, k, v, alpha, eta, eps, chunk=0, S0=None, k_prev=None, n0=None, threads=None):
    """Falcon-2 / Falcon-2A (rule 5 / 6, optionally | SAME_STEP): chunk = 0 runs the literal
    recurrence, chunk >= 1 the blocked form. Returns (o, S_out, k_last, n_out) as float64, n_out
    being the running per-column key energies that a continuation starts from."""
    lib = _load()
    q, k, v, alpha, eta, S0, k_prev, (B, H, T, dk, dv) = _prep(q, k, v, alpha, eta, S0, k_prev)
    n0 = _d(n0)
    if n0 is not None:
        assert n0.shape == (B, H, dk)
    o, S, kl = _outs(B, H, T, dk, dv)
    n_out = np.zeros((B, H, dk))
    rc = lib.falcon_oracle_f2(int(rule), B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(eta),
                              float(eps), int(chunk), _ptr(S0), _ptr(k_prev), _ptr(n0), _ptr(o), _ptr(S),
                              _ptr(kl), _ptr(n_out), int(threads or max_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle falcon2 failed ({rc})")
    return o, S, kl, n_out
