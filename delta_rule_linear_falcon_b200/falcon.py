"""Thin ctypes binding of libfalcon (include/falcon.h), same entry-point names.

Argument marshalling only: every step of the forward pass runs in the CUDA
library. PyTorch supplies device memory and the current stream. The library
must have been built in-tree (``python -m delta_rule_linear_falcon_b200.build``);
there is no fallback, so a missing library raises at the first call.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfalcon.so")

FALCON_OK, FALCON_ERR_INVALID_ARG, FALCON_ERR_UNSUPPORTED = 0, 1, 2
FALCON_ERR_WORKSPACE, FALCON_ERR_CUDA, FALCON_ERR_TIMEOUT = 3, 4, 5
FALCON_RULE_1, FALCON_RULE_1A, FALCON_RULE_3, FALCON_RULE_3A = 1, 2, 3, 4
FALCON_RULE_2, FALCON_RULE_2A = 5, 6
FALCON_F32, FALCON_BF16 = 0, 1
FALCON_SAME_STEP = 0x100  # OR into a rule code: pair (k_t, v_t) at step t (same-step association)
RULES = {"falcon1": FALCON_RULE_1, "falcon1a": FALCON_RULE_1A, "falcon3": FALCON_RULE_3,
         "falcon3a": FALCON_RULE_3A, "falcon2": FALCON_RULE_2, "falcon2a": FALCON_RULE_2A}


class FalconError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {falcon_status_string(status)} (status {status})")
        self.status = status


class FalconArgs(ctypes.Structure):
    """Mirror of falcon_args_t."""
    _fields_ = [
        ("rule", ctypes.c_int), ("io_dtype", ctypes.c_int),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
        ("dk", ctypes.c_int), ("dv", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("eta", ctypes.c_void_p),
        ("eps", ctypes.c_float), ("window", ctypes.c_int), ("chunk", ctypes.c_int),
        ("S0", ctypes.c_void_p), ("k_prev", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("S_out", ctypes.c_void_p), ("k_last", ctypes.c_void_p),
        ("n0", ctypes.c_void_p), ("n_out", ctypes.c_void_p),
    ]


class FalconGrads(ctypes.Structure):
    """Mirror of falcon_grads_t."""
    _fields_ = [
        ("dO", ctypes.c_void_p), ("dS_T", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("dalpha", ctypes.c_void_p), ("deta", ctypes.c_void_p),
        ("dS0", ctypes.c_void_p), ("dk_prev", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libfalcon.so from the package directory (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m delta_rule_linear_falcon_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER(FalconArgs)
            vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            L.falcon_workspace_size.argtypes = [P]
            L.falcon_workspace_size.restype = ctypes.c_size_t
            L.falcon_fwd_chunk.argtypes = [P, vp, ctypes.c_size_t, vp]
            L.falcon_fwd_chunk.restype = i
            L.falcon_fwd_recurrent.argtypes = [P, vp]
            L.falcon_fwd_recurrent.restype = i
            L.falcon_bwd_workspace_size.argtypes = [P]
            L.falcon_bwd_workspace_size.restype = ctypes.c_size_t
            L.falcon_bwd_recurrent.argtypes = [P, ctypes.POINTER(FalconGrads), vp, ctypes.c_size_t, vp]
            L.falcon_bwd_recurrent.restype = i
            L.falcon_decode_step.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, f, vp, vp]
            L.falcon_decode_step.restype = i
            L.falcon_status_string.argtypes = [i]
            L.falcon_status_string.restype = ctypes.c_char_p
            L.falcon_check_device_errors.argtypes = [vp]
            L.falcon_check_device_errors.restype = i
            L.falcon_version.argtypes = []
            L.falcon_version.restype = i
            L.falcon_debug_stall_next_call.argtypes = [i, ctypes.c_longlong]
            L.falcon_debug_stall_next_call.restype = i
            _lib = L
    return _lib


def falcon_status_string(status: int) -> str:
    return lib().falcon_status_string(int(status)).decode()


def falcon_version() -> int:
    return int(lib().falcon_version())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FALCON_BF16
    if t.dtype == torch.float32:
        return FALCON_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need(t, name, dtype=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _rule_code(rule) -> int:
    """A rule name or code; FALCON_SAME_STEP may be OR-ed into a code, or a name may end in
    '+same_step'."""
    if isinstance(rule, str):
        name, _, flag = rule.partition("+")
        return RULES[name] | (FALCON_SAME_STEP if flag == "same_step" else 0)
    return int(rule)


def make_args(q, k, v, alpha, eta, *, rule, eps=1e-6, window=1, chunk=64, S0=None, k_prev=None,
              o=None, S_out=None, k_last=None, n0=None, n_out=None) -> FalconArgs:
    """Fill falcon_args_t from tensors (shapes taken from k and v)."""
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    io = _dtype_code(k)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (k_prev, "k_prev"), (k_last, "k_last")):
        _need(t, n, k.dtype)
    for t, n in ((alpha, "alpha"), (eta, "eta"), (S0, "S0"), (S_out, "S_out"), (n0, "n0"), (n_out, "n_out")):
        _need(t, n, torch.float32)
    return FalconArgs(_rule_code(rule), io, B, H, T, dk, dv, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                      alpha.data_ptr(), eta.data_ptr(), float(eps), int(window), int(chunk),
                      _ptr(S0), _ptr(k_prev), o.data_ptr() if o is not None else None,
                      _ptr(S_out), _ptr(k_last), _ptr(n0), _ptr(n_out))


def _outputs(k, v, o, S_out, k_last, want_state: bool):
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, T, dv), dtype=k.dtype, device=k.device)
    if S_out is None and want_state:
        S_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=k.device)
    if k_last is None and want_state:
        k_last = torch.empty((B, H, dk), dtype=k.dtype, device=k.device)
    return o, S_out, k_last


def falcon_workspace_size(args: FalconArgs) -> int:
    return int(lib().falcon_workspace_size(ctypes.byref(args)))


def falcon_fwd_chunk(q, k, v, alpha, eta, *, rule, eps=1e-6, window=1, chunk=64, S0=None,
                     k_prev=None, o=None, S_out=None, k_last=None, want_state=True,
                     workspace=None, stream=None):
    """Chunk-parallel forward pass. Returns (o, S_out, k_last).

    ``workspace`` is an optional contiguous CUDA tensor of at least
    ``falcon_workspace_size(args)`` bytes (nonzero where the library splits the sequence of
    an inner-product problem with few heads, and for the two-pass path of the regression
    rules, whose blocks' solved tiles it holds); when the size is nonzero and no tensor is
    given, one is allocated here with torch for the call (on the current stream, recorded
    on ``stream`` when that is another torch stream; pass your own when ``stream`` is a raw
    handle of a different stream). A smaller tensor runs the regression rules in one
    kernel."""
    o, S_out, k_last = _outputs(k, v, o, S_out, k_last, want_state)
    args = make_args(q, k, v, alpha, eta, rule=rule, eps=eps, window=window, chunk=chunk, S0=S0,
                     k_prev=k_prev, o=o, S_out=S_out, k_last=k_last)
    need = falcon_workspace_size(args)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace")
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    elif need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
        ws_ptr, ws_bytes = workspace.data_ptr(), need
        if isinstance(stream, torch.cuda.Stream):
            # the caching allocator may hand the block out again once this call returns; tie its
            # reuse to the kernels queued on the caller's stream
            workspace.record_stream(stream)
    st = lib().falcon_fwd_chunk(ctypes.byref(args), ws_ptr, ws_bytes, _stream(stream))
    if st != FALCON_OK:
        raise FalconError(st, "falcon_fwd_chunk")
    return o, S_out, k_last


def falcon_fwd_recurrent(q, k, v, alpha, eta, *, rule, eps=1e-6, window=1, S0=None, k_prev=None,
                         o=None, S_out=None, k_last=None, want_state=True, n0=None, n_out=None,
                         stream=None):
    """Recurrent forward pass (fp32 arithmetic). Returns (o, S_out, k_last); for Falcon-2/2A
    pass n_out (B, H, dk) fp32 to receive the running column energies (n0 to start from them)."""
    o, S_out, k_last = _outputs(k, v, o, S_out, k_last, want_state)
    args = make_args(q, k, v, alpha, eta, rule=rule, eps=eps, window=window, chunk=64, S0=S0,
                     k_prev=k_prev, o=o, S_out=S_out, k_last=k_last, n0=n0, n_out=n_out)
    st = lib().falcon_fwd_recurrent(ctypes.byref(args), _stream(stream))
    if st != FALCON_OK:
        raise FalconError(st, "falcon_fwd_recurrent")
    return o, S_out, k_last


def falcon_bwd_workspace_size(args: FalconArgs) -> int:
    return int(lib().falcon_bwd_workspace_size(ctypes.byref(args)))


def falcon_bwd_recurrent(q, k, v, alpha, eta, dO, *, rule, eps=1e-6, window=1, S0=None, k_prev=None,
                         dS_T=None, want_dS0=True, workspace=None, stream=None):
    """Gradients of the recurrent form for upstream gradients dO (B, H, T, dv) fp32 of the
    outputs and dS_T (B, H, dv, dk) fp32 (or None) of the final state. Returns a dict of fp32
    tensors dq, dk, dv, dalpha, deta, dS0 (None unless want_dS0) and dk_prev (None without
    k_prev). ``workspace``: a CUDA tensor of at least falcon_bwd_workspace_size(args) bytes, or
    None to allocate one here for the call."""
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    dev = k.device
    f32 = torch.float32
    _need(dO, "dO", f32)
    _need(dS_T, "dS_T", f32)
    out = {"dq": torch.empty((B, H, T, dk), dtype=f32, device=dev),
           "dk": torch.empty((B, H, T, dk), dtype=f32, device=dev),
           "dv": torch.empty((B, H, T, dv), dtype=f32, device=dev),
           "dalpha": torch.empty((B, H, T), dtype=f32, device=dev),
           "deta": torch.empty((B, H, T), dtype=f32, device=dev),
           "dS0": torch.empty((B, H, dv, dk), dtype=f32, device=dev) if want_dS0 else None,
           "dk_prev": torch.empty((B, H, dk), dtype=f32, device=dev) if k_prev is not None else None}
    args = make_args(q, k, v, alpha, eta, rule=rule, eps=eps, window=window, chunk=64, S0=S0, k_prev=k_prev)
    grads = FalconGrads(dO.data_ptr(), _ptr(dS_T), out["dq"].data_ptr(), out["dk"].data_ptr(),
                        out["dv"].data_ptr(), out["dalpha"].data_ptr(), out["deta"].data_ptr(),
                        _ptr(out["dS0"]), _ptr(out["dk_prev"]))
    need = falcon_bwd_workspace_size(args)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().falcon_bwd_recurrent(ctypes.byref(args), ctypes.byref(grads), ws_ptr, ws_bytes, _stream(stream))
    if st != FALCON_OK:
        raise FalconError(st, "falcon_bwd_recurrent")
    return out


def falcon_decode_step(S, k_prev, q, k, v, alpha, eta, *, rule="falcon1", eps=1e-6, o=None,
                       stream=None):
    """One decode token for (N, H) heads; S and k_prev are updated in place. Returns o."""
    N, H, dv, dk = S.shape
    _need(S, "S", torch.float32)
    for t, n in ((k_prev, "k_prev"), (q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(alpha, "alpha", torch.float32)
    _need(eta, "eta", torch.float32)
    if o is None:
        o = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _need(o, "o", q.dtype)
    st = lib().falcon_decode_step(_rule_code(rule), _dtype_code(q), N, H, dk, dv, S.data_ptr(),
                                  k_prev.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  alpha.data_ptr(), eta.data_ptr(), float(eps), o.data_ptr(),
                                  _stream(stream))
    if st != FALCON_OK:
        raise FalconError(st, "falcon_decode_step")
    return o


def falcon_debug_stall_next_call(block: int, wait_budget_cycles: int) -> int:
    """Test hook: the next chunk call of this thread stalls its TMA producers at ``block`` and
    gives up its waits after ``wait_budget_cycles`` SM clocks (see include/falcon.h)."""
    return int(lib().falcon_debug_stall_next_call(int(block), int(wait_budget_cycles)))


def falcon_check_device_errors(stream=None) -> int:
    return int(lib().falcon_check_device_errors(_stream(stream)))
